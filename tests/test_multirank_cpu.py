"""The multi-rank path of the benchmark on CPU: two gloo ranks as separate processes (the
data-parallel replica scheme: every rank its own token rows, the same weights, no data-path
collective; the job's time is the slowest rank's), plus the weak-scaling value of the JSON line.
"""
import datetime
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=60))
    try:
        out = {"rank": rank, "max": bench.ranks_max([1.0 + 2 * rank, 5.0 - 3 * rank, 7.0], "cpu")}
        for workload, name in (("llama8b", "o"), ("stress", "frac0.01-r32")):
            layers, _ = bench.layer_set(workload)
            L = [l for l in layers if l["name"] == name][0]
            M = 8
            d = L["gen"](M, rank * M)
            x = torch.from_numpy(d["x"].astype(np.int32))
            xs = [torch.zeros_like(x) for _ in range(world)]
            torch.distributed.all_gather(xs, x)
            w = torch.tensor([float(np.asarray(d["w"], np.uint64).sum()), float(d["w"].shape[0])], dtype=torch.float64)
            wsum = [torch.zeros_like(w) for _ in range(world)]
            torch.distributed.all_gather(wsum, w)
            out[workload] = (torch.cat(xs).numpy().astype(np.uint16), [t.tolist() for t in wsum])
        # the replica scheme's quantization of this rank's own rows: the rank's tensor scale is the
        # amax of its own shard; with one 4-byte all-reduce(max) of the amax the ranks would share
        # the single-process scale instead
        import oracle as O

        d = W.llama8b("o", rows=M, row0=rank * M, w_rows=8)
        idx = O.calibrate(W.llama8b("o", rows=2 * M, with_w=False)["x"], 32)
        a_mine = O.amax(d["x"])
        s_mine = O.tensor_scale(a_mine)
        c_mine, sf_mine = O.quantize_act(d["x"], idx, s_mine)
        a_all = torch.tensor([a_mine], dtype=torch.float64)
        torch.distributed.all_reduce(a_all, op=torch.distributed.ReduceOp.MAX)
        s_glob = O.tensor_scale(float(a_all.item()))
        c_glob, sf_glob = O.quantize_act(d["x"], idx, s_glob)
        out["shard"] = dict(s_mine=s_mine, c_mine=c_mine, sf_mine=sf_mine, s_glob=s_glob, c_glob=c_glob,
                            sf_glob=sf_glob, idx=idx)
        bench._barrier(world)
        q.put(out)
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted((q.get(timeout=180) for _ in range(2)), key=lambda o: o["rank"])
    for p in ps:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the job's times: element-wise maximum over the ranks, on every rank
    for o in res:
        assert o["max"] == [3.0, 5.0, 7.0]
    # every rank its own rows: together they are exactly the rows one process would generate
    for workload, gen in (("llama8b", lambda: W.llama8b("o", rows=16, with_w=False)["x"]),
                          ("stress", lambda: W.stress(0.01, rows=16, w_rows=8)["x"])):
        gathered, wsums = res[0][workload]
        np.testing.assert_array_equal(gathered, gen())
        assert not np.array_equal(gathered[:8], gathered[8:])
        assert wsums[0] == wsums[1]  # the same weights on both ranks
    # each rank's codes of its own rows equal the single-process oracle on the same rows with
    # that rank's scale; with the all-reduced scale they equal the single-process quantization of
    # the whole batch, row for row
    import oracle as O

    full = W.llama8b("o", rows=16, with_w=False)["x"]
    idx = res[0]["shard"]["idx"]
    s_one = O.tensor_scale(O.amax(full))
    c_one, sf_one = O.quantize_act(full, idx, s_one)
    for o in res:
        sh, r0 = o["shard"], 8 * o["rank"]
        c_rows, sf_rows = O.quantize_act(full[r0:r0 + 8], idx, sh["s_mine"])
        np.testing.assert_array_equal(sh["c_mine"], c_rows)
        np.testing.assert_array_equal(sh["sf_mine"], sf_rows)
        assert sh["s_glob"] == s_one
        np.testing.assert_array_equal(sh["c_glob"], c_one[r0:r0 + 8])
        np.testing.assert_array_equal(sh["sf_glob"], sf_one[r0:r0 + 8])
    # the per-rank scales differ from the whole batch's on at least one rank (the replica scheme
    # does not reproduce the single-process scale bit for bit, and says so)
    assert any(o["shard"]["s_mine"] != s_one for o in res)


def test_value_is_the_whole_job_throughput():
    # weak scaling: the same per-rank step time with twice the ranks is twice the job's value
    class A:
        steps, warmup, workload, no_e2e, reorder, format = 10, 3, "llama8b", True, False, "nvfp4"

    layers, desc = bench.layer_set("llama8b")
    res = dict(total_ms=6.4, q_ms=1.2, g_ms=5.0, e2e_ms=float("nan"), per_layer={}, clocks={}, h2d=0, d2h=0,
               launches=120)
    one = bench.layers_line(A, 1, layers, desc, res)
    two = bench.layers_line(A, 2, layers, desc, res)
    assert abs(two["value"] - 2 * one["value"]) < 1e-9 * one["value"]
    assert two["n_gpus"] == 2 and two["scaling"] == "weak"
    flops = sum(bench.layer_flops(L) for L in layers)
    assert abs(one["value"] - flops * 10 / 6.4e-3 / 1e12) < 1e-9 * one["value"]


def test_bench_launcher_refuses_more_gpus_than_visible():
    # without a launcher, --gpus N starts one process per GPU; with fewer visible GPUs it refuses
    import subprocess
    import sys

    if torch.cuda.device_count() >= 2:
        return
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    p = subprocess.run([sys.executable, bench.__file__, "--gpus", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, timeout=300, env=env)
    assert p.returncode == 2
    assert "CUDA device(s) are visible" in p.stderr


def test_spawned_rank_environment(monkeypatch):
    # a spawned rank sees the rendezvous torchrun would give it
    seen = {}

    def fake_run(args, ap):
        seen.update({k: os.environ[k] for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT")})

    class A:
        gpus = 4

    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        monkeypatch.delenv(k, raising=False)
    monkeypatch.setattr(bench, "run", fake_run)
    bench._rank_main(3, A, 29555)
    assert seen == {"RANK": "3", "LOCAL_RANK": "3", "WORLD_SIZE": "4", "MASTER_ADDR": "127.0.0.1",
                    "MASTER_PORT": "29555"}
