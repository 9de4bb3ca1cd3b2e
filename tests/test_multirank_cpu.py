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
