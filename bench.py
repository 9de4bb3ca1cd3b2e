#!/usr/bin/env python
"""Benchmark of the NVFP4 + augmented-residual-channel prefill path on B200.

One step = the Llama-3-8B-shaped prefill projections on one token batch of M = 4096:
for each of qkv (K=4096, N=6144), o (4096, 4096), gateup (4096, 28672), down (14336, 4096):
  dynamic-scale activation quantization with r = 128 residual channels (abs-max pass, fused
  quantize + residual stash, residual tail) -> block-scaled NVFP4 GEMM of depth K + r -> bf16 Y.
Weights are packed and outlier channels calibrated once, before timing (offline steps).

Metric: NVFP4 ARC GEMM TFLOP/s = sum over the step of 2*M*N*(K+r) / step time, with the fused
activation quantizer's GB/s (read X + write codes + scale bytes) reported beside it.
Timing: CUDA events on the launching stream around every step and every kernel call; the L2 is
flushed (a 256 MiB write) before every timed step, outside the events. Multi-GPU: one process
per GPU, each rank runs the same step on its own token batch (weak scaling, no data-path
collective); time = max over ranks.

--impl reference times the CPU oracle (the plain C restatement of the method) on a bounded
row sample of the same step, on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

PROJ = [("qkv", 4096, 6144), ("o", 4096, 4096), ("gateup", 4096, 28672), ("down", 14336, 4096)]
M_TOKENS = 4096
R = 128
METRIC = "NVFP4 ARC GEMM TFLOP/s (% FP4 peak) + fused act-quant GB/s, 1×B200"
UNIT = "TFLOP/s"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)


def step_flops(M=M_TOKENS):
    return sum(2.0 * M * N * (K + R) for _, K, N in PROJ)


def quant_bytes(M=M_TOKENS):
    """Algorithmic bytes of the quantizer: read X once, write codes and scale bytes."""
    tot = 0
    for _, K, _ in PROJ:
        kp = (K + R + 63) // 64 * 64
        tot += 2 * M * K + M * kp // 2 + M * kp // 16
    return tot


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def gemm_kernel_fingerprint():
    h = hashlib.sha256()
    for f in ("arc_device.cuh", "gemm.cuh"):
        h.update(open(os.path.join(ROOT, "nvfp4_block_scaled_arc_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic():
    """Per-launch DRAM bytes of the GEMM from the committed ncu summary, if it was taken on the
    current kernel source; otherwise None."""
    p = os.path.join(ROOT, "profiles", "gemm_nvfp4_llama8b.md")
    if not os.path.exists(p):
        return None
    fp, traffic = None, None
    for line in open(p):
        if line.startswith("kernel_source_fingerprint:"):
            fp = line.split(":", 1)[1].strip()
        if line.startswith("dram_bytes_per_launch_step_avg:"):
            traffic = float(line.split(":", 1)[1].strip())
    return traffic if fp == gemm_kernel_fingerprint() else None


class ClockSampler:
    """Samples SM clock, power and clock-event reasons through NVML from a background thread
    (every ~2 ms) while the timed region runs. The device is matched by PCI bus id."""

    REASONS = (("hw_slowdown", 0x08), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x04), ("hw_power_brake_slowdown", 0x80))

    def __init__(self, device):
        self.device = device
        self.rows = []
        self.err = None
        self._stop = None

    def _handle(self, nv):
        p = torch.cuda.get_device_properties(self.device)
        bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        return nv.nvmlDeviceGetHandleByPciBusId(bus.encode())

    def __enter__(self):
        import threading

        try:
            import pynvml as nv

            nv.nvmlInit()
            self.nv = nv
            self.h = self._handle(nv)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception as e:  # no NVML: the line says so
            self.err = f"nvml unavailable: {e}"
            return self
        self._stop = threading.Event()

        def run():
            nv, h = self.nv, self.h
            while not self._stop.is_set():
                try:
                    self.rows.append((nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                      nv.nvmlDeviceGetCurrentClocksEventReasons(h),
                                      nv.nvmlDeviceGetPowerUsage(h) / 1000.0))
                except Exception as e:
                    self.err = str(e)
                    return
                time.sleep(0.002)

        self._t = threading.Thread(target=run, daemon=True)
        self._t.start()
        return self

    def __exit__(self, *a):
        if self._stop is not None:
            self._stop.set()
            self._t.join(timeout=5)

    def summary(self):
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "unsampled"]}
        seen = sorted({n for _, r, _ in self.rows for n, bit in self.REASONS if r & bit})
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": seen, "samples": len(self.rows), "power_w_max": max(r[2] for r in self.rows),
                "source": "nvml"}


# ---------------------------------------------------------------------------------------------
# Our arm
# ---------------------------------------------------------------------------------------------

def make_inputs(rank: int, device):
    import workloads as W

    xs, ws = {}, {}
    for name, K, N in PROJ:
        d = W.llama8b(name, rows=M_TOKENS, row0=rank * M_TOKENS)
        xs[name] = W.to_torch_bf16(d["x"])
        ws[name] = W.to_torch_bf16(d["w"]).to(device)
    return xs, ws


def run_ours(args, rank, world, device):
    import nvfp4_block_scaled_arc_b200 as arc

    stream = torch.cuda.Stream(device=device)
    xs_host, ws = make_inputs(rank, device)
    with torch.cuda.stream(stream):
        xs = {k: v.to(device, non_blocking=False) for k, v in xs_host.items()}
        idx, packed, qa, ys, wsp = {}, {}, {}, {}, {}
        for name, K, N in PROJ:
            idx[name] = arc.calibrate_outliers(xs[name], R, stream=stream)
            packed[name] = arc.pack_weight_nvfp4(ws[name], idx[name], stream=stream)
            qa[name] = arc.quantize_act_nvfp4(xs[name], idx[name], stream=stream)
            ys[name] = torch.empty(M_TOKENS, N, dtype=torch.bfloat16, device=device)
            wsp[name] = torch.empty(arc.quantize_workspace_bytes(M_TOKENS, R), dtype=torch.uint8, device=device)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream.synchronize()
    del ws

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    def step(rec):
        for name, K, N in PROJ:
            e0, e1, e2 = (ev(), ev(), ev()) if rec is not None else (None, None, None)
            if e0 is not None:
                e0.record(stream)
            arc.quantize_act_nvfp4(xs[name], idx[name], out=qa[name], workspace=wsp[name], stream=stream)
            if e1 is not None:
                e1.record(stream)
            arc.gemm_nvfp4(qa[name], packed[name], out=ys[name], stream=stream)
            if e2 is not None:
                e2.record(stream)
                rec.append((e0, e1, e2))

    # warm-up
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            step(None)
    stream.synchronize()
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during warm-up")

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    step_ev, kern = [], []
    barrier()
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                flush.zero_()
                s0, s1 = ev(), ev()
                s0.record(stream)
                rec = []
                step(rec)
                s1.record(stream)
                step_ev.append((s0, s1))
                kern.append(rec)
        torch.cuda.synchronize(device)
    barrier()
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the timed steps")
    step_ms = [a.elapsed_time(b) for a, b in step_ev]
    total_ms = sum(step_ms)
    q_ms = sum(r[0].elapsed_time(r[1]) for rec in kern for r in rec)
    g_ms = sum(r[1].elapsed_time(r[2]) for rec in kern for r in rec)
    per_proj = {}
    for i, (name, K, N) in enumerate(PROJ):
        gq = [rec[i][0].elapsed_time(rec[i][1]) for rec in kern]
        gg = [rec[i][1].elapsed_time(rec[i][2]) for rec in kern]
        kp = (K + R + 63) // 64 * 64
        per_proj[name] = {
            "quant_us": 1e3 * statistics.mean(gq),
            "quant_gbs": (2 * M_TOKENS * K + M_TOKENS * kp // 2 + M_TOKENS * kp // 16) / (statistics.mean(gq) * 1e-3) / 1e9,
            "gemm_us": 1e3 * statistics.mean(gg),
            "gemm_tflops": 2.0 * M_TOKENS * N * (K + R) / (statistics.mean(gg) * 1e-3) / 1e12,
        }
    clocks = clk.summary()

    # e2e through the public API with host buffers: pinned X in, Y out, every step
    xs_pin = {k: v.pin_memory() for k, v in xs_host.items()}
    ys_pin = {name: torch.empty(M_TOKENS, N, dtype=torch.bfloat16).pin_memory() for name, _, N in PROJ}
    h2d = sum(v.numel() * 2 for v in xs_pin.values())
    d2h = sum(v.numel() * 2 for v in ys_pin.values())

    def e2e_step():
        for name, K, N in PROJ:
            xs[name].copy_(xs_pin[name], non_blocking=True)
            arc.quantize_act_nvfp4(xs[name], idx[name], out=qa[name], workspace=wsp[name], stream=stream)
            arc.gemm_nvfp4(qa[name], packed[name], out=ys[name], stream=stream)
            ys_pin[name].copy_(ys[name], non_blocking=True)

    e2e_ms = float("nan")
    if not args.no_e2e:
        with torch.cuda.stream(stream):
            for _ in range(max(1, min(args.warmup, 2))):
                e2e_step()
        stream.synchronize()
        barrier()
        e2e_ev = []
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                a, b = ev(), ev()
                a.record(stream)
                e2e_step()
                b.record(stream)
                e2e_ev.append((a, b))
        stream.synchronize()
        barrier()
        e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)

    t = torch.tensor([total_ms, q_ms, g_ms, e2e_ms], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    total_ms, q_ms, g_ms, e2e_ms = t.tolist()
    return dict(total_ms=total_ms, q_ms=q_ms, g_ms=g_ms, e2e_ms=e2e_ms, per_proj=per_proj, clocks=clocks,
                h2d=h2d, d2h=d2h, launches=args.steps * len(PROJ) * 2)


# ---------------------------------------------------------------------------------------------
# Oracle arm (CPU)
# ---------------------------------------------------------------------------------------------

def oracle_sample_step(rows: int, cache: dict):
    """One bounded sample of the step on the CPU oracle: `rows` token rows of every projection
    through calibration-free quantization (idx from the full-batch calibration cached up
    front), and the FP64 GEMM of those rows against all N outputs. Returns algorithmic flops."""
    import oracle as O

    flops = 0.0
    for name, K, N in PROJ:
        c = cache[name]
        x = c["x"][:rows]
        ac, asf = O.quantize_act(x, c["idx"], c["sa"])
        O.gemm_nvfp4_f64(ac, asf, c["sa"], c["bc"], c["bsf"], c["sw"])
        flops += 2.0 * rows * N * (K + R)
    return flops


def oracle_cache(n_rows: int):
    import oracle as O
    import workloads as W

    cache = {}
    for name, K, N in PROJ:
        d = W.llama8b(name, rows=n_rows)
        idx = O.calibrate(d["x"], R)
        sa = O.tensor_scale(O.amax(d["x"]))
        sw = O.tensor_scale(O.amax(d["w"]))
        bc, bsf = O.pack_weight(d["w"], idx, sw)
        cache[name] = dict(x=d["x"], idx=idx, sa=sa, sw=sw, bc=bc, bsf=bsf)
    return cache


def cpu_baseline(rows: int | None = None):
    """The oracle on the host cores: `rows` token rows (default two per host thread, so every
    thread works) of each projection, about 10-30 s of CPU work."""
    import oracle as O

    rows = rows or 2 * O._threads()
    cache = oracle_cache(max(rows, 64))
    t0 = time.perf_counter()
    flops = oracle_sample_step(rows, cache)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": min(O._threads(), rows), "kind": "oracle",
            "sample": f"{rows} token row(s) of each of the 4 projections (quantize + FP64 GEMM against all N), "
                      f"{dt:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle as O

    rows = O._threads()  # one token row per host thread per step
    cache = oracle_cache(max(rows, 64))
    for _ in range(args.warmup):
        oracle_sample_step(rows, cache)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(rows, cache)
    dt = time.perf_counter() - t0
    v = flops / dt / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama8b-prefill-projections M=4096 r=128 (oracle on a row sample)",
                       "sample_rows_per_projection": rows},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": O._threads(), "kind": "oracle",
                             "sample": f"{rows} token rows of each of the 4 projections per step "
                                       f"(quantize + FP64 GEMM against all N)"},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--proj", default="all", help="profiling: run only this projection (qkv, o, gateup, down)")
    args = ap.parse_args()
    if args.proj != "all":
        global PROJ
        PROJ = [p for p in PROJ if p[0] == args.proj]
        if not PROJ:
            ap.error("unknown --proj")
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=180))
    try:
        res = run_ours(args, rank, world, device)
        if rank == 0:
            pk, src = peaks()
            flops = step_flops() * world
            value = flops * args.steps / (res["total_ms"] * 1e-3) / 1e12
            gemm_flops_launch = step_flops()  # all GEMM launches of a step (one rank)
            g_avg_s = res["g_ms"] * 1e-3 / args.steps
            achieved = gemm_flops_launch / g_avg_s / 1e12
            peak = pk["bf16_tflops"] * FP4_OVER_BF16
            traffic = ncu_traffic()
            line = {
                "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": res["total_ms"] / args.steps, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "e2m1 x e2m1 -> f32 (bf16 out)",
                "data": "synthetic (seeded; random weights and activations of the stated shapes)",
                "config": {"workload": "llama8b-prefill-projections: M=4096 tokens, qkv/o/gateup/down, r=128",
                           "tokens_per_gpu": M_TOKENS, "r": R, "l2": "flushed (256 MiB write) before every step",
                           "parallelism": f"replicas x{world}"},
                "quant_gbs": quant_bytes() * args.steps / (res["q_ms"] * 1e-3) / 1e9,
                "gemm_only_tflops": achieved,
                "pct_fp4_peak": 100.0 * value / peak,
                "per_projection": res["per_proj"],
                "roofline": {"bound": "tensor", "kernel": "k_gemm<nvfp4> (all 4 launches of a step)",
                             "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                             "peak_source": f"{src} bf16 burst {pk['bf16_tflops']} TFLOP/s x {FP4_OVER_BF16:g} "
                                            f"(nominal FP4/BF16 dense ratio)",
                             "traffic": traffic},
                "quant_roofline": {"bound": "hbm", "achieved": quant_bytes() * args.steps / (res["q_ms"] * 1e-3) / 1e9,
                                   "peak": pk["hbm_gbs"], "unit": "GB/s",
                                   "frac": quant_bytes() * args.steps / (res["q_ms"] * 1e-3) / 1e9 / pk["hbm_gbs"]},
                "clocks": res["clocks"],
                "e2e": None if args.no_e2e else {
                    "value": flops * args.steps / (res["e2e_ms"] * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
                "gpu_launches": res["launches"],
            }
            if not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline()
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
