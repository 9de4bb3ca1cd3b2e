#!/usr/bin/env python
"""Benchmark of the NVFP4 + augmented-residual-channel prefill path on B200.

Default workload (the headline): the Llama-3-8B-shaped prefill projections on one token batch of
M = 4096. One step = for each of qkv (K=4096, N=6144), o (4096, 4096), gateup (4096, 28672),
down (14336, 4096): dynamic-scale activation quantization with r = 128 residual channels
(abs-max pass, then the coding pass with the residual blocks) -> block-scaled NVFP4 GEMM of
depth K + r -> bf16 Y. Weights are packed and outlier channels calibrated once, before timing
(offline steps).

Other workloads (--workload), same timing rules:
  mlp70b     M = 16384: gate|up 8192 -> 57344, down 28672 -> 8192, r = 256
  stress     M = 2048, K = N = 4096, Student-t(3) activations, outlier fraction {0, 0.1, 1, 5} %
             x r in {0, 32, 128, 256}; also the relative error of each output against the BF16
             product (the library's own BF16 GEMM of the same inputs)
  recurrent  the shared 2-sublayer SwiGLU block (d = 2048, ffn = 8192, RMSNorm, residual add)
             applied T = 16 times to H [4096, 2048]: one prefill per k_low in {0, 8, 12, 16}
             (steps before k_low in NVFP4 + ARC with r = 64, the rest BF16); time per prefill,
             speedup against k_low = 0 and the hidden-state error against all-BF16; after the
             timed region: a schedule study at 12 of 16 NVFP4 steps (RAMP's order, BF16 first,
             interleaved, random placements), RAMP's own T = 32 / K = 24 instantiation with FP8
             W8A8 steps next to NVFP4 + ARC steps, and the placement study on a block built to
             contract (measured contraction factor; RAMP order vs Early-BF16 vs 24 random)

Variants of the linear-layer workloads:
  --reorder      channels reordered by calibration abs-max before the primary quantization
                 (the outlier set is the first r of the order); adds the error against BF16
  --format fp8   FP8 W8A8 with per-tensor scales instead of NVFP4 + ARC (metric: FP8 GEMM
                 TFLOP/s against 2 x the measured BF16 peak); adds the error against BF16
  --format mxfp4 MXFP4 with augmented residual channels (E2M1 codes, one power-of-two E8M0 scale
                 per 32 values, no tensor scale: the quantizer is one pass over X); adds the
                 error against BF16

Metric: NVFP4 ARC GEMM TFLOP/s = sum over the step of 2*M*N*(K+r) / step time, with the fused
activation quantizer's GB/s (read X + write codes + scale bytes) beside it.
Timing: CUDA events on the launching stream; two timed passes of --steps steps each, the L2
flushed before every step, outside the events (a 256 MiB buffer written, then read back, so the
lines it leaves in L2 are clean). The first pass has events around each step only and gives the
step time (value, ms_per_step): events between the kernels would add gaps of their own and keep a
kernel from starting while the one before it finishes. The second pass has events around every
kernel call and gives the per-kernel times (roofline, per_projection). Multi-GPU: one process
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

METRIC = "NVFP4 ARC GEMM TFLOP/s (% FP4 peak) + fused act-quant GB/s, 1×B200"
METRIC_FP8 = "FP8 W8A8 GEMM TFLOP/s (% FP8 peak) + act-quant GB/s, 1×B200"
METRIC_MX = "MXFP4 ARC GEMM TFLOP/s (% FP4 peak) + fused act-quant GB/s, 1×B200"
UNIT = "TFLOP/s"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor ratio (9 / 2.25 PFLOP/s)


# ---------------------------------------------------------------------------------------------
# Workloads: lists of linear layers (name, M, K, N, r, generator)
# ---------------------------------------------------------------------------------------------

def layer_set(workload: str):
    import workloads as W

    out = []
    if workload == "llama8b":
        M = W.LLAMA8B_M
        for name, (_, K, N) in W.LLAMA8B_PROJ.items():
            out.append(dict(name=name, M=M, K=K, N=N, r=W.LLAMA8B_R,
                            gen=lambda rows, row0, name=name: W.llama8b(name, rows=rows, row0=row0)))
        desc = f"llama8b-prefill-projections: M={M} tokens, qkv/o/gateup/down, r={W.LLAMA8B_R}"
    elif workload == "mlp70b":
        M = W.MLP70B_M
        for name, (_, K, N) in W.MLP70B_PROJ.items():
            out.append(dict(name=name, M=M, K=K, N=N, r=W.MLP70B_R,
                            gen=lambda rows, row0, name=name: W.mlp70b(name, rows=rows, row0=row0)))
        desc = f"mlp70b-prefill: M={M} tokens, gateup 8192->57344, down 28672->8192, r={W.MLP70B_R}"
    elif workload == "stress":
        c = W.STRESS
        cache = {}

        def gen(rows, row0, frac):
            key = (frac, rows, row0)
            if key not in cache:
                cache.clear()
                cache[key] = W.stress(frac, rows=rows, row0=row0)
            return cache[key]

        for frac in c["fracs"]:
            for r in c["rs"]:
                out.append(dict(name=f"frac{frac:g}-r{r}", M=c["M"], K=c["K"], N=c["N"], r=r,
                                gen=lambda rows, row0, frac=frac: gen(rows, row0, frac)))
        desc = (f"outlier-stress sweep: M={c['M']}, K=N={c['K']}, Student-t(3), outlier fraction "
                f"{list(c['fracs'])} x r {list(c['rs'])}")
    else:
        raise ValueError(workload)
    return out, desc


def kpad(k):
    return (k + 63) // 64 * 64


def layer_flops(L):
    return 2.0 * L["M"] * L["N"] * (L["K"] + L["r"])


def layer_quant_bytes(L):
    """Algorithmic bytes of the quantizer: read X once, write codes and scale bytes (FP8: one
    byte per value, no block scales)."""
    if L.get("fp8"):
        return 3 * L["M"] * L["K"]
    kp = kpad(L["K"] + L["r"])
    if L.get("mx"):  # one E8M0 byte per 32 values
        return 2 * L["M"] * L["K"] + L["M"] * kp // 2 + L["M"] * kp // 32
    return 2 * L["M"] * L["K"] + L["M"] * kp // 2 + L["M"] * kp // 16


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


def _ev():
    return torch.cuda.Event(enable_timing=True)


def flush_l2(buf):
    """Write a buffer about twice the L2's size, then read it back: no input stays in L2, and the
    lines left there are clean, so no write-back of the flush buffer lands in the timed work."""
    buf.zero_()
    buf.view(torch.int64).max()


def _barrier(world):
    if world > 1:
        torch.distributed.barrier()


def ranks_max(vals, device):
    """Element-wise maximum over the ranks (a job's time is its slowest rank's); the values
    themselves on one rank. Works with any process-group backend (NCCL on the GPUs, gloo in the
    CPU tests)."""
    t = torch.tensor([float(v) for v in vals], dtype=torch.float64, device=device)
    if torch.distributed.is_available() and torch.distributed.is_initialized() and \
            torch.distributed.get_world_size() > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


# ---------------------------------------------------------------------------------------------
# Our arm: linear-layer workloads
# ---------------------------------------------------------------------------------------------

def run_layers(args, rank, world, device, layers, with_error=False):
    import nvfp4_block_scaled_arc_b200 as arc
    import workloads as W

    stream = torch.cuda.Stream(device=device)
    reorder = getattr(args, "reorder", False)
    fp8 = getattr(args, "format", "nvfp4") == "fp8"
    mx = getattr(args, "format", "nvfp4") == "mxfp4"
    gemm = arc.gemm_fp8 if fp8 else arc.gemm_mxfp4 if mx else arc.gemm_nvfp4
    xs_host, xs, idx, packed, qa, ys, wsp, errs = {}, {}, {}, {}, {}, {}, {}, {}
    rs = {L["name"]: L["r"] for L in layers}

    def quant(name, **kw):
        # the step's quantizer: FP8, or NVFP4 in the natural channel order with the outlier list,
        # or NVFP4 reordered
        if fp8:
            return arc.quantize_fp8(xs[name], stream=stream, **kw)
        if mx:
            kw.pop("workspace", None)  # the MXFP4 quantizer needs none
            return arc.quantize_act_mxfp4(xs[name], idx[name], stream=stream, **kw)
        if reorder:
            return arc.quantize_act_nvfp4_reordered(xs[name], idx[name], rs[name], stream=stream, **kw)
        return arc.quantize_act_nvfp4(xs[name], idx[name], stream=stream, **kw)

    with torch.cuda.stream(stream):
        for L in layers:
            name, M, r = L["name"], L["M"], L["r"]
            d = L["gen"](M, rank * M)
            xs_host[name] = W.to_torch_bf16(d["x"])
            xs[name] = xs_host[name].to(device)
            w = W.to_torch_bf16(d["w"]).to(device)
            if fp8:
                idx[name] = None
                packed[name] = arc.quantize_fp8(w, stream=stream)  # weights: their own tensor scale
            elif mx:
                idx[name] = arc.calibrate_outliers(xs[name], r, stream=stream) if r else None
                packed[name] = arc.pack_weight_mxfp4(w, idx[name], stream=stream)
            elif reorder:
                # idx holds the full calibration order; its first r channels are the outliers
                idx[name] = arc.calibrate_order(xs[name], stream=stream)
                packed[name] = arc.pack_weight_nvfp4_reordered(w, idx[name], r, stream=stream)
            else:
                idx[name] = arc.calibrate_outliers(xs[name], r, stream=stream) if r else None
                packed[name] = arc.pack_weight_nvfp4(w, idx[name], stream=stream)
            qa[name] = quant(name)
            ys[name] = torch.empty(M, L["N"], dtype=torch.bfloat16, device=device)
            wsp[name] = torch.empty(arc.quantize_workspace_bytes(M, r), dtype=torch.uint8, device=device)
            if with_error:
                # relative error of the NVFP4 + ARC output against the BF16 product of the inputs,
                # over all rows and over the rows holding the maxima of the 32 largest channels
                # (where the residual channels act)
                y = gemm(qa[name], packed[name], stream=stream).float()
                yb = arc.gemm_bf16(xs[name], w, stream=stream).float()
                errs[name] = (torch.linalg.norm(y - yb) / torch.linalg.norm(yb)).item()
                xa = xs[name].float().abs()
                top = torch.topk(xa.amax(dim=0), k=min(32, xa.shape[1])).indices
                rows = torch.unique(xa[:, top].argmax(dim=0))
                errs[name + "/outlier_rows"] = (torch.linalg.norm(y[rows] - yb[rows]) /
                                                torch.linalg.norm(yb[rows])).item()
                del xa
            del w
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream.synchronize()

    def step(rec):
        for L in layers:
            name = L["name"]
            e0, e1, e2 = (_ev(), _ev(), _ev()) if rec is not None else (None, None, None)
            if e0 is not None:
                e0.record(stream)
            quant(name, out=qa[name], workspace=wsp[name])
            if e1 is not None:
                e1.record(stream)
            gemm(qa[name], packed[name], out=ys[name], stream=stream)
            if e2 is not None:
                e2.record(stream)
                rec.append((e0, e1, e2))

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush_l2(flush)
            step(None)
    stream.synchronize()
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during warm-up")

    # two timed passes of K steps each, the L2 flushed before every step: the first with events
    # around each step only (the step's time: events between the kernels would add their own
    # gaps and keep a kernel from starting while the one before it finishes), the second with
    # events around every kernel call (the per-kernel times of the roofline)
    step_ev, kern = [], []
    _barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device) as clk:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                flush_l2(flush)
                s0, s1 = _ev(), _ev()
                s0.record(stream)
                step(None)
                s1.record(stream)
                step_ev.append((s0, s1))
            for _ in range(args.steps):
                flush_l2(flush)
                rec = []
                step(rec)
                kern.append(rec)
        torch.cuda.synchronize(device)
    _barrier(world)
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the timed steps")
    total_ms = sum(a.elapsed_time(b) for a, b in step_ev)
    q_ms = sum(r[0].elapsed_time(r[1]) for rec in kern for r in rec)
    g_ms = sum(r[1].elapsed_time(r[2]) for rec in kern for r in rec)
    per_layer = {}
    for i, L in enumerate(layers):
        gq = statistics.mean(rec[i][0].elapsed_time(rec[i][1]) for rec in kern)
        gg = statistics.mean(rec[i][1].elapsed_time(rec[i][2]) for rec in kern)
        per_layer[L["name"]] = {"quant_us": 1e3 * gq, "quant_gbs": layer_quant_bytes(L) / (gq * 1e-3) / 1e9,
                                "gemm_us": 1e3 * gg, "gemm_tflops": layer_flops(L) / (gg * 1e-3) / 1e12}
        if with_error:
            per_layer[L["name"]]["rel_err_vs_bf16"] = errs[L["name"]]
            per_layer[L["name"]]["rel_err_vs_bf16_outlier_rows"] = errs[L["name"] + "/outlier_rows"]
    clocks = clk.summary()

    # e2e through the public API with host buffers: pinned X in, Y out, every step
    e2e_ms, h2d, d2h = float("nan"), 0, 0
    if not args.no_e2e:
        xs_pin = {k: v.pin_memory() for k, v in xs_host.items()}
        ys_pin = {L["name"]: torch.empty(L["M"], L["N"], dtype=torch.bfloat16).pin_memory() for L in layers}
        h2d = sum(v.numel() * 2 for v in xs_pin.values())
        d2h = sum(v.numel() * 2 for v in ys_pin.values())

        # three streams: host-to-device copies, compute, device-to-host copies. Within a step the
        # upload of the next projection's X and the download of the previous Y overlap the
        # compute (PCIe is full duplex); events order each copy against the work that uses it.
        # A step starts after its start event and ends after its last download.
        up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
        x_ready = {L["name"]: torch.cuda.Event() for L in layers}
        y_ready = {L["name"]: torch.cuda.Event() for L in layers}

        def e2e_step(start):
            up.wait_event(start)
            for L in layers:
                name = L["name"]
                with torch.cuda.stream(up):
                    xs[name].copy_(xs_pin[name], non_blocking=True)
                x_ready[name].record(up)
            for L in layers:
                name = L["name"]
                stream.wait_event(x_ready[name])
                quant(name, out=qa[name], workspace=wsp[name])
                gemm(qa[name], packed[name], out=ys[name], stream=stream)
                y_ready[name].record(stream)
                down.wait_event(y_ready[name])
                with torch.cuda.stream(down):
                    ys_pin[name].copy_(ys[name], non_blocking=True)
            stream.wait_stream(down)

        with torch.cuda.stream(stream):
            for _ in range(max(1, min(args.warmup, 2))):
                s0 = _ev()
                s0.record(stream)
                e2e_step(s0)
        stream.synchronize()
        _barrier(world)
        e2e_ev = []
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                a, b = _ev(), _ev()
                a.record(stream)
                e2e_step(a)
                b.record(stream)
                e2e_ev.append((a, b))
        stream.synchronize()
        _barrier(world)
        e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_ev)

    total_ms, q_ms, g_ms, e2e_ms = ranks_max([total_ms, q_ms, g_ms, e2e_ms], device)
    # kernels per layer and step: the quantizer's (MXFP4: one; the others: abs-max + coding) and
    # the GEMM
    per_layer_launches = 2 if mx else 3
    return dict(total_ms=total_ms, q_ms=q_ms, g_ms=g_ms, e2e_ms=e2e_ms, per_layer=per_layer, clocks=clocks,
                h2d=h2d, d2h=d2h, launches=2 * args.steps * len(layers) * per_layer_launches)


def layers_line(args, world, layers, desc, res):
    pk, src = peaks()
    step_flops = sum(layer_flops(L) for L in layers)
    qbytes = sum(layer_quant_bytes(L) for L in layers)
    value = step_flops * world * args.steps / (res["total_ms"] * 1e-3) / 1e12
    achieved = step_flops * args.steps / (res["g_ms"] * 1e-3) / 1e12
    quant_gbs = qbytes * args.steps / (res["q_ms"] * 1e-3) / 1e9
    fmt = getattr(args, "format", "nvfp4")
    fp8, mx = fmt == "fp8", fmt == "mxfp4"
    ratio = 2.0 if fp8 else FP4_OVER_BF16  # nominal dense FP8 / BF16 = 2, FP4 / BF16 = 4
    peak = pk["bf16_tflops"] * ratio
    qkern = ("k_amax + k_quant_fp8" if fp8 else "k_quant_mx_rows" if mx else
             "k_amax + k_quant_reordered" if getattr(args, "reorder", False) else "k_amax + k_quant_rows")
    return {
        "metric": METRIC_FP8 if fp8 else METRIC_MX if mx else METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": res["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> f32 (bf16 out)" if fp8 else "e2m1 x e2m1 -> f32 (bf16 out)",
        "data": "synthetic (seeded; random weights and activations of the stated shapes)",
        "config": {"workload": desc, "l2": "flushed before every step (256 MiB written, then read back)",
                   "timing": "step time from a pass with events around each step only; kernel times from a "
                             "second pass with events around every kernel call",
                   "parallelism": f"replicas x{world}",
                   "channel_order": "reordered by calibration abs-max" if getattr(args, "reorder", False)
                   else "natural (outlier list)"},
        "quant_gbs": quant_gbs,
        "gemm_only_tflops": achieved,
        ("pct_fp8_peak" if fp8 else "pct_fp4_peak"): 100.0 * value / peak,
        "per_projection": res["per_layer"],
        "roofline": {"bound": "tensor",
                     "kernel": f"k_gemm<{fmt}> (all {len(layers)} launches of a step)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{src} bf16 burst {pk['bf16_tflops']} TFLOP/s x {ratio:g} "
                                    f"(nominal {'FP8' if fp8 else 'FP4'}/BF16 dense ratio)",
                     "traffic": ncu_traffic() if args.workload == "llama8b" and not getattr(args, "reorder", False)
                     and fmt == "nvfp4" else None},
        "quant_roofline": {"bound": "hbm",
                           "kernel": qkern,
                           "achieved": quant_gbs,
                           "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": quant_gbs / pk["hbm_gbs"],
                           "peak_source": f"{src} copy bandwidth"},
        "clocks": res["clocks"],
        "e2e": None if args.no_e2e else {
            "value": step_flops * world * args.steps / (res["e2e_ms"] * 1e-3) / 1e12, "unit": UNIT,
            "h2d_bytes_per_step": res["h2d"], "d2h_bytes_per_step": res["d2h"]},
        "gpu_launches": res["launches"],
    }


# ---------------------------------------------------------------------------------------------
# Our arm: the RAMP-style recurrent prefill
# ---------------------------------------------------------------------------------------------

def run_recurrent(args, rank, world, device):
    import nvfp4_block_scaled_arc_b200 as arc
    import workloads as W

    c = W.RECURRENT
    S, d, F, T, r, eps = c["S"], c["d"], c["ffn"], c["T"], c["r"], c["eps"]
    rec = W.recurrent()
    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        h0 = W.to_torch_bf16(rec["h"]).to(device)
        subs = []
        for L in rec["layers"]:
            wgu, wd, gain = (W.to_torch_bf16(L[k]).to(device) for k in ("wgu", "wd", "gain"))
            # offline calibration on a BF16 pass of the block's first step
            n = arc.rmsnorm_bf16(h0, gain, eps, stream=stream)
            idx_gu = arc.calibrate_outliers(n, r, stream=stream)
            act = arc.silu_mul_bf16(arc.gemm_bf16(n, wgu, stream=stream), stream=stream)
            idx_d = arc.calibrate_outliers(act, r, stream=stream)
            subs.append(dict(gain=gain, wgu=wgu, wd=wd, idx_gu=idx_gu, idx_d=idx_d,
                             gu_q=arc.pack_weight_nvfp4(wgu, idx_gu, stream=stream),
                             d_q=arc.pack_weight_nvfp4(wd, idx_d, stream=stream),
                             gu_f8=arc.quantize_fp8(wgu, stream=stream), d_f8=arc.quantize_fp8(wd, stream=stream)))
        blk = arc.RecurrentBlock(d, F, eps, subs)
        wsp = torch.empty(blk.workspace_bytes(S), dtype=torch.uint8, device=device)
        h = torch.empty_like(h0)
        flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream.synchronize()
    k_lows = list(c["k_lows"])
    # GEMM flops of one prefill (both sublayers, every step): gate|up and down; NVFP4 steps run
    # depth K + r
    f_bf16 = 2 * (2.0 * S * (2 * F * d + d * F))
    f_fp4 = 2 * (2.0 * S * (2 * F * (d + r) + d * (F + r)))

    def prefill(k):
        h.copy_(h0)
        arc.recurrent_prefill(h, blk, T, k, workspace=wsp, stream=stream)

    out = {}
    with torch.cuda.stream(stream):
        for k in k_lows:
            prefill(k)
            out[k] = h.float().clone()
    stream.synchronize()
    ref = out[0]
    fidelity = {k: (torch.linalg.norm(out[k] - ref) / torch.linalg.norm(ref)).item() for k in k_lows}
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            for k in k_lows:
                flush_l2(flush)
                prefill(k)
    stream.synchronize()
    times = {k: [] for k in k_lows}
    _barrier(world)
    torch.cuda.synchronize(device)
    evs = []
    with ClockSampler(device) as clk:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                for k in k_lows:
                    flush_l2(flush)
                    a, b = _ev(), _ev()
                    a.record(stream)
                    prefill(k)
                    b.record(stream)
                    evs.append((k, a, b))
        torch.cuda.synchronize(device)
    _barrier(world)
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the timed prefills")
    for k, a, b in evs:
        times[k].append(a.elapsed_time(b))
    ms = dict(zip(k_lows, ranks_max([statistics.mean(times[k]) for k in k_lows], device)))
    per = {}
    for k in k_lows:
        fl = (k * f_fp4 + (T - k) * f_bf16) * world
        per[f"k_low={k}"] = {"ms": ms[k], "speedup_vs_all_bf16": ms[k_lows[0]] / ms[k],
                             "gemm_tflops": fl / (ms[k] * 1e-3) / 1e12,
                             "hidden_state_rel_err_vs_all_bf16": fidelity[k]}
    kk = 12 if 12 in ms else k_lows[-1]
    study = ramp_fp8 = contractive = None
    if not args.no_studies:
        study = schedule_study(arc, h, h0, blk, wsp, flush, stream, T, kk, out[0], device)
        ramp_fp8 = ramp_instantiations(arc, h, h0, blk, wsp, flush, stream, device)
        contractive = contractive_study(arc, device, stream, T=T, budget=kk, r=r)
    # kernels per prefill: NVFP4 step = 2 x (2 quantizer launches + GEMM + SiLU + 2 quantizer
    # launches + GEMM), BF16 step = 2 x (RMSNorm + GEMM + SiLU + GEMM)
    launches = args.steps * sum(k * 2 * 7 + (T - k) * 2 * 4 for k in k_lows)
    return {
        "metric": f"RAMP-style recurrent prefill time (T={T}, first {kk} steps NVFP4+ARC then BF16), 1×B200",
        "value": ms[kk], "unit": "ms", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": sum(ms.values()), "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "e2m1 x e2m1 -> f32 (NVFP4 steps), bf16 x bf16 -> f32 (BF16 steps); bf16 hidden state",
        "data": "synthetic (seeded; random weights and hidden state of the stated shapes)",
        "config": {"workload": f"recurrent SwiGLU block: S={S}, d={d}, ffn={F}, 2 pre-norm sublayers, T={T}, "
                               f"k_low in {k_lows}, r={r}",
                   "l2": "flushed before every prefill (256 MiB written, then read back)", "parallelism": f"replicas x{world}"},
        "per_k_low": per, "schedule_study": study, "ramp_t32_k24": ramp_fp8, "contractive_study": contractive,
        "clocks": clk.summary(),
        "e2e": None, "gpu_launches": launches,
    }


def contractive_study(arc, device, stream, S=1024, d=2048, F=8192, T=16, budget=12, r=64, beta=0.5, eps=1.0,
                      n_random=24, w_scale=4.0, e_std=1.0):
    """RAMP's placement result (section 3, Theorem 3.2: with locally contractive steps, low
    precision early and BF16 late minimises the final-error bound; late placement maximises it;
    random schedules fall between) checked on a block built to contract towards a nonzero fixed
    point: the damped residual with input injection h <- beta h + e + F(h), beta = 1/2, e ~ N(0, 1)
    (a recurrence that re-reads its input every step), RMSNorm eps = 1, the recurrent workload's
    weights times 4 (std 0.02, as the linear-layer workloads). The contraction factor is measured (BF16 step map, the ratio of output to input
    perturbation norms); each schedule's final hidden-state error is against the all-BF16 run.
    Fidelity only: nothing here is timed."""
    import workloads as W

    rec = W.recurrent(S=S, d=d, ffn=F)
    with torch.cuda.stream(stream):
        h0 = W.to_torch_bf16(rec["h"]).to(device)
        e = W.to_torch_bf16(W.matrix_bf16(W.RECURRENT["seed"], 99, S, d, e_std)).to(device)
        subs = []
        for L in rec["layers"]:
            wgu, wd, gain = (W.to_torch_bf16(L[k]).to(device) for k in ("wgu", "wd", "gain"))
            wgu, wd = (wgu.float() * w_scale).bfloat16(), (wd.float() * w_scale).bfloat16()
            n = arc.rmsnorm_bf16(h0, gain, eps, stream=stream)
            idx_gu = arc.calibrate_outliers(n, r, stream=stream)
            act = arc.silu_mul_bf16(arc.gemm_bf16(n, wgu, stream=stream), stream=stream)
            idx_d = arc.calibrate_outliers(act, r, stream=stream)
            subs.append(dict(gain=gain, wgu=wgu, wd=wd, idx_gu=idx_gu, idx_d=idx_d,
                             gu_q=arc.pack_weight_nvfp4(wgu, idx_gu, stream=stream),
                             d_q=arc.pack_weight_nvfp4(wd, idx_d, stream=stream)))
        blk = arc.RecurrentBlock(d, F, eps, subs, beta, inject=e)
        ws = torch.empty(blk.workspace_bytes(S), dtype=torch.uint8, device=device)

        def run(flags, h_in=None):
            h = (h0 if h_in is None else h_in).clone()
            arc.recurrent_prefill_schedule(h, blk, flags, workspace=ws, stream=stream)
            return h

        # contraction factor of the BF16 step map along the reference trajectory
        rng = torch.Generator(device="cpu").manual_seed(7)
        rho, h = [], h0.clone()
        for t in range(T):
            dlt = (torch.randn(h.shape, generator=rng) * 1e-2 * h.float().pow(2).mean().sqrt().item()).to(device)
            hp = (h.float() + dlt).bfloat16()
            a, b = run([0], h), run([0], hp)
            rho.append((torch.linalg.norm(b.float() - a.float()) / torch.linalg.norm(hp.float() - h.float())).item())
            h = a
        ref = run([0] * T).float()

        def err(flags):
            return (torch.linalg.norm(run(flags).float() - ref) / torch.linalg.norm(ref)).item()

        k = T - budget
        sch = {"ramp": [1] * budget + [0] * k, "early_bf16": [0] * k + [1] * budget,
               "interleaved": [0 if (t % (T // k)) == T // k - 1 else 1 for t in range(T)]}
        gen = np.random.default_rng(11)
        seen = {tuple(v) for v in sch.values()}
        rand = []
        while len(rand) < n_random:
            f = np.zeros(T, np.int64)
            f[gen.choice(T, size=budget, replace=False)] = 1
            if tuple(f.tolist()) not in seen:
                seen.add(tuple(f.tolist()))
                rand.append(f.tolist())
        out = {name: {"schedule": "".join("L" if f else "B" for f in flags), "err": err(flags)}
               for name, flags in sch.items()}
        rerr = [err(f) for f in rand]
    stream.synchronize()
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the contractive study")
    return {"block": f"damped residual with input injection (h <- beta h + e + F(h)), beta={beta}, e~N(0,{e_std}^2), "
                     f"weights x{w_scale} of the recurrent workload's, "
                     f"RMSNorm eps={eps}, S={S}, d={d}, ffn={F}, r={r}, T={T}, {budget} NVFP4 + {k} BF16 steps",
            "contraction_factor": {"median": statistics.median(rho), "max": max(rho)},
            "schedules": out,
            "random": {"n": n_random, "min": min(rerr), "median": statistics.median(rerr), "max": max(rerr)},
            "ordering_holds": out["ramp"]["err"] <= min(rerr) and max(rerr) <= out["early_bf16"]["err"]}


def ramp_instantiations(arc, h, h0, blk, wsp, flush, stream, device, T=32, K=24, reps=5):
    """RAMP's own instantiation ("RAMP…" §4.2: T = 32 recurrent steps, the first K = 24 in FP8 W8A8
    with dynamic per-tensor FP8 activations, the last 8 in BF16) next to the same schedule with
    NVFP4 + ARC low-precision steps and the all-BF16 prefill: prefill time (median of reps, L2
    flushed before each) and final hidden-state error against all-BF16. Run after the timed
    region."""
    sch = {"all_bf16": [arc.STEP_BF16] * T,
           "ramp_fp8": [arc.STEP_FP8] * K + [arc.STEP_BF16] * (T - K),
           "ramp_nvfp4_arc": [arc.STEP_NVFP4] * K + [arc.STEP_BF16] * (T - K),
           "uniform_fp8": [arc.STEP_FP8] * T}
    res, ref = {}, None
    for name, fmts in sch.items():
        with torch.cuda.stream(stream):
            h.copy_(h0)
            arc.recurrent_prefill_schedule(h, blk, fmts, workspace=wsp, stream=stream)
            out = h.float().clone()
            ts = []
            for _ in range(reps):
                flush_l2(flush)
                h.copy_(h0)
                a, b = _ev(), _ev()
                a.record(stream)
                arc.recurrent_prefill_schedule(h, blk, fmts, workspace=wsp, stream=stream)
                b.record(stream)
                ts.append((a, b))
        stream.synchronize()
        if ref is None:
            ref = out
        res[name] = {"ms": statistics.median(a.elapsed_time(b) for a, b in ts),
                     "hidden_state_rel_err_vs_all_bf16": (torch.linalg.norm(out - ref) / torch.linalg.norm(ref)).item()}
    for name in res:
        res[name]["speedup_vs_all_bf16"] = res["all_bf16"]["ms"] / res[name]["ms"]
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the RAMP instantiations")
    return res


def schedule_study(arc, h, h0, blk, wsp, flush, stream, T, budget, ref, device, reps=5):
    """Where the BF16 steps go at a fixed budget of NVFP4 steps (RAMP's matched-budget comparison:
    low precision first and BF16 last, against Early-BF16 and random placements): hidden-state
    error against all-BF16 and the prefill time of each schedule. Run after the timed region."""
    rng = np.random.default_rng(3)
    sch = {"ramp (NVFP4 first)": [1] * budget + [0] * (T - budget),
           "early_bf16 (BF16 first)": [0] * (T - budget) + [1] * budget,
           "interleaved": [0 if (t % (T // max(1, T - budget))) == T // max(1, T - budget) - 1 else 1
                           for t in range(T)]}
    for i in range(3):
        f = np.zeros(T, np.int64)
        f[rng.choice(T, size=budget, replace=False)] = 1
        sch[f"random {i}"] = f.tolist()
    res = {}
    for name, flags in sch.items():
        with torch.cuda.stream(stream):
            h.copy_(h0)
            arc.recurrent_prefill_schedule(h, blk, flags, workspace=wsp, stream=stream)
            err = (torch.linalg.norm(h.float() - ref) / torch.linalg.norm(ref)).item()
            ts = []
            for _ in range(reps):
                flush_l2(flush)
                h.copy_(h0)
                a, b = _ev(), _ev()
                a.record(stream)
                arc.recurrent_prefill_schedule(h, blk, flags, workspace=wsp, stream=stream)
                b.record(stream)
                ts.append((a, b))
        stream.synchronize()
        res[name] = {"schedule": "".join("L" if f else "B" for f in flags), "nvfp4_steps": int(sum(flags)),
                     "ms": statistics.median(a.elapsed_time(b) for a, b in ts),
                     "hidden_state_rel_err_vs_all_bf16": err}
    if arc.last_device_status(stream) != 0:
        raise RuntimeError("device status set during the schedule study")
    return res


# ---------------------------------------------------------------------------------------------
# Oracle arm (CPU)
# ---------------------------------------------------------------------------------------------

def oracle_cache(layers, n_rows: int, reorder: bool = False, fmt: str = "nvfp4"):
    import oracle as O

    cache = {}
    for L in layers:
        d = L["gen"](n_rows, 0)
        x = d["x"][:n_rows]
        if fmt == "mxfp4":
            idx = O.calibrate(x, L["r"]) if L["r"] else np.zeros(0, np.int32)
            bc, bsc = O.pack_weight_mxfp4(d["w"], idx)
            cache[L["name"]] = dict(x=x, idx=idx, bc=bc, bsc=bsc, fmt=fmt)
            continue
        if fmt == "fp8":
            sa, sw = O.fp8_scale(O.amax(x)), O.fp8_scale(O.amax(d["w"]))
            cache[L["name"]] = dict(x=x, sa=sa, sw=sw, bc=O.quantize_fp8(d["w"], sw), fmt=fmt)
            continue
        sa = O.tensor_scale(O.amax(x))
        sw = O.tensor_scale(O.amax(d["w"]))
        if reorder:
            idx = O.calibrate_order(x)
            bc, bsf = O.pack_weight_reordered(d["w"], idx, L["r"], sw)
        else:
            idx = O.calibrate(x, L["r"]) if L["r"] else np.zeros(0, np.int32)
            bc, bsf = O.pack_weight(d["w"], idx, sw)  # every output column needs the full weight
        cache[L["name"]] = dict(x=x, idx=idx, sa=sa, sw=sw, bc=bc, bsf=bsf, reorder=reorder, fmt=fmt)
    return cache


def oracle_sample_step(layers, rows: int, cache: dict):
    """One bounded sample of the step on the CPU oracle: `rows` token rows of every layer through
    quantization (idx from the sample's calibration, cached up front) and the FP64 GEMM of those
    rows against all N outputs. Returns algorithmic flops."""
    import oracle as O

    flops = 0.0
    for L in layers:
        c = cache[L["name"]]
        if c["fmt"] == "mxfp4":
            ac, asc = O.quantize_act_mxfp4(c["x"][:rows], c["idx"])
            O.gemm_mxfp4_f64(ac, asc, c["bc"], c["bsc"])
            flops += 2.0 * rows * L["N"] * (L["K"] + L["r"])
            continue
        if c["fmt"] == "fp8":
            O.gemm_fp8_f64(O.quantize_fp8(c["x"][:rows], c["sa"]), c["sa"], c["bc"], c["sw"])
            flops += 2.0 * rows * L["N"] * L["K"]
            continue
        if c["reorder"]:
            ac, asf = O.quantize_act_reordered(c["x"][:rows], c["idx"], L["r"], c["sa"])
        else:
            ac, asf = O.quantize_act(c["x"][:rows], c["idx"], c["sa"])
        O.gemm_nvfp4_f64(ac, asf, c["sa"], c["bc"], c["bsf"], c["sw"])
        flops += 2.0 * rows * L["N"] * (L["K"] + L["r"])
    return flops


def cpu_baseline(layers, rows: int | None = None, reorder: bool = False, fmt: str = "nvfp4"):
    """The oracle on the host cores: `rows` token rows (default two per host thread, so every
    thread works) of each layer, about 10-30 s of CPU work."""
    import oracle as O

    rows = rows or 2 * O._threads()
    cache = oracle_cache(layers, max(rows, 64), reorder, fmt)
    t0 = time.perf_counter()
    flops = oracle_sample_step(layers, rows, cache)
    dt = time.perf_counter() - t0
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": min(O._threads(), rows), "kind": "oracle",
            "sample": f"{rows} token row(s) of each of the {len(layers)} layers (quantize + FP64 GEMM against "
                      f"all N), {dt:.1f} s"}


def run_reference(args, rank, world, layers, desc):
    if rank != 0:
        return
    import oracle as O

    rows = O._threads()  # one token row per host thread per step
    cache = oracle_cache(layers, max(rows, 64), getattr(args, "reorder", False), getattr(args, "format", "nvfp4"))
    for _ in range(args.warmup):
        oracle_sample_step(layers, rows, cache)
    t0 = time.perf_counter()
    flops = 0.0
    for _ in range(args.steps):
        flops += oracle_sample_step(layers, rows, cache)
    dt = time.perf_counter() - t0
    v = flops / dt / 1e12
    fmt = getattr(args, "format", "nvfp4")
    metric = METRIC_FP8 if fmt == "fp8" else METRIC_MX if fmt == "mxfp4" else METRIC
    line = {"impl": "reference", "metric": metric, "value": v, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": f"{desc} (oracle on a row sample)", "sample_rows_per_projection": rows},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": O._threads(), "kind": "oracle",
                             "sample": f"{rows} token rows of each of the {len(layers)} layers per step "
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
    ap.add_argument("--workload", default="llama8b", choices=["llama8b", "mlp70b", "stress", "recurrent"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end pass")
    ap.add_argument("--proj", default="all", help="profiling: run only this layer (e.g. qkv, gateup)")
    ap.add_argument("--no-studies", action="store_true",
                    help="recurrent workload: the k_low sweep only (no schedule, RAMP T=32 or contractive study)")
    ap.add_argument("--format", default="nvfp4", choices=["nvfp4", "mxfp4", "fp8"],
                    help="linear-layer workloads: NVFP4 + ARC (default), MXFP4 + ARC (32-value blocks, "
                         "power-of-two scales, no tensor scale) or FP8 W8A8 with per-tensor scales")
    ap.add_argument("--reorder", action="store_true",
                    help="linear-layer workloads: channels reordered by calibration abs-max before the primary "
                         "quantization (the outlier set is the first r of the order)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    if "WORLD_SIZE" in os.environ:
        # launched by torchrun (or another launcher): one process per GPU already
        if int(os.environ["WORLD_SIZE"]) != args.gpus:
            ap.error(f"--gpus {args.gpus} but WORLD_SIZE={os.environ['WORLD_SIZE']}")
        run(args, ap)
    elif args.gpus > 1 and args.impl == "ours":
        # no launcher: start one process per GPU here (spawned, NCCL over the visible GPUs)
        n = torch.cuda.device_count()
        if n < args.gpus:
            ap.error(f"--gpus {args.gpus} but only {n} CUDA device(s) are visible")
        spawn_ranks(args)
    else:
        # one GPU; or the oracle arm, which rank 0 alone runs (the other ranks have no work)
        os.environ.setdefault("WORLD_SIZE", str(args.gpus))
        run(args, ap)


def _free_port() -> int:
    import socket

    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def _rank_main(local_rank: int, args, port: int):
    os.environ.update({"RANK": str(local_rank), "LOCAL_RANK": str(local_rank), "WORLD_SIZE": str(args.gpus),
                       "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    run(args, None)


def spawn_ranks(args):
    """One process per GPU (ranks 0..N-1 on devices 0..N-1), the same rendezvous torchrun would
    give them; rank 0 prints the JSON line. A rank that fails makes the launch raise."""
    import torch.multiprocessing as mp

    mp.start_processes(_rank_main, args=(args, _free_port()), nprocs=args.gpus, start_method="spawn", join=True)


def run(args, ap):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    def fail(msg):
        if ap is not None:
            ap.error(msg)
        raise SystemExit(msg)

    layers, desc = None, None
    if args.workload != "recurrent":
        layers, desc = layer_set(args.workload)
        if args.proj != "all":
            layers = [L for L in layers if L["name"] == args.proj]
            if not layers:
                fail("unknown --proj")
    if args.format == "mxfp4" and layers is not None:
        if args.reorder:
            fail("--reorder applies to the NVFP4 format")
        for L in layers:
            L["mx"] = True
        desc = f"{desc}; run in MXFP4 + ARC (32-value blocks, E8M0 scales)"
    if args.format == "fp8" and layers is not None:
        if args.reorder:
            fail("--reorder applies to the NVFP4 format")
        for L in layers:
            L["r"], L["fp8"] = 0, True
        desc = f"{desc}; run in FP8 W8A8 (per-tensor scales, no residual channels)"
    if args.impl == "reference":
        if layers is None:
            if rank == 0:
                print(json.dumps({"impl": "reference",
                                  "unavailable": "the oracle arm times the linear-layer workloads only"}))
            return
        run_reference(args, rank, world, layers, desc)
        return
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", device_id=device, timeout=datetime.timedelta(seconds=180))
    try:
        if args.workload == "recurrent":
            line = run_recurrent(args, rank, world, device)
        else:
            res = run_layers(args, rank, world, device, layers,
                             with_error=args.workload == "stress" or args.reorder or args.format != "nvfp4")
            line = layers_line(args, world, layers, desc, res) if rank == 0 else None
            if rank == 0 and not args.no_cpu_baseline:
                line["cpu_baseline"] = cpu_baseline(layers, reorder=args.reorder, fmt=args.format)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
