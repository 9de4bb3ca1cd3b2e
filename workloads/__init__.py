"""Seeded synthetic workloads (shared by tests, benchmark and oracle checks).

Holds no quantization or GEMM arithmetic: only the draws of ``gen.c`` (counter-based SplitMix64,
Box-Muller normals, Student-t(3), partial Fisher-Yates channel sets, log-uniform magnitudes) and
the recipes that turn them into the benchmark's synthetic tensors. Stream numbering per tensor
id t: X = 1+16t, W = 2+16t, outlier channel set = 3+16t, outlier magnitudes = 4+16t.

Recipes (shapes, value distributions; the weights and activations are random, nothing is loaded):
  tiny      M=16, K=N=256, X~N(0,1) with channels {7, 131} x40, W~N(0,0.02), r=16, seed 0
  llama8b   M=4096 token batch, projections qkv (K=4096,N=6144), o (4096,4096),
            gateup (4096,28672), down (14336,4096); X~N(0,1) with 1% channels x LogU[20,80];
            W~N(0,0.02); r=128; seed 1
  stress    M=2048, K=N=4096; X~Student-t(3) with a fraction {0,0.1%,1%,5%} of channels
            x LogU[10,200]; W~N(0,0.02); r in {0,32,128,256}; seed 2
  recurrent H [4096,2048]~N(0,1); two SwiGLU sublayers d=2048, ffn=8192, gate|up fused to
            N=16384; W~N(0,0.02/sqrt(16)); RMSNorm gain 1; T=16, k_low in {0,8,12,16}; r=64; seed 3
  mlp70b    M=16384, gateup (K=8192,N=57344), down (K=28672,N=8192); X~N(0,1) with 0.5%
            channels x50; W~N(0,0.015); r=256; seed 4
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.c")
_LIB = os.path.join(_HERE, "libgen.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _L():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P, I64, U64, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_double
            L.gen_matrix_bf16.argtypes = [U64, U64, ctypes.c_int, I64, D, P, I64, I64, P, I64]
            L.gen_matrix_bf16.restype = None
            L.gen_channel_set.argtypes = [U64, U64, I64, I64, P, P]
            L.gen_channel_set.restype = None
            L.gen_log_uniform.argtypes = [U64, U64, I64, D, D, P]
            L.gen_log_uniform.restype = None
            L.gen_u01.argtypes = [U64, U64]
            L.gen_u01.restype = D
            L.gen_key.argtypes = [U64, U64]
            L.gen_key.restype = U64
            L.gen_normal.argtypes = [U64, U64]
            L.gen_normal.restype = D
            _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def stream_id(tensor: int, kind: int) -> int:
    return kind + 16 * tensor


def matrix_bf16(seed: int, stream: int, rows: int, cols: int, std: float = 1.0, dist: str = "normal",
                col_mult=None, row0: int = 0, threads: int | None = None) -> np.ndarray:
    """[rows, cols] bf16 bits (uint16), element (m, k) at counter (row0 + m) * cols + k."""
    out = np.empty((rows, cols), np.uint16)
    cm = None if col_mult is None else np.ascontiguousarray(col_mult, dtype=np.float64)
    L = _L()
    d = 1 if dist == "t3" else 0
    t = threads or min(64, os.cpu_count() or 1)
    t = max(1, min(t, rows))
    step = (rows + t - 1) // t

    def run(r0):
        r1 = min(rows, r0 + step)
        L.gen_matrix_bf16(seed, stream, d, cols, float(std), _p(cm) if cm is not None else None,
                          row0 + r0, row0 + r1, out[r0:].ctypes.data_as(ctypes.c_void_p), cols)

    if t == 1:
        run(0)
    else:
        with ThreadPoolExecutor(max_workers=t) as ex:
            list(ex.map(run, range(0, rows, step)))
    return out


def channel_set(seed: int, stream: int, K: int, n: int) -> np.ndarray:
    scratch = np.empty(K, np.int32)
    out = np.empty(max(n, 1), np.int32)
    if n > 0:
        _L().gen_channel_set(seed, stream, K, n, _p(scratch), _p(out))
    return out[:n].copy()


def log_uniform(seed: int, stream: int, n: int, lo: float, hi: float) -> np.ndarray:
    out = np.empty(max(n, 1), np.float64)
    if n > 0:
        _L().gen_log_uniform(seed, stream, n, lo, hi, _p(out))
    return out[:n].copy()


def outlier_multipliers(seed: int, tensor: int, K: int, n: int, lo: float, hi: float) -> np.ndarray:
    """Per-channel multipliers: n random channels scaled by LogU[lo, hi] (lo == hi: fixed)."""
    mult = np.ones(K, np.float64)
    ch = channel_set(seed, stream_id(tensor, 3), K, n)
    if lo == hi:
        mags = np.full(n, lo, np.float64)
    else:
        mags = log_uniform(seed, stream_id(tensor, 4), n, lo, hi)
    mult[ch] = mags
    return mult


def to_torch_bf16(bits: np.ndarray):
    import torch

    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)


# --------------------------------------------------------------------------------------------
# Recipes
# --------------------------------------------------------------------------------------------

TINY = dict(name="tiny", seed=0, M=16, K=256, N=256, r=16)

LLAMA8B_M = 4096
LLAMA8B_PROJ = {  # name: (tensor id, K, N)
    "qkv": (0, 4096, 6144),
    "o": (1, 4096, 4096),
    "gateup": (2, 4096, 28672),
    "down": (3, 14336, 4096),
}
LLAMA8B_R = 128

STRESS = dict(seed=2, M=2048, K=4096, N=4096, fracs=(0.0, 0.001, 0.01, 0.05), rs=(0, 32, 128, 256))

RECURRENT = dict(seed=3, S=4096, d=2048, ffn=8192, T=16, k_lows=(0, 8, 12, 16), r=64, eps=1e-6)

MLP70B_M = 16384
MLP70B_PROJ = {"gateup": (0, 8192, 57344), "down": (1, 28672, 8192)}
MLP70B_R = 256


def tiny(rows: int | None = None):
    """X [16, 256] with channels {7, 131} x40 and W [256, 256] ~ N(0, 0.02)."""
    c = TINY
    M = rows or c["M"]
    mult = np.ones(c["K"], np.float64)
    mult[[7, 131]] = 40.0
    x = matrix_bf16(c["seed"], stream_id(0, 1), M, c["K"], 1.0, col_mult=mult)
    w = matrix_bf16(c["seed"], stream_id(0, 2), c["N"], c["K"], 0.02)
    return dict(x=x, w=w, r=c["r"], K=c["K"], N=c["N"], M=M)


def llama8b(proj: str, rows: int | None = None, row0: int = 0, with_w: bool = True, w_rows: int | None = None):
    """One projection of the Llama-3-8B-shaped prefill batch (rows/w_rows shrink it for tests)."""
    t, K, N = LLAMA8B_PROJ[proj]
    seed = 1
    M = LLAMA8B_M if rows is None else rows
    n_out = int(round(0.01 * K))
    mult = outlier_multipliers(seed, t, K, n_out, 20.0, 80.0)
    x = matrix_bf16(seed, stream_id(t, 1), M, K, 1.0, col_mult=mult, row0=row0)
    w = matrix_bf16(seed, stream_id(t, 2), N if w_rows is None else w_rows, K, 0.02) if with_w else None
    return dict(x=x, w=w, r=LLAMA8B_R, K=K, N=N, M=M, outliers=np.nonzero(mult != 1.0)[0])


def stress(frac: float, rows: int | None = None, w_rows: int | None = None, row0: int = 0):
    c = STRESS
    t = list(c["fracs"]).index(frac)
    K = c["K"]
    M = c["M"] if rows is None else rows
    n_out = int(round(frac * K))
    mult = outlier_multipliers(c["seed"], t, K, n_out, 10.0, 200.0)
    x = matrix_bf16(c["seed"], stream_id(t, 1), M, K, 1.0, dist="t3", col_mult=mult, row0=row0)
    w = matrix_bf16(c["seed"], stream_id(0, 2), c["N"] if w_rows is None else w_rows, K, 0.02)
    return dict(x=x, w=w, K=K, N=c["N"], M=M, outliers=np.nonzero(mult != 1.0)[0])


def recurrent(S: int | None = None, d: int | None = None, ffn: int | None = None):
    """Hidden state and the two sublayers' weights (gate|up fused [2*ffn, d], down [d, ffn])."""
    c = RECURRENT
    S = S or c["S"]
    d = d or c["d"]
    ffn = ffn or c["ffn"]
    seed = c["seed"]
    std = 0.02 / math.sqrt(c["T"])
    h = matrix_bf16(seed, stream_id(0, 1), S, d, 1.0)
    layers = []
    for s in range(2):
        wgu = matrix_bf16(seed, stream_id(1 + 2 * s, 2), 2 * ffn, d, std)
        wd = matrix_bf16(seed, stream_id(2 + 2 * s, 2), d, ffn, std)
        layers.append(dict(wgu=wgu, wd=wd, gain=np.full(d, 0x3F80, np.uint16)))
    return dict(h=h, layers=layers, S=S, d=d, ffn=ffn, T=c["T"], r=c["r"], eps=c["eps"])


def mlp70b(proj: str, rows: int | None = None, row0: int = 0, with_w: bool = True, w_rows: int | None = None):
    t, K, N = MLP70B_PROJ[proj]
    seed = 4
    M = MLP70B_M if rows is None else rows
    n_out = int(round(0.005 * K))
    mult = outlier_multipliers(seed, t, K, n_out, 50.0, 50.0)
    x = matrix_bf16(seed, stream_id(t, 1), M, K, 1.0, col_mult=mult, row0=row0)
    w = matrix_bf16(seed, stream_id(t, 2), N if w_rows is None else w_rows, K, 0.015) if with_w else None
    return dict(x=x, w=w, r=MLP70B_R, K=K, N=N, M=M, outliers=np.nonzero(mult != 1.0)[0])
