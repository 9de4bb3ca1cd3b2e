"""CPU oracle for the NVFP4 + augmented-residual-channel path (test infrastructure).

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` import
this package. It wraps ``arc_oracle.c`` (plain C, IEEE fp32 with no FMA contraction, FP64 / exact
int64 GEMM sums) through ctypes and splits rows across threads. It shares no code with the CUDA
library and never calls it.

Every function names the passage it follows in the C source. The pages are:
  * "ARCQuant: Boosting NVFP4 Quantization with Augmented Residual Channels for LLMs",
    Methodologie (outlier identification, dual-stage quantization, augmented matrix
    multiplication, unified GEMM, fused kernel);
  * "Day 0 LLM Inference Support: Hierarchical Quantization and Memory Access Optimization
    Practices", section V (numerical safety, per-group quantization pseudo-code);
  * "RAMP: Recurrent Adaptive Mixed Precision for Efficient Prefill in Recurrent-Depth Language
    Models", sections 2.1, 4.1, 4.2 (recurrent block, precision switch, BF16 hidden state).

Parity unpinned (no check against the pages or mathematics is possible): none of the functions
here; the recurrent fidelity figure (final hidden-state error of a mixed schedule) is reported,
not pinned.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "arc_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile arc_oracle.c into liboracle.so next to it (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I64 = ctypes.c_int64
            I32 = ctypes.c_int32
            F = ctypes.c_float
            D = ctypes.c_double
            sig = {
                "oracle_e2m1_encode": (ctypes.c_uint8, [F]),
                "oracle_e2m1_decode": (F, [ctypes.c_uint8]),
                "oracle_e4m3_encode_nonneg": (ctypes.c_uint8, [F]),
                "oracle_e4m3_decode": (F, [ctypes.c_uint8]),
                "oracle_tensor_scale": (F, [F]),
                "oracle_amax_bf16": (F, [P, I64, I64, I64]),
                "oracle_kpad": (I64, [I64]),
                "oracle_encode_block": (None, [P, F, P, P, P]),
                "oracle_row_sumsq": (D, [P, I64]),
                "oracle_rms_inv": (D, [P, I64, D]),
                "oracle_rmsnorm_rows": (None, [P, I64, I64, P, D, P, I64, I64, I64]),
                "oracle_quantize_act_rows": (None, [P, I64, I64, P, I32, P, I32, D, F, P, P, P, I64, I64]),
                "oracle_pack_weight_rows": (None, [P, I64, I64, P, I32, F, P, P, I64, I64]),
                "oracle_dequant_rows": (None, [P, P, I64, P, I64, I64]),
                "oracle_sf_swizzled_bytes": (I64, [I64, I64]),
                "oracle_sf_swizzle": (None, [P, I64, I64, P]),
                "oracle_sf_unswizzle": (None, [P, I64, I64, P]),
                "oracle_gemm_nvfp4_f64": (None, [P, P, F, P, P, F, I64, I64, P, I64, I64, I64, P]),
                "oracle_quantize_mxfp4_arc_rows": (None, [P, I64, I64, P, I32, I32, P, P, P, I64, I64]),
                "oracle_gemm_nvfp4_i64": (None, [P, P, P, P, I64, I64, P, I64, I64, I64, P]),
                "oracle_gemm_bf16_f64": (None, [P, I64, P, I64, I64, I64, P, I64, P]),
                "oracle_channel_absmax": (None, [P, I64, I64, I64, P]),
                "oracle_top_channels": (None, [P, I64, I32, P]),
                "oracle_silu_mul_rows": (None, [P, I64, I64, P, I64, I64, I64]),
                "oracle_e2m1_encode_array": (None, [P, I64, P]),
                "oracle_e4m3_encode_array": (None, [P, I64, P]),
                "oracle_fp8_scale": (F, [F]),
                "oracle_mxfp4_scale_byte": (ctypes.c_uint8, [F]),
                "oracle_quantize_mxfp4_rows": (None, [P, I64, I64, P, P, I64, I64]),
                "oracle_gemm_mxfp4_f64": (None, [P, P, P, P, I64, I64, P, I64, P]),
                "oracle_e4m3_encode_signed": (ctypes.c_uint8, [F]),
                "oracle_quantize_fp8_rows": (None, [P, I64, I64, F, P, I64, I64, I64]),
                "oracle_e4m3_decode_array": (None, [P, I64, P]),
                "oracle_e2m1_decode_array": (None, [P, I64, P]),
                "oracle_e2m1_of_quotient_array": (None, [P, I64, F, P]),
                "oracle_bf16_to_f32": (F, [ctypes.c_uint16]),
                "oracle_f32_to_bf16": (ctypes.c_uint16, [F]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
            _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _threads() -> int:
    return int(os.environ.get("ARC_ORACLE_THREADS", os.cpu_count() or 1))


def _split_rows(nrows: int, fn, min_rows: int = 1):
    """Run fn(r0, r1) over row chunks on a thread pool (ctypes releases the GIL)."""
    t = max(1, min(_threads(), (nrows + min_rows - 1) // min_rows))
    if t == 1 or nrows <= 1:
        fn(0, nrows)
        return
    step = (nrows + t - 1) // t
    with ThreadPoolExecutor(max_workers=t) as ex:
        futs = [ex.submit(fn, r0, min(nrows, r0 + step)) for r0 in range(0, nrows, step)]
        for f in futs:
            f.result()


def as_u16(x) -> np.ndarray:
    """bf16 data as uint16 bits (accepts numpy uint16/int16 or a CPU torch bfloat16 tensor)."""
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x.view(np.uint16))
    import torch

    assert x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return np.ascontiguousarray(x.contiguous().view(torch.int16).numpy().view(np.uint16))


def kpad(k_aug: int) -> int:
    return (k_aug + 63) // 64 * 64


# --------------------------------------------------------------------------------------------
# Element codecs (arc_oracle.c: E2M1 / E4M3 sections)
# --------------------------------------------------------------------------------------------

def e2m1_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e2m1_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e2m1_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, dtype=np.uint8))
    out = np.empty(c.shape, np.float32)
    lib().oracle_e2m1_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def e4m3_encode(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode(c) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(c, dtype=np.uint8))
    out = np.empty(c.shape, np.float32)
    lib().oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def e2m1_of_quotient(x, d: float) -> np.ndarray:
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, np.uint8)
    lib().oracle_e2m1_of_quotient_array(_ptr(x), x.size, float(np.float32(d)), _ptr(out))
    return out


def encode_block(x16, s_t: float):
    """One 16-element block -> (codes[16], sf byte, decode scale d)."""
    x16 = np.ascontiguousarray(np.asarray(x16, dtype=np.float32))
    assert x16.size == 16
    codes = np.zeros(16, np.uint8)
    sf = np.zeros(1, np.uint8)
    d = np.zeros(1, np.float32)
    lib().oracle_encode_block(_ptr(x16), float(np.float32(s_t)), _ptr(codes), _ptr(sf), _ptr(d))
    return codes, int(sf[0]), float(d[0])


# --------------------------------------------------------------------------------------------
# Tensor scale, amax, calibration
# --------------------------------------------------------------------------------------------

def amax(x) -> float:
    x = as_u16(x)
    rows, cols = x.shape
    parts = []

    def run(r0, r1):
        parts.append(lib().oracle_amax_bf16(_ptr(x[r0:r1]) if r1 > r0 else _ptr(x), r1 - r0, cols, cols))

    _split_rows(rows, run, min_rows=64)
    return float(np.float32(max(parts) if parts else 0.0))


def tensor_scale(amax_value: float) -> float:
    return float(lib().oracle_tensor_scale(float(np.float32(amax_value))))


def channel_absmax(x) -> np.ndarray:
    x = as_u16(x)
    rows, cols = x.shape
    out = np.zeros(cols, np.float32)
    lib().oracle_channel_absmax(_ptr(x), rows, cols, cols, _ptr(out))
    return out


def calibrate(x, r: int) -> np.ndarray:
    """Top-r channels by calibration abs-max, descending, ties by ascending index."""
    a = channel_absmax(x)
    idx = np.zeros(max(r, 1), np.int32)
    lib().oracle_top_channels(_ptr(a), a.size, int(r), _ptr(idx))
    return idx[:r].copy()


def calibrate_order(x) -> np.ndarray:
    """All K channels ordered by calibration abs-max, descending, ties by ascending index: the
    channel reorder of ARCQuant's adaptive outlier identification ("reorders the channels by
    their absolute maxima and selects a top-S subset", Methodologie). The first r entries are
    calibrate(x, r)."""
    x = as_u16(x)
    return calibrate(x, x.shape[1])


# --------------------------------------------------------------------------------------------
# Quantization (arc_oracle.c: activation quantization with augmented residual channels)
# --------------------------------------------------------------------------------------------

def quantize_act(x, idx, s_t: float, rms_gain=None, use_rms: bool = False, eps: float = 1e-6,
                 want_residual: bool = False):
    """X [M, K] bf16 -> (codes [M, K_pad/2] u8, canonical sf [M, K_pad/16] u8[, res [M, r] f32])."""
    x = as_u16(x)
    M, K = x.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
    r = idx.size
    kp = kpad(K + r)
    codes = np.zeros((M, kp // 2), np.uint8)
    sf = np.zeros((M, kp // 16), np.uint8)
    res = np.zeros((M, r), np.float32) if (want_residual and r > 0) else None
    g = None
    if rms_gain is not None:
        g = as_u16(rms_gain).reshape(-1)
        use_rms = True
    L = lib()

    def run(r0, r1):
        L.oracle_quantize_act_rows(_ptr(x), K, K, _ptr(idx) if r else None, r,
                                   _ptr(g) if g is not None else None, 1 if use_rms else 0, float(eps),
                                   float(np.float32(s_t)), _ptr(codes), _ptr(sf),
                                   _ptr(res) if res is not None else None, r0, r1)

    _split_rows(M, run, min_rows=16)
    if want_residual:
        return codes, sf, (res if res is not None else np.zeros((M, 0), np.float32))
    return codes, sf


def pack_weight(w, idx, s_w: float):
    """W [N, K] bf16 -> W_aug = [W | W[:, idx]] as (codes [N, K_pad/2], canonical sf [N, K_pad/16])."""
    w = as_u16(w)
    N, K = w.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
    r = idx.size
    kp = kpad(K + r)
    codes = np.zeros((N, kp // 2), np.uint8)
    sf = np.zeros((N, kp // 16), np.uint8)
    L = lib()

    def run(r0, r1):
        L.oracle_pack_weight_rows(_ptr(w), K, K, _ptr(idx) if r else None, r, float(np.float32(s_w)),
                                  _ptr(codes), _ptr(sf), r0, r1)

    _split_rows(N, run, min_rows=16)
    return codes, sf


def quantize_act_reordered(x, perm, r: int, s_t: float, rms_gain=None, use_rms: bool = False,
                           eps: float = 1e-6, want_residual: bool = False):
    """Dual-stage quantization of the reordered activation (ARCQuant, Methodologie: the primary
    stage quantizes the reordered input block-wise, the residual stage the top-S outlier
    channels). Primary channel p of the output is input channel perm[p]; the outlier channels
    are perm[:r], i.e. the first r columns of the reordered X, so this is quantize_act of
    X[:, perm] with idx = 0..r-1 (an RMSNorm gain is reordered with X; the row statistics do not
    depend on the channel order)."""
    x = as_u16(x)
    perm = np.ascontiguousarray(np.asarray(perm, dtype=np.int64).reshape(-1))
    assert perm.size == x.shape[1] and 0 <= r <= perm.size
    g = None if rms_gain is None else as_u16(rms_gain).reshape(-1)[perm]
    return quantize_act(np.ascontiguousarray(x[:, perm]), np.arange(r, dtype=np.int32), s_t, rms_gain=g,
                        use_rms=use_rms, eps=eps, want_residual=want_residual)


def pack_weight_reordered(w, perm, r: int, s_w: float):
    """W_aug = [W[:, perm] | W[:, perm[:r]]] packed as NVFP4: the weight side of the reordered
    augmented GEMM (ARCQuant, Methodologie: weights reordered like the activation and their
    outlier columns duplicated)."""
    w = as_u16(w)
    perm = np.ascontiguousarray(np.asarray(perm, dtype=np.int64).reshape(-1))
    assert perm.size == w.shape[1] and 0 <= r <= perm.size
    return pack_weight(np.ascontiguousarray(w[:, perm]), np.arange(r, dtype=np.int32), s_w)


def fp8_scale(amax_value: float) -> float:
    """Per-tensor FP8 scale amax / 448 with the all-zero guard (arc_oracle.c, FP8 W8A8)."""
    return float(lib().oracle_fp8_scale(float(np.float32(amax_value))))


def e4m3_encode_signed(v) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32)).reshape(-1)
    L = lib()
    return np.array([L.oracle_e4m3_encode_signed(float(t)) for t in v], np.uint8)


def quantize_fp8(x, s: float) -> np.ndarray:
    """X [M, K] bf16 -> E4M3 codes [M, K] of x / s (RAMP's FP8 weights and activations with one
    per-tensor scale; arc_oracle.c, FP8 W8A8)."""
    x = as_u16(x)
    M, K = x.shape
    codes = np.zeros((M, K), np.uint8)
    L = lib()

    def run(r0, r1):
        L.oracle_quantize_fp8_rows(_ptr(x), K, K, float(np.float32(s)), _ptr(codes), K, r0, r1)

    _split_rows(M, run, min_rows=16)
    return codes


def gemm_fp8_f64(a_codes, s_a: float, b_codes, s_b: float, rows=None) -> np.ndarray:
    """Y = (s_a s_b) * E4M3(A) E4M3(B)^T in FP64 (a library matmul of the decoded operands)."""
    a = np.ascontiguousarray(a_codes if rows is None else a_codes[rows])
    A = e4m3_decode(a).astype(np.float64)
    B = e4m3_decode(np.ascontiguousarray(b_codes)).astype(np.float64)
    return (float(np.float32(s_a)) * float(np.float32(s_b))) * (A @ B.T)


def mxfp4_scale_byte(amax_block: float) -> int:
    """E8M0 scale byte of a 32-value MXFP4 block with abs-max amax_block (arc_oracle.c, MXFP4)."""
    return int(lib().oracle_mxfp4_scale_byte(float(np.float32(amax_block))))


def quantize_mxfp4(x):
    """X [M, K] bf16 -> MXFP4 (OCP microscaling reading of ARCQuant's MXFP4 extension): codes
    [M, K/2] (element k at byte k/2, low nibble for even k) and E8M0 scale bytes [M, K/32]."""
    x = as_u16(x)
    M, K = x.shape
    assert K % 32 == 0
    codes = np.zeros((M, K // 2), np.uint8)
    scales = np.zeros((M, K // 32), np.uint8)
    L = lib()

    def run(r0, r1):
        L.oracle_quantize_mxfp4_rows(_ptr(x), K, K, _ptr(codes), _ptr(scales), r0, r1)

    _split_rows(M, run, min_rows=16)
    return codes, scales


def _mxfp4_arc(x, idx, dup: bool, want_residual: bool = False):
    x = as_u16(x)
    M, K = x.shape
    idx = np.ascontiguousarray(np.asarray(idx, dtype=np.int32).reshape(-1))
    r = idx.size
    assert K % 32 == 0 and r % 32 == 0 and r <= K
    kp = kpad(K + r)
    codes = np.zeros((M, kp // 2), np.uint8)
    scales = np.zeros((M, kp // 32), np.uint8)
    res = np.zeros((M, r), np.float32) if (want_residual and r > 0) else None
    L = lib()

    def run(r0, r1):
        L.oracle_quantize_mxfp4_arc_rows(_ptr(x), K, K, _ptr(idx) if r else None, r, 1 if dup else 0, _ptr(codes),
                                         _ptr(scales), _ptr(res) if res is not None else None, r0, r1)

    _split_rows(M, run, min_rows=16)
    if want_residual:
        return codes, scales, (res if res is not None else np.zeros((M, 0), np.float32))
    return codes, scales


def quantize_act_mxfp4(x, idx, want_residual: bool = False):
    """MXFP4 with augmented residual channels (arc_oracle.c, MXFP4 with augmented residual
    channels): X [M, K] bf16 -> (codes [M, K_pad/2], canonical E8M0 scale bytes [M, K_pad/32]
    [, residuals [M, r] f32]); K and r multiples of 32."""
    return _mxfp4_arc(x, idx, dup=False, want_residual=want_residual)


def pack_weight_mxfp4(w, idx):
    """W_aug = [W | W[:, idx]] in MXFP4: (codes [N, K_pad/2], canonical scale bytes [N, K_pad/32])."""
    return _mxfp4_arc(w, idx, dup=True)


def gemm_mxfp4_f64(a_codes, a_scales, b_codes, b_scales, rows=None) -> np.ndarray:
    """Y[rows, N] = sum_k E2M1(a) 2^(sa-127) E2M1(b) 2^(sb-127) in FP64."""
    a_codes, a_scales = np.ascontiguousarray(a_codes), np.ascontiguousarray(a_scales)
    b_codes, b_scales = np.ascontiguousarray(b_codes), np.ascontiguousarray(b_scales)
    M, K = a_codes.shape[0], a_codes.shape[1] * 2
    N = b_codes.shape[0]
    rows = _rows_arg(rows, M)
    y = np.zeros((rows.size, N), np.float64)
    L = lib()

    def run(t0, t1):
        L.oracle_gemm_mxfp4_f64(_ptr(a_codes), _ptr(a_scales), _ptr(b_codes), _ptr(b_scales), N, K,
                                _ptr(rows[t0:t1]) if t1 > t0 else None, t1 - t0,
                                y[t0:].ctypes.data_as(ctypes.c_void_p))

    _split_rows(rows.size, run)
    return y


def dequant(codes, sf) -> np.ndarray:
    """Canonical codes/sf -> fp32 values without the tensor scale."""
    codes = np.ascontiguousarray(codes)
    sf = np.ascontiguousarray(sf)
    rows, half = codes.shape
    kp = half * 2
    out = np.zeros((rows, kp), np.float32)
    lib().oracle_dequant_rows(_ptr(codes), _ptr(sf), kp, _ptr(out), 0, rows)
    return out


def sf_swizzle(canon) -> np.ndarray:
    canon = np.ascontiguousarray(canon, dtype=np.uint8)
    rows, nsf = canon.shape
    out = np.zeros(lib().oracle_sf_swizzled_bytes(rows, nsf), np.uint8)
    lib().oracle_sf_swizzle(_ptr(canon), rows, nsf, _ptr(out))
    return out


def sf_unswizzle(swz, rows: int, nsf: int) -> np.ndarray:
    swz = np.ascontiguousarray(np.asarray(swz, dtype=np.uint8).reshape(-1))
    assert swz.size >= lib().oracle_sf_swizzled_bytes(rows, nsf)
    out = np.zeros((rows, nsf), np.uint8)
    lib().oracle_sf_unswizzle(_ptr(swz), rows, nsf, _ptr(out))
    return out


def sf_swizzled_bytes(rows: int, nsf: int) -> int:
    return int(lib().oracle_sf_swizzled_bytes(rows, nsf))


# --------------------------------------------------------------------------------------------
# GEMMs
# --------------------------------------------------------------------------------------------

def _rows_arg(rows, M):
    if rows is None:
        rows = np.arange(M, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))


def gemm_nvfp4_f64(a_codes, a_sf, s_a, b_codes, b_sf, s_b, rows=None, k_range=None) -> np.ndarray:
    """Y[rows, N] = s_A s_W sum_k deqA deqB over K_aug, FP64 (canonical sf)."""
    a_codes = np.ascontiguousarray(a_codes)
    a_sf = np.ascontiguousarray(a_sf)
    b_codes = np.ascontiguousarray(b_codes)
    b_sf = np.ascontiguousarray(b_sf)
    M = a_codes.shape[0]
    N = b_codes.shape[0]
    kp = a_codes.shape[1] * 2
    assert b_codes.shape[1] * 2 == kp
    rows = _rows_arg(rows, M)
    k_lo, k_hi = (0, kp) if k_range is None else k_range
    y = np.zeros((rows.size, N), np.float64)
    L = lib()

    def run(t0, t1):
        L.oracle_gemm_nvfp4_f64(_ptr(a_codes), _ptr(a_sf), float(np.float32(s_a)), _ptr(b_codes), _ptr(b_sf),
                                float(np.float32(s_b)), N, kp, _ptr(rows[t0:t1]) if t1 > t0 else None,
                                t1 - t0, k_lo, k_hi, y[t0:].ctypes.data_as(ctypes.c_void_p))

    _split_rows(rows.size, run)
    return y


def gemm_nvfp4_f64_matmul(a_codes, a_sf, s_a, b_codes, b_sf, s_b, rows=None) -> np.ndarray:
    """Same result as gemm_nvfp4_f64 with a library matmul as the summation step: operands are
    dequantized exactly (E2M1 * E4M3 products are exact in fp32), then an FP64 matmul."""
    a_codes = np.ascontiguousarray(a_codes)
    M = a_codes.shape[0]
    rows = _rows_arg(rows, M)
    A = dequant(np.ascontiguousarray(a_codes[rows]), np.ascontiguousarray(np.asarray(a_sf)[rows])).astype(np.float64)
    B = dequant(b_codes, b_sf).astype(np.float64)
    return (np.float64(np.float32(s_a)) * np.float64(np.float32(s_b))) * (A @ B.T)


def gemm_nvfp4_i64(a_codes, a_sf, b_codes, b_sf, rows=None, k_range=None) -> np.ndarray:
    """Exact integer sums sum_k a'b' (a' = 2 E2M1 * 512 E4M3); Y = sum * 2^-20 * s_A s_W."""
    a_codes = np.ascontiguousarray(a_codes)
    a_sf = np.ascontiguousarray(a_sf)
    b_codes = np.ascontiguousarray(b_codes)
    b_sf = np.ascontiguousarray(b_sf)
    M = a_codes.shape[0]
    N = b_codes.shape[0]
    kp = a_codes.shape[1] * 2
    rows = _rows_arg(rows, M)
    k_lo, k_hi = (0, kp) if k_range is None else k_range
    y = np.zeros((rows.size, N), np.int64)
    L = lib()

    def run(t0, t1):
        L.oracle_gemm_nvfp4_i64(_ptr(a_codes), _ptr(a_sf), _ptr(b_codes), _ptr(b_sf), N, kp,
                                _ptr(rows[t0:t1]) if t1 > t0 else None, t1 - t0, k_lo, k_hi,
                                y[t0:].ctypes.data_as(ctypes.c_void_p))

    _split_rows(rows.size, run)
    return y


def gemm_bf16_f64(x, w, rows=None) -> np.ndarray:
    """Y[rows, N] = X W^T over bf16 inputs, FP64 sums."""
    x = as_u16(x)
    w = as_u16(w)
    M, K = x.shape
    N = w.shape[0]
    rows = _rows_arg(rows, M)
    y = np.zeros((rows.size, N), np.float64)
    L = lib()

    def run(t0, t1):
        L.oracle_gemm_bf16_f64(_ptr(x), K, _ptr(w), K, N, K, _ptr(rows[t0:t1]) if t1 > t0 else None, t1 - t0,
                               y[t0:].ctypes.data_as(ctypes.c_void_p))

    _split_rows(rows.size, run)
    return y


# --------------------------------------------------------------------------------------------
# Recurrent block pieces
# --------------------------------------------------------------------------------------------

def row_sumsq(h_row) -> float:
    h = as_u16(h_row).reshape(-1)
    return float(lib().oracle_row_sumsq(_ptr(h), h.size))


def rmsnorm(h, gain=None, eps: float = 1e-6) -> np.ndarray:
    """bf16 RMSNorm rows (exact sum of squares, double inverse root), returns uint16 bits."""
    h = as_u16(h)
    M, d = h.shape
    g = as_u16(gain).reshape(-1) if gain is not None else None
    out = np.zeros((M, d), np.uint16)
    L = lib()

    def run(r0, r1):
        L.oracle_rmsnorm_rows(_ptr(h), d, d, _ptr(g) if g is not None else None, float(eps), _ptr(out), d, r0, r1)

    _split_rows(M, run, min_rows=16)
    return out


def silu_mul(gu) -> np.ndarray:
    """[M, 2F] gate|up bf16 -> [M, F] bf16 bits of silu(gate) * up."""
    gu = as_u16(gu)
    M, F2 = gu.shape
    F = F2 // 2
    out = np.zeros((M, F), np.uint16)
    L = lib()

    def run(r0, r1):
        L.oracle_silu_mul_rows(_ptr(gu), F, F2, _ptr(out), F, r0, r1)

    _split_rows(M, run, min_rows=16)
    return out


def f64_to_bf16_bits(y: np.ndarray) -> np.ndarray:
    """Round FP64 results to bf16 (via fp32, both round-to-nearest-even)."""
    f = np.ascontiguousarray(y.astype(np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
