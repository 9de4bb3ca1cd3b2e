"""Python binding of the B200 NVFP4 + augmented-residual-channel library (libarc.so).

Argument marshalling only: every step of the path runs in the library's CUDA kernels. PyTorch
provides device memory and streams. There is no fallback: if libarc.so is missing or the GPU is
not an sm_100 device, calls raise.

The C ABI is documented in include/arc.h; the functions below carry the same names without the
``arc_`` prefix and allocate their outputs (and scratch) with torch when none are passed.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libarc.so")
_lib = None

ARC_STATUS = {0: "ARC_OK", 1: "ARC_ERR_INVALID_ARG", 2: "ARC_ERR_ALIGNMENT", 3: "ARC_ERR_UNSUPPORTED",
              4: "ARC_ERR_CUDA", 5: "ARC_ERR_TIMEOUT", 6: "ARC_ERR_WORKSPACE"}


class ArcError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} failed: {ARC_STATUS.get(code, code)}")
        self.code = code


class SwigluSublayer(ctypes.Structure):
    _fields_ = [
        ("rms_gain_bf16", ctypes.c_void_p), ("w_gateup_bf16", ctypes.c_void_p), ("w_down_bf16", ctypes.c_void_p),
        ("gateup_codes", ctypes.c_void_p), ("gateup_sf", ctypes.c_void_p), ("gateup_scale", ctypes.c_void_p),
        ("down_codes", ctypes.c_void_p), ("down_sf", ctypes.c_void_p), ("down_scale", ctypes.c_void_p),
        ("idx_gateup", ctypes.c_void_p), ("r_gateup", ctypes.c_int32),
        ("idx_down", ctypes.c_void_p), ("r_down", ctypes.c_int32),
        ("gateup_fp8", ctypes.c_void_p), ("gateup_fp8_scale", ctypes.c_void_p),
        ("down_fp8", ctypes.c_void_p), ("down_fp8_scale", ctypes.c_void_p),
    ]


class SwigluBlock(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int64), ("ffn", ctypes.c_int64), ("eps", ctypes.c_float),
                ("n_sublayers", ctypes.c_int32), ("sublayers", ctypes.POINTER(SwigluSublayer)),
                ("residual_scale", ctypes.c_float), ("inject_bf16", ctypes.c_void_p)]


STEP_BF16, STEP_NVFP4, STEP_FP8 = 0, 1, 2  # per-step formats of arc_recurrent_prefill_schedule


_SIGS = {
    "arc_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "arc_kpad": (ctypes.c_int64, [ctypes.c_int64]),
    "arc_nvfp4_codes_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "arc_nvfp4_sf_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "arc_quantize_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int32]),
    "arc_calibrate_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64]),
    "arc_quantize_act_nvfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_float,
                                              ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_pack_weight_nvfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_calibrate_outliers": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t,
                                              ctypes.c_void_p]),
    "arc_calibrate_order": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                           ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_quantize_act_nvfp4_reordered": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                        ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32,
                                                        ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_pack_weight_nvfp4_reordered": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                       ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32,
                                                       ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                       ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_gemm_nvfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.c_void_p]),
    "arc_mxfp4_sf_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int64]),
    "arc_quantize_act_mxfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                              ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                              ctypes.c_void_p]),
    "arc_pack_weight_mxfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                             ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p,
                                             ctypes.c_void_p]),
    "arc_gemm_mxfp4": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]),
    "arc_gemm_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_int64, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                     ctypes.c_int64, ctypes.c_void_p]),
    "arc_rmsnorm_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p, ctypes.c_int64,
                                        ctypes.c_void_p]),
    "arc_silu_mul_bf16": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                         ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p]),
    "arc_recurrent_workspace_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.POINTER(SwigluBlock)]),
    "arc_recurrent_prefill": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.POINTER(SwigluBlock),
                                             ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p, ctypes.c_size_t,
                                             ctypes.c_void_p]),
    "arc_recurrent_prefill_schedule": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64,
                                                      ctypes.POINTER(SwigluBlock), ctypes.c_int32,
                                                      ctypes.POINTER(ctypes.c_uint8), ctypes.c_void_p,
                                                      ctypes.c_size_t, ctypes.c_void_p]),
    "arc_quantize_fp8": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64,
                                        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                        ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p]),
    "arc_gemm_fp8": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                    ctypes.c_int64, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
                                    ctypes.c_int64, ctypes.c_void_p]),
    "arc_last_device_status": (ctypes.c_int, [ctypes.c_void_p]),
    "arc_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64]),
    "arc_debug_inject": (ctypes.c_int, [ctypes.c_int32]),
    "arc_quantize_act_nvfp4_static_scratch": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                                                             ctypes.c_int64, ctypes.c_void_p, ctypes.c_int32,
                                                             ctypes.c_void_p, ctypes.c_float, ctypes.c_void_p,
                                                             ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                                             ctypes.c_void_p]),
}


def lib() -> ctypes.CDLL:
    """Load libarc.so (built in-tree by __graft_entry__.build()); raise if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run __graft_entry__.build() (nvcc, sm_100a)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def exported_symbols() -> list[str]:
    return list(_SIGS)


def _check(fn: str, code: int):
    if code != 0:
        raise ArcError(fn, code)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("arc: tensors must be CUDA tensors")


def kpad(k_aug: int) -> int:
    return int(lib().arc_kpad(k_aug))


def codes_bytes(rows: int, k_aug: int) -> int:
    return int(lib().arc_nvfp4_codes_bytes(rows, k_aug))


def sf_bytes(rows: int, k_aug: int) -> int:
    return int(lib().arc_nvfp4_sf_bytes(rows, k_aug))


def quantize_workspace_bytes(rows: int, r: int) -> int:
    return int(lib().arc_quantize_workspace_bytes(rows, r))


def _u8(n: int, device):
    return torch.empty(max(n, 16), dtype=torch.uint8, device=device)


def _ws(n: int, device):
    # torch's caching allocator returns 512-byte aligned blocks
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device)


@dataclass
class NVFP4Tensor:
    """Packed NVFP4 operand: codes [rows, K_pad/2] u8, swizzled scale bytes, fp32 tensor scale."""
    codes: torch.Tensor
    sf: torch.Tensor
    scale: torch.Tensor
    rows: int
    k_aug: int


def quantize_act_nvfp4(x: torch.Tensor, idx: torch.Tensor | None = None, rms_gain: torch.Tensor | None = None,
                       eps: float = 1e-6, static_scale: torch.Tensor | None = None, out: NVFP4Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None) -> NVFP4Tensor:
    """arc_quantize_act_nvfp4: X [M, K] bf16 (row stride x.stride(0)) -> NVFP4 with r appended channels."""
    _need_cuda(x, idx, rms_gain, static_scale)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    r = 0 if idx is None else int(idx.numel())
    if out is None:
        out = NVFP4Tensor(_u8(codes_bytes(M, K + r), x.device), _u8(sf_bytes(M, K + r), x.device),
                          torch.empty(1, dtype=torch.float32, device=x.device), M, K + r)
    nws = quantize_workspace_bytes(M, r)
    if workspace is None:
        workspace = _ws(nws, x.device)
    _check("arc_quantize_act_nvfp4", lib().arc_quantize_act_nvfp4(
        _p(x), M, K, x.stride(0), _p(idx), r, _p(rms_gain), float(eps), _p(static_scale), _p(out.codes),
        _p(out.sf), _p(out.scale), _p(workspace), workspace.numel(), _stream(stream)))
    return out


def pack_weight_nvfp4(w: torch.Tensor, idx: torch.Tensor | None = None, out: NVFP4Tensor | None = None,
                      workspace: torch.Tensor | None = None, stream=None) -> NVFP4Tensor:
    """arc_pack_weight_nvfp4: W [N, K] bf16 -> NVFP4 of [W | W[:, idx]] with its own tensor scale."""
    _need_cuda(w, idx)
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    N, K = w.shape
    r = 0 if idx is None else int(idx.numel())
    if out is None:
        out = NVFP4Tensor(_u8(codes_bytes(N, K + r), w.device), _u8(sf_bytes(N, K + r), w.device),
                          torch.empty(1, dtype=torch.float32, device=w.device), N, K + r)
    nws = quantize_workspace_bytes(N, r)
    if workspace is None:
        workspace = _ws(nws, w.device)
    _check("arc_pack_weight_nvfp4", lib().arc_pack_weight_nvfp4(
        _p(w), N, K, w.stride(0), _p(idx), r, _p(out.codes), _p(out.sf), _p(out.scale), _p(workspace),
        workspace.numel(), _stream(stream)))
    return out


def calibrate_outliers(x: torch.Tensor, r: int, stream=None) -> torch.Tensor:
    """arc_calibrate_outliers: top-r channels of X by abs-max (device int32[r])."""
    _need_cuda(x)
    M, K = x.shape
    idx = torch.empty(r, dtype=torch.int32, device=x.device)
    ws = _ws(int(lib().arc_calibrate_workspace_bytes(K)), x.device)
    _check("arc_calibrate_outliers", lib().arc_calibrate_outliers(_p(x), M, K, x.stride(0), r, _p(idx), _p(ws),
                                                                  ws.numel(), _stream(stream)))
    return idx


def calibrate_order(x: torch.Tensor, stream=None) -> torch.Tensor:
    """arc_calibrate_order: all K channels of X by descending abs-max (device int32[K])."""
    _need_cuda(x)
    M, K = x.shape
    perm = torch.empty(K, dtype=torch.int32, device=x.device)
    ws = _ws(int(lib().arc_calibrate_workspace_bytes(K)), x.device)
    _check("arc_calibrate_order", lib().arc_calibrate_order(_p(x), M, K, x.stride(0), _p(perm), _p(ws), ws.numel(),
                                                            _stream(stream)))
    return perm


def quantize_act_nvfp4_reordered(x: torch.Tensor, perm: torch.Tensor, r: int, rms_gain: torch.Tensor | None = None,
                                 eps: float = 1e-6, static_scale: torch.Tensor | None = None,
                                 out: NVFP4Tensor | None = None, workspace: torch.Tensor | None = None,
                                 stream=None) -> NVFP4Tensor:
    """arc_quantize_act_nvfp4_reordered: X [M, K] bf16 -> NVFP4 of X[:, perm] with the residuals of
    the r channels perm[:r] appended."""
    _need_cuda(x, perm, rms_gain, static_scale)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    assert perm.dtype == torch.int32 and perm.numel() == x.shape[1]
    M, K = x.shape
    if out is None:
        out = NVFP4Tensor(_u8(codes_bytes(M, K + r), x.device), _u8(sf_bytes(M, K + r), x.device),
                          torch.empty(1, dtype=torch.float32, device=x.device), M, K + r)
    if workspace is None:
        workspace = _ws(quantize_workspace_bytes(M, r), x.device)
    _check("arc_quantize_act_nvfp4_reordered", lib().arc_quantize_act_nvfp4_reordered(
        _p(x), M, K, x.stride(0), _p(perm), int(r), _p(rms_gain), float(eps), _p(static_scale), _p(out.codes),
        _p(out.sf), _p(out.scale), _p(workspace), workspace.numel(), _stream(stream)))
    return out


def pack_weight_nvfp4_reordered(w: torch.Tensor, perm: torch.Tensor, r: int, out: NVFP4Tensor | None = None,
                                workspace: torch.Tensor | None = None, stream=None) -> NVFP4Tensor:
    """arc_pack_weight_nvfp4_reordered: W [N, K] bf16 -> NVFP4 of [W[:, perm] | W[:, perm[:r]]]."""
    _need_cuda(w, perm)
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    assert perm.dtype == torch.int32 and perm.numel() == w.shape[1]
    N, K = w.shape
    if out is None:
        out = NVFP4Tensor(_u8(codes_bytes(N, K + r), w.device), _u8(sf_bytes(N, K + r), w.device),
                          torch.empty(1, dtype=torch.float32, device=w.device), N, K + r)
    if workspace is None:
        workspace = _ws(quantize_workspace_bytes(N, r), w.device)
    _check("arc_pack_weight_nvfp4_reordered", lib().arc_pack_weight_nvfp4_reordered(
        _p(w), N, K, w.stride(0), _p(perm), int(r), _p(out.codes), _p(out.sf), _p(out.scale), _p(workspace),
        workspace.numel(), _stream(stream)))
    return out


def gemm_nvfp4(a: NVFP4Tensor, b: NVFP4Tensor, out: torch.Tensor | None = None, add: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """arc_gemm_nvfp4: Y [M, N] bf16 = s_A s_B * A_aug B_aug^T (+ add)."""
    assert a.k_aug == b.k_aug, "A and B must share the augmented depth K + r"
    M, N = a.rows, b.rows
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _check("arc_gemm_nvfp4", lib().arc_gemm_nvfp4(
        _p(a.codes), _p(a.sf), _p(a.scale), _p(b.codes), _p(b.sf), _p(b.scale), M, N, a.k_aug, _p(out),
        out.stride(0), _p(add), 0 if add is None else add.stride(0), _stream(stream)))
    return out


def gemm_bf16(x: torch.Tensor, w: torch.Tensor, out: torch.Tensor | None = None, add: torch.Tensor | None = None,
              stream=None) -> torch.Tensor:
    """arc_gemm_bf16: Y [M, N] = bf16(X W^T (+ add))."""
    _need_cuda(x, w, out, add)
    M, K = x.shape
    N = w.shape[0]
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=x.device)
    _check("arc_gemm_bf16", lib().arc_gemm_bf16(
        _p(x), x.stride(0), _p(w), w.stride(0), M, N, K, _p(out), out.stride(0), _p(add),
        0 if add is None else add.stride(0), _stream(stream)))
    return out


def rmsnorm_bf16(h: torch.Tensor, gain: torch.Tensor, eps: float = 1e-6, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    S, d = h.shape
    if out is None:
        out = torch.empty_like(h)
    _check("arc_rmsnorm_bf16", lib().arc_rmsnorm_bf16(_p(h), S, d, h.stride(0), _p(gain), float(eps), _p(out),
                                                      out.stride(0), _stream(stream)))
    return out


def silu_mul_bf16(gu: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    S, F2 = gu.shape
    F = F2 // 2
    if out is None:
        out = torch.empty(S, F, dtype=torch.bfloat16, device=gu.device)
    _check("arc_silu_mul_bf16", lib().arc_silu_mul_bf16(_p(gu), S, F, gu.stride(0), _p(out), out.stride(0),
                                                        _stream(stream)))
    return out


class RecurrentBlock:
    """Host description of the shared SwiGLU block (keeps the ctypes structs and tensors alive).
    Each sublayer dict holds gain, wgu, wd (bf16), gu_q, d_q (packed NVFP4 weights), idx_gu,
    idx_d, and optionally gu_f8, d_f8 (FP8Tensor weights, needed by FP8 steps).
    residual_scale is the damped residual's beta and inject an optional bf16 [S, d] term e added to
    it (h <- beta h + e + F(h); 1 and None: the plain residual block)."""

    def __init__(self, d: int, ffn: int, eps: float, sublayers: list[dict], residual_scale: float = 1.0,
                 inject: torch.Tensor | None = None):
        self.d, self.ffn, self.eps = d, ffn, eps
        self.sub = sublayers
        arr = (SwigluSublayer * len(sublayers))()
        for i, L in enumerate(sublayers):
            f8g, f8d = L.get("gu_f8"), L.get("d_f8")
            arr[i] = SwigluSublayer(
                L["gain"].data_ptr(), L["wgu"].data_ptr(), L["wd"].data_ptr(),
                L["gu_q"].codes.data_ptr(), L["gu_q"].sf.data_ptr(), L["gu_q"].scale.data_ptr(),
                L["d_q"].codes.data_ptr(), L["d_q"].sf.data_ptr(), L["d_q"].scale.data_ptr(),
                L["idx_gu"].data_ptr(), int(L["idx_gu"].numel()), L["idx_d"].data_ptr(), int(L["idx_d"].numel()),
                f8g.codes.data_ptr() if f8g is not None else None, f8g.scale.data_ptr() if f8g is not None else None,
                f8d.codes.data_ptr() if f8d is not None else None, f8d.scale.data_ptr() if f8d is not None else None)
        self._arr = arr
        self._inject = inject
        self.block = SwigluBlock(d, ffn, float(eps), len(sublayers), arr, float(residual_scale),
                                 inject.data_ptr() if inject is not None else None)

    def workspace_bytes(self, S: int) -> int:
        return int(lib().arc_recurrent_workspace_bytes(S, ctypes.byref(self.block)))


def recurrent_prefill(h: torch.Tensor, block: RecurrentBlock, T: int, k_low: int,
                      workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """arc_recurrent_prefill: apply the block T times in place (steps < k_low in NVFP4 + ARC)."""
    S = h.shape[0]
    n = block.workspace_bytes(S)
    if workspace is None:
        workspace = _ws(n, h.device)
    _check("arc_recurrent_prefill", lib().arc_recurrent_prefill(_p(h), S, ctypes.byref(block.block), T, k_low,
                                                                _p(workspace), workspace.numel(), _stream(stream)))
    return h


def recurrent_prefill_schedule(h: torch.Tensor, block: RecurrentBlock, schedule, workspace: torch.Tensor | None = None,
                               stream=None) -> torch.Tensor:
    """arc_recurrent_prefill_schedule: apply the block len(schedule) times in place; step t in
    the format schedule[t]: STEP_BF16 (0 / False), STEP_NVFP4 (1 / True) or STEP_FP8 (2)."""
    S = h.shape[0]
    flags = (ctypes.c_uint8 * max(1, len(schedule)))(*[int(f) for f in schedule])
    n = block.workspace_bytes(S)
    if workspace is None:
        workspace = _ws(n, h.device)
    _check("arc_recurrent_prefill_schedule", lib().arc_recurrent_prefill_schedule(
        _p(h), S, ctypes.byref(block.block), len(schedule), flags, _p(workspace), workspace.numel(),
        _stream(stream)))
    return h


@dataclass
class MXFP4Tensor:
    """Packed MXFP4 operand: codes [rows, K_pad/2] u8 and swizzled E8M0 scale bytes (no tensor scale)."""
    codes: torch.Tensor
    sf: torch.Tensor
    rows: int
    k_aug: int


def mxfp4_sf_bytes(rows: int, k_aug: int) -> int:
    return int(lib().arc_mxfp4_sf_bytes(rows, k_aug))


def _mx_out(rows, k_aug, device):
    return MXFP4Tensor(_u8(codes_bytes(rows, k_aug), device), _u8(mxfp4_sf_bytes(rows, k_aug), device), rows, k_aug)


def quantize_act_mxfp4(x: torch.Tensor, idx: torch.Tensor | None = None, out: MXFP4Tensor | None = None,
                       stream=None) -> MXFP4Tensor:
    """arc_quantize_act_mxfp4: X [M, K] bf16 -> MXFP4 with r appended residual channels."""
    _need_cuda(x, idx)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    r = 0 if idx is None else int(idx.numel())
    if out is None:
        out = _mx_out(M, K + r, x.device)
    _check("arc_quantize_act_mxfp4", lib().arc_quantize_act_mxfp4(_p(x), M, K, x.stride(0), _p(idx), r, _p(out.codes),
                                                                  _p(out.sf), _stream(stream)))
    return out


def pack_weight_mxfp4(w: torch.Tensor, idx: torch.Tensor | None = None, out: MXFP4Tensor | None = None,
                      stream=None) -> MXFP4Tensor:
    """arc_pack_weight_mxfp4: W [N, K] bf16 -> W_aug = [W | W[:, idx]] in MXFP4."""
    _need_cuda(w, idx)
    assert w.dtype == torch.bfloat16 and w.dim() == 2 and w.stride(1) == 1
    N, K = w.shape
    r = 0 if idx is None else int(idx.numel())
    if out is None:
        out = _mx_out(N, K + r, w.device)
    _check("arc_pack_weight_mxfp4", lib().arc_pack_weight_mxfp4(_p(w), N, K, w.stride(0), _p(idx), r, _p(out.codes),
                                                                _p(out.sf), _stream(stream)))
    return out


def gemm_mxfp4(a: MXFP4Tensor, b: MXFP4Tensor, out: torch.Tensor | None = None, add: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """arc_gemm_mxfp4: Y [M, N] bf16 = MXFP4(A) MXFP4(B)^T over depth K_aug (+ add)."""
    assert a.k_aug == b.k_aug
    M, N = a.rows, b.rows
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _check("arc_gemm_mxfp4", lib().arc_gemm_mxfp4(
        _p(a.codes), _p(a.sf), _p(b.codes), _p(b.sf), M, N, a.k_aug, _p(out), out.stride(0), _p(add),
        0 if add is None else add.stride(0), _stream(stream)))
    return out


class FP8Tensor:
    """E4M3 codes [rows, K] (row stride K bytes) and the device fp32 tensor scale."""

    def __init__(self, codes: torch.Tensor, scale: torch.Tensor):
        self.codes, self.scale = codes, scale
        self.rows, self.k = codes.shape


def quantize_fp8(x: torch.Tensor, static_scale: torch.Tensor | None = None, out: FP8Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> FP8Tensor:
    """arc_quantize_fp8: X [M, K] bf16 -> E4M3 codes with one per-tensor scale (amax/448)."""
    _need_cuda(x, static_scale)
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    M, K = x.shape
    if out is None:
        out = FP8Tensor(torch.empty(M, K, dtype=torch.uint8, device=x.device),
                        torch.empty(1, dtype=torch.float32, device=x.device))
    if workspace is None:
        workspace = _ws(quantize_workspace_bytes(M, 0), x.device)
    _check("arc_quantize_fp8", lib().arc_quantize_fp8(_p(x), M, K, x.stride(0), _p(static_scale), _p(out.codes),
                                                      out.codes.stride(0), _p(out.scale), _p(workspace),
                                                      workspace.numel(), _stream(stream)))
    return out


def gemm_fp8(a: FP8Tensor, b: FP8Tensor, out: torch.Tensor | None = None, add: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    """arc_gemm_fp8: Y [M, N] bf16 = s_A s_B * E4M3(A) E4M3(B)^T (+ add)."""
    assert a.k == b.k
    M, N, K = a.rows, b.rows, a.k
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.codes.device)
    _check("arc_gemm_fp8", lib().arc_gemm_fp8(
        _p(a.codes), a.codes.stride(0), _p(a.scale), _p(b.codes), b.codes.stride(0), _p(b.scale), M, N, K,
        _p(out), out.stride(0), _p(add), 0 if add is None else add.stride(0), _stream(stream)))
    return out


def last_device_status(stream=None) -> int:
    return int(lib().arc_last_device_status(_stream(stream)))


def set_wait_limit_ns(ns: int):
    _check("arc_set_wait_limit_ns", lib().arc_set_wait_limit_ns(int(ns)))


def debug_inject(kind: int):
    _check("arc_debug_inject", lib().arc_debug_inject(int(kind)))
