"""Out-of-bounds write checks without a sanitizer: every output buffer of the library's kernels is
placed between two canary margins (and, for row-pitched outputs, given padding columns between
rows); after each call on ragged shapes the canary bytes must be untouched. The outputs themselves
are checked against the oracle elsewhere; here only where the kernels write is checked.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import workloads as W
from tests._helpers import to_dev

pytestmark = pytest.mark.gpu

MARGIN = 4096  # bytes on each side (keeps the guarded view 16-byte aligned)
CANARY = 0xA5


class Guarded:
    """A byte buffer of n bytes between two canary margins."""

    def __init__(self, n: int):
        self.n = n
        self.full = torch.full((n + 2 * MARGIN,), CANARY, dtype=torch.uint8, device="cuda")
        self.view = self.full[MARGIN:MARGIN + n]

    def check(self, what: str):
        torch.cuda.synchronize()
        head = self.full[:MARGIN].cpu().numpy()
        tail = self.full[MARGIN + self.n:].cpu().numpy()
        assert np.all(head == CANARY), f"{what}: write before the buffer"
        assert np.all(tail == CANARY), f"{what}: write past the buffer"


class GuardedRows:
    """A bf16 [rows, cols] output with row pitch ld >= cols, between canary margins; the padding
    columns [cols, ld) of every row are canary too."""

    def __init__(self, rows: int, cols: int, ld: int):
        self.rows, self.cols, self.ld = rows, cols, ld
        self.g = Guarded(rows * ld * 2)
        self.t = self.g.view.view(torch.bfloat16).view(rows, ld)[:, :cols]

    def check(self, what: str):
        self.g.check(what)
        if self.ld > self.cols:
            pad = self.g.view.view(torch.bfloat16).view(self.rows, self.ld)[:, self.cols:]
            assert np.all(pad.contiguous().view(torch.uint8).cpu().numpy() == CANARY), f"{what}: write in row padding"


def _nvfp4_out(rows, k_aug):
    c, s = Guarded(arc.codes_bytes(rows, k_aug)), Guarded(arc.sf_bytes(rows, k_aug))
    sc = Guarded(4)
    return arc.NVFP4Tensor(c.view, s.view, sc.view.view(torch.float32), rows, k_aug), (c, s, sc)


def _mx_out(rows, k_aug):
    c, s = Guarded(arc.codes_bytes(rows, k_aug)), Guarded(arc.mxfp4_sf_bytes(rows, k_aug))
    return arc.MXFP4Tensor(c.view, s.view, rows, k_aug), (c, s)


def _check_all(gs, what):
    for i, g in enumerate(gs):
        g.check(f"{what} [{i}]")


def _x(M, K, seed=51):
    return to_dev(W.matrix_bf16(seed, 1, M, K, 1.0, col_mult=W.outlier_multipliers(seed, 0, K, max(1, K // 40), 10.0, 60.0)))


@pytest.mark.parametrize("M,K,r", [(1, 64, 0), (7, 208, 48), (131, 4160, 64), (300, 272, 16), (129, 1024, 256)])
def test_nvfp4_quantizers_write_only_their_outputs(M, K, r):
    x = _x(M, K)
    idx = arc.calibrate_outliers(x, r) if r else None
    out, gs = _nvfp4_out(M, K + r)
    arc.quantize_act_nvfp4(x, idx, out=out)
    _check_all(gs, "quantize_act_nvfp4")
    out, gs = _nvfp4_out(M, K + r)
    arc.quantize_act_nvfp4(x, idx, rms_gain=to_dev(W.matrix_bf16(52, 1, 1, K, 1.0)).view(-1), out=out)
    _check_all(gs, "quantize_act_nvfp4 + RMSNorm")
    out, gs = _nvfp4_out(M, K + r)
    arc.pack_weight_nvfp4(x, idx, out=out)
    _check_all(gs, "pack_weight_nvfp4")
    if K % 2 == 0 and r > 0:
        perm = arc.calibrate_order(x)
        out, gs = _nvfp4_out(M, K + r)
        arc.quantize_act_nvfp4_reordered(x, perm, r, out=out)
        _check_all(gs, "quantize_act_nvfp4_reordered")


@pytest.mark.parametrize("M,K,r", [(1, 64, 0), (7, 224, 32), (131, 4160, 64), (300, 96, 32)])
def test_mxfp4_and_fp8_quantizers_write_only_their_outputs(M, K, r):
    x = _x(M, K)
    idx = arc.calibrate_outliers(x, r) if r else None
    out, gs = _mx_out(M, K + r)
    arc.quantize_act_mxfp4(x, idx, out=out)
    _check_all(gs, "quantize_act_mxfp4")
    c, sc = Guarded(M * K), Guarded(4)
    arc.quantize_fp8(x, out=arc.FP8Tensor(c.view.view(M, K), sc.view.view(torch.float32)))
    _check_all([c, sc], "quantize_fp8")


@pytest.mark.parametrize("M,N,K,r,ld_pad", [(1, 8, 64, 0, 8), (129, 264, 512, 64, 24), (300, 136, 208, 48, 0),
                                            (257, 520, 1024, 0, 8)])
def test_gemms_write_only_their_outputs(M, N, K, r, ld_pad):
    x, w = _x(M, K, 53), to_dev(W.matrix_bf16(53, 2, N, K, 0.02))
    idx = arc.calibrate_outliers(x, r) if r else None
    A, B = arc.quantize_act_nvfp4(x, idx), arc.pack_weight_nvfp4(w, idx)
    add = to_dev(W.matrix_bf16(53, 3, M, N, 0.5))
    for with_add in (False, True):
        y = GuardedRows(M, N, N + ld_pad)
        arc.gemm_nvfp4(A, B, out=y.t, add=add if with_add else None)
        y.check(f"gemm_nvfp4 add={with_add}")
        y = GuardedRows(M, N, N + ld_pad)
        arc.gemm_bf16(x, w, out=y.t, add=add if with_add else None)
        y.check(f"gemm_bf16 add={with_add}")
        y = GuardedRows(M, N, N + ld_pad)
        arc.gemm_fp8(arc.quantize_fp8(x), arc.quantize_fp8(w), out=y.t, add=add if with_add else None)
        y.check(f"gemm_fp8 add={with_add}")
    if K % 32 == 0 and r % 32 == 0:
        Am, Bm = arc.quantize_act_mxfp4(x, idx), arc.pack_weight_mxfp4(w, idx)
        y = GuardedRows(M, N, N + ld_pad)
        arc.gemm_mxfp4(Am, Bm, out=y.t)
        y.check("gemm_mxfp4")
    assert arc.last_device_status() == 0


def test_elementwise_kernels_write_only_their_outputs():
    S, d, F = 131, 264, 520
    h = to_dev(W.matrix_bf16(54, 1, S, d, 1.0))
    g = to_dev(W.matrix_bf16(54, 2, 1, d, 1.0)).view(-1)
    y = GuardedRows(S, d, d + 8)
    arc.rmsnorm_bf16(h, g, 1e-6, out=y.t)
    y.check("rmsnorm_bf16")
    gu = to_dev(W.matrix_bf16(54, 3, S, 2 * F, 1.0))
    y = GuardedRows(S, F, F + 16)
    arc.silu_mul_bf16(gu, out=y.t)
    y.check("silu_mul_bf16")
