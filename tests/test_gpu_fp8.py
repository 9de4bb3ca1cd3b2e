"""GPU parity of the FP8 W8A8 path (per-tensor E4M3 quantizer, kind::f8f6f4 GEMM) against the
CPU oracle: codes and tensor scales bit for bit, GEMM outputs within 2e-3 of the oracle's FP64
GEMM normalised by ||x_m|| ||w_n||.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import GEMM_TOL, normalized_gemm_error, row_norms, to_bits, to_dev

pytestmark = pytest.mark.gpu


def quant_and_compare(x_bits, static=None):
    st = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
    q = arc.quantize_fp8(to_dev(x_bits), static_scale=st)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    s = float(np.float32(static)) if static is not None else O.fp8_scale(O.amax(x_bits))
    assert q.scale.item() == np.float32(s)
    want = O.quantize_fp8(x_bits, s)
    got = q.codes.cpu().numpy()
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        m, k = bad[0]
        raise AssertionError(f"{len(bad)} codes differ, first at ({m}, {k}): {got[m, k]:#04x} vs {want[m, k]:#04x}")
    return q, want, s


@pytest.mark.parametrize("M,K", [(16, 256), (37, 96), (300, 4096), (5, 16)])
def test_quantizer_matches_oracle(M, K):
    x = W.matrix_bf16(31, 1, M, K, 1.0, col_mult=W.outlier_multipliers(31, 0, K, max(1, K // 50), 10.0, 80.0))
    quant_and_compare(x)


def test_quantizer_static_scales_and_special_values():
    x = W.matrix_bf16(32, 1, 24, 128, 2.0)
    for s in (1.0, 0.01, 1e-30, 3e29):  # the last two take the plain-divide path
        quant_and_compare(x, static=s)
    z = np.zeros((8, 64), np.uint16)
    z[:, 1::2] = 0x8000  # -0.0
    q, want, _ = quant_and_compare(z)
    assert (want[:, 1::2] == 0x80).all() and (want[:, ::2] == 0).all()


@pytest.mark.parametrize("which", ["tiny", "qkv", "down_ragged"])
def test_gemm_matches_oracle(which):
    if which == "tiny":
        d = W.tiny()
        x_bits, w_bits = d["x"], d["w"]
    elif which == "qkv":
        d = W.llama8b("qkv", rows=300, w_rows=520)
        x_bits, w_bits = d["x"], d["w"]
    else:
        d = W.llama8b("down", rows=130, w_rows=264)
        x_bits, w_bits = d["x"], d["w"]
    A, ac, sa = quant_and_compare(x_bits)
    B, bc, sw = quant_and_compare(w_bits)
    y = arc.gemm_fp8(A, B)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    ref = O.gemm_fp8_f64(ac, sa, bc, sw)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(x_bits), row_norms(w_bits))
    assert err <= GEMM_TOL, err


def test_gemm_residual_add():
    d = W.llama8b("o", rows=200, w_rows=256)
    A, ac, sa = quant_and_compare(d["x"])
    B, bc, sw = quant_and_compare(d["w"])
    h = W.matrix_bf16(33, 3, 200, 256, 1.0)
    y = arc.gemm_fp8(A, B, add=to_dev(h))
    torch.cuda.synchronize()
    ref = O.gemm_fp8_f64(ac, sa, bc, sw) + O.bf16_bits_to_f32(h).astype(np.float64)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(d["x"]), row_norms(d["w"]), with_add=True)
    assert err <= GEMM_TOL, err


def test_gemm_k_not_multiple_of_32():
    x = W.matrix_bf16(34, 1, 64, 272, 1.0)
    w = W.matrix_bf16(34, 2, 256, 272, 0.05)
    A, ac, sa = quant_and_compare(x)
    B, bc, sw = quant_and_compare(w)
    y = arc.gemm_fp8(A, B)
    torch.cuda.synchronize()
    ref = O.gemm_fp8_f64(ac, sa, bc, sw)
    assert normalized_gemm_error(to_bits(y), ref, row_norms(x), row_norms(w)) <= GEMM_TOL
