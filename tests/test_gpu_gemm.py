"""GPU parity of the tcgen05 GEMMs (block-scaled NVFP4 of depth K + r, and BF16).

The NVFP4 GEMM is first checked on operands produced by the oracle (codes as they are, scale
bytes put in the tensor-core layout by the oracle's own swizzle), so a quantizer fault cannot
hide or cause a GEMM fault; then end to end from bf16 inputs through the GPU quantizer.
Rule: max |Y_gpu - Y_ref| / (||x_m|| ||w_n||) <= 2e-3 (Y_ref in FP64).
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import GEMM_TOL, normalized_gemm_error, row_norms, to_bits, to_dev

pytestmark = pytest.mark.gpu


def oracle_operands(x_bits, w_bits, r, idx=None):
    if idx is None:
        idx = O.calibrate(x_bits, r) if r else np.zeros(0, np.int32)
    sa = O.tensor_scale(O.amax(x_bits))
    sw = O.tensor_scale(O.amax(w_bits))
    ac, asf = O.quantize_act(x_bits, idx, sa)
    bc, bsf = O.pack_weight(w_bits, idx, sw)
    return idx, sa, sw, ac, asf, bc, bsf


def upload(codes, sf_canon, scale, rows, k_aug):
    c = torch.from_numpy(codes.reshape(-1).copy()).cuda()
    s = torch.from_numpy(O.sf_swizzle(sf_canon)).cuda()
    sc = torch.tensor([scale], dtype=torch.float32, device="cuda")
    return arc.NVFP4Tensor(c, s, sc, rows, k_aug)


def check_gemm(x_bits, w_bits, r, sample_rows=None, add_bits=None):
    M, K = x_bits.shape
    N = w_bits.shape[0]
    idx, sa, sw, ac, asf, bc, bsf = oracle_operands(x_bits, w_bits, r)
    A = upload(ac, asf, sa, M, K + len(idx))
    B = upload(bc, bsf, sw, N, K + len(idx))
    add = None if add_bits is None else to_dev(add_bits)
    y = arc.gemm_nvfp4(A, B, add=add)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    rows = np.arange(M) if sample_rows is None else np.asarray(sample_rows)
    ref = O.gemm_nvfp4_f64_matmul(ac, asf, sa, bc, bsf, sw, rows=rows)
    if add_bits is not None:
        ref = ref + O.bf16_bits_to_f32(add_bits[rows]).astype(np.float64)
    yb = to_bits(y)[rows]
    err = normalized_gemm_error(yb, ref, row_norms(x_bits[rows]), row_norms(w_bits), with_add=add_bits is not None)
    assert err <= GEMM_TOL, err
    # a tighter look for the record: the GPU result is within a few bf16 ulps of the FP64 value
    yf = O.bf16_bits_to_f32(yb).astype(np.float64)
    rel = np.abs(yf - ref) / np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max())
    assert np.median(rel) < 2 ** -8
    return err


def test_tiny_config_all_outputs():
    d = W.tiny()
    check_gemm(d["x"], d["w"], 16)


@pytest.mark.parametrize("M,N,K,r", [(16, 136, 256, 16), (300, 520, 512, 64), (129, 256, 4096, 128),
                                     (1, 8, 64, 0), (257, 768, 1024, 0), (200, 384, 208, 48)])
def test_ragged_shapes(M, N, K, r):
    mult = W.outlier_multipliers(13, 0, K, max(1, K // 64), 10.0, 80.0)
    x = W.matrix_bf16(13, 1, M, K, 1.0, col_mult=mult)
    w = W.matrix_bf16(13, 2, N, K, 0.02)
    check_gemm(x, w, r)


@pytest.mark.parametrize("proj", ["qkv", "o", "down"])
def test_llama_projection_rows(proj):
    d = W.llama8b(proj, rows=384)
    rows = np.r_[0:8, 127:131, 250:260, 376:384]
    check_gemm(d["x"], d["w"], 128, sample_rows=rows)


@pytest.mark.parametrize("frac,r", [(0.0, 0), (0.01, 128), (0.05, 256)])
def test_stress_rows(frac, r):
    d = W.stress(frac, rows=256)
    check_gemm(d["x"], d["w"], r, sample_rows=np.r_[0:16, 120:136, 240:256])


def test_residual_add_epilogue():
    x = W.matrix_bf16(17, 1, 200, 512, 1.0)
    w = W.matrix_bf16(17, 2, 264, 512, 0.05)
    add = W.matrix_bf16(17, 3, 200, 264, 1.0)
    check_gemm(x, w, 32, add_bits=add)


def test_add_may_alias_output():
    x = W.matrix_bf16(18, 1, 130, 256, 1.0)
    w = W.matrix_bf16(18, 2, 256, 256, 0.05)
    h = W.matrix_bf16(18, 3, 130, 256, 1.0)
    idx = O.calibrate(x, 16)
    xd, wd, hd = to_dev(x), to_dev(w), to_dev(h)
    di = torch.from_numpy(idx).cuda()
    A = arc.quantize_act_nvfp4(xd, di)
    B = arc.pack_weight_nvfp4(wd, di)
    y_sep = arc.gemm_nvfp4(A, B, add=hd)
    arc.gemm_nvfp4(A, B, out=hd, add=hd)
    torch.cuda.synchronize()
    assert torch.equal(y_sep, hd)


def test_end_to_end_through_gpu_quantizer():
    d = W.llama8b("qkv", rows=256, w_rows=512)
    idx = O.calibrate(d["x"], 128)
    di = torch.from_numpy(idx).cuda()
    A = arc.quantize_act_nvfp4(to_dev(d["x"]), di)
    B = arc.pack_weight_nvfp4(to_dev(d["w"]), di)
    y = arc.gemm_nvfp4(A, B)
    torch.cuda.synchronize()
    _, sa, sw, ac, asf, bc, bsf = oracle_operands(d["x"], d["w"], 128, idx=idx)
    ref = O.gemm_nvfp4_f64_matmul(ac, asf, sa, bc, bsf, sw)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(d["x"]), row_norms(d["w"]))
    assert err <= GEMM_TOL


def test_arc_reduces_error_vs_plain_nvfp4():
    # the augmented residual channels bring the quantized product closer to the bf16 product
    d = W.llama8b("qkv", rows=128, w_rows=256)
    x, w = d["x"], d["w"]
    exact = O.gemm_bf16_f64(x, w)
    errs = {}
    for r in (0, 128):
        idx = O.calibrate(x, r) if r else None
        di = None if idx is None else torch.from_numpy(idx).cuda()
        A = arc.quantize_act_nvfp4(to_dev(x), di)
        B = arc.pack_weight_nvfp4(to_dev(w), di)
        y = O.bf16_bits_to_f32(to_bits(arc.gemm_nvfp4(A, B))).astype(np.float64)
        errs[r] = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert errs[128] < errs[0]


# ------------------------------------------------------------------------------------------
# BF16 switch
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("M,N,K", [(16, 256, 256), (300, 520, 200), (129, 2048, 1024), (1, 8, 8)])
def test_bf16_gemm(M, N, K):
    x = W.matrix_bf16(23, 1, M, K, 1.0)
    w = W.matrix_bf16(23, 2, N, K, 0.05)
    y = arc.gemm_bf16(to_dev(x), to_dev(w))
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    ref = O.gemm_bf16_f64(x, w)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(x), row_norms(w))
    assert err <= GEMM_TOL, err


def test_bf16_gemm_add():
    x = W.matrix_bf16(24, 1, 130, 512, 1.0)
    w = W.matrix_bf16(24, 2, 512, 512, 0.05)
    h = W.matrix_bf16(24, 3, 130, 512, 1.0)
    y = arc.gemm_bf16(to_dev(x), to_dev(w), add=to_dev(h))
    torch.cuda.synchronize()
    ref = O.gemm_bf16_f64(x, w) + O.bf16_bits_to_f32(h).astype(np.float64)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(x), row_norms(w), with_add=True)
    assert err <= GEMM_TOL, err
