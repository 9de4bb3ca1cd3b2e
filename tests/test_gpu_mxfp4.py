"""GPU parity of the MXFP4 path with augmented residual channels (ARCQuant's MXFP4 extension):
the quantizer's codes and E8M0 scale bytes bit for bit against the oracle (whole tensors, scale
bytes compared in canonical form and the swizzled buffer compared whole, padding included), and
the kind::mxf4nvf4 scale_vec::2X GEMM within 2e-3 of the oracle's FP64 GEMM normalised by
||x_m|| ||w_n||, first on oracle-built operands, then end to end.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import GEMM_TOL, assert_codes_equal, normalized_gemm_error, row_norms, to_bits, to_dev

pytestmark = pytest.mark.gpu


def _idx(x_bits, r):
    return O.calibrate(x_bits, r) if r else np.zeros(0, np.int32)


def _dev_idx(idx):
    return torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda() if len(idx) else None


def _check_quant(x_bits, r, dup=False):
    M, K = x_bits.shape
    idx = _idx(x_bits, r)
    x = to_dev(x_bits)
    q = (arc.pack_weight_mxfp4 if dup else arc.quantize_act_mxfp4)(x, _dev_idx(idx))
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    c_ref, s_ref = (O.pack_weight_mxfp4 if dup else O.quantize_act_mxfp4)(x_bits, idx)
    kp = O.kpad(K + r)
    got_c = q.codes[: M * kp // 2].cpu().numpy().reshape(M, kp // 2)
    assert_codes_equal(got_c, c_ref)
    swz = q.sf[: O.sf_swizzled_bytes(M, kp // 32)].cpu().numpy()
    assert_codes_equal(O.sf_unswizzle(swz, M, kp // 32), s_ref, "scale bytes")
    np.testing.assert_array_equal(swz, O.sf_swizzle(s_ref))  # padding rows and columns are zero
    return q, idx, c_ref, s_ref


@pytest.mark.parametrize("M,K,r", [(16, 256, 32), (37, 96, 32), (300, 4096, 128), (5, 64, 32), (130, 1024, 0),
                                   (200, 512, 256), (64, 4096, 64), (1, 32, 0)])
def test_quantizer_matches_oracle(M, K, r):
    mult = W.outlier_multipliers(41, 0, K, max(1, K // 64), 10.0, 80.0)
    x = W.matrix_bf16(41, 1, M, K, 1.0, col_mult=mult)
    _check_quant(x, r)


@pytest.mark.parametrize("N,K,r", [(256, 256, 32), (520, 4096, 128), (24, 320, 64)])
def test_weight_pack_matches_oracle(N, K, r):
    w = W.matrix_bf16(42, 2, N, K, 0.02)
    x = W.matrix_bf16(42, 1, 64, K, 1.0, col_mult=W.outlier_multipliers(42, 0, K, max(1, K // 50), 10.0, 80.0))
    idx = _idx(x, r)
    q = arc.pack_weight_mxfp4(to_dev(w), _dev_idx(idx))
    torch.cuda.synchronize()
    c_ref, s_ref = O.pack_weight_mxfp4(w, idx)
    kp = O.kpad(K + r)
    assert_codes_equal(q.codes[: N * kp // 2].cpu().numpy().reshape(N, kp // 2), c_ref)
    swz = q.sf[: O.sf_swizzled_bytes(N, kp // 32)].cpu().numpy()
    np.testing.assert_array_equal(swz, O.sf_swizzle(s_ref))


def test_quantizer_special_values():
    # all-zero blocks (negative zeros included), signed zeros inside nonzero blocks, subnormal
    # bf16 maxima, the largest bf16 magnitudes, values that saturate (above 6 X)
    M, K = 8, 256
    v = np.random.default_rng(5).standard_normal((M, K)).astype(np.float32)
    v[0, :32] = 0.0
    v[1, :32] = -0.0
    v[2, 5] = -0.0
    v[3, 32:64] = np.float32(2.0 ** -130)
    v[4, 64:96] = np.float32(3.0e38)
    v[5, 96] = 7.9  # the block maximum reaches 7.9 X: saturates to 6 X
    bits = (v.view(np.uint32) >> 16).astype(np.uint16)
    r = 32
    _check_quant(bits, r)
    _check_quant(bits, r, dup=True)


def _upload(codes, sc_canon, rows, k_aug):
    c = torch.from_numpy(codes.reshape(-1).copy()).cuda()
    s = torch.from_numpy(O.sf_swizzle(sc_canon)).cuda()
    return arc.MXFP4Tensor(c, s, rows, k_aug)


def _check_gemm(x_bits, w_bits, r, rows=None, add_bits=None, gpu_quant=False):
    M, K = x_bits.shape
    N = w_bits.shape[0]
    idx = _idx(x_bits, r)
    ac, asc = O.quantize_act_mxfp4(x_bits, idx)
    bc, bsc = O.pack_weight_mxfp4(w_bits, idx)
    if gpu_quant:
        A = arc.quantize_act_mxfp4(to_dev(x_bits), _dev_idx(idx))
        B = arc.pack_weight_mxfp4(to_dev(w_bits), _dev_idx(idx))
    else:
        A = _upload(ac, asc, M, K + r)
        B = _upload(bc, bsc, N, K + r)
    add = None if add_bits is None else to_dev(add_bits)
    y = arc.gemm_mxfp4(A, B, add=add)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    rows = np.arange(M) if rows is None else np.asarray(rows)
    ref = O.gemm_mxfp4_f64(ac, asc, bc, bsc, rows=rows)
    if add_bits is not None:
        ref = ref + O.bf16_bits_to_f32(add_bits[rows]).astype(np.float64)
    yb = to_bits(y)[rows]
    err = normalized_gemm_error(yb, ref, row_norms(x_bits[rows]), row_norms(w_bits), with_add=add_bits is not None)
    assert err <= GEMM_TOL, err
    yf = O.bf16_bits_to_f32(yb).astype(np.float64)
    rel = np.abs(yf - ref) / np.maximum(np.abs(ref), 1e-3 * np.abs(ref).max())
    assert np.median(rel) < 2 ** -8
    return err


@pytest.mark.parametrize("M,N,K,r", [(16, 256, 256, 32), (300, 520, 512, 64), (129, 256, 4096, 128),
                                     (1, 8, 64, 0), (257, 768, 1024, 0), (200, 384, 224, 32), (64, 136, 96, 32)])
def test_gemm_on_oracle_operands(M, N, K, r):
    mult = W.outlier_multipliers(43, 0, K, max(1, K // 64), 10.0, 80.0)
    x = W.matrix_bf16(43, 1, M, K, 1.0, col_mult=mult)
    w = W.matrix_bf16(43, 2, N, K, 0.02)
    _check_gemm(x, w, r)


def test_gemm_residual_add_epilogue():
    x = W.matrix_bf16(44, 1, 200, 512, 1.0)
    w = W.matrix_bf16(44, 2, 264, 512, 0.05)
    add = W.matrix_bf16(44, 3, 200, 264, 0.5)
    _check_gemm(x, w, 64, add_bits=add)


@pytest.mark.parametrize("proj", ["qkv", "down"])
def test_end_to_end_llama_projection_rows(proj):
    d = W.llama8b(proj, rows=512)
    _check_gemm(d["x"], d["w"], 128, rows=np.r_[0:8, 250:260, 500:512], gpu_quant=True)


@pytest.mark.slow
def test_full_size_llama_quantizer_and_sampled_gemm():
    # the llama8b gate|up input (4096 x 4096) at full size: codes and scale bytes of the whole
    # tensor, GEMM rows sampled against all 28672 outputs
    d = W.llama8b("gateup")
    q, idx, c_ref, s_ref = _check_quant(d["x"], 128)
    B = arc.pack_weight_mxfp4(to_dev(d["w"]), _dev_idx(idx))
    y = arc.gemm_mxfp4(q, B)
    torch.cuda.synchronize()
    bc, bsc = O.pack_weight_mxfp4(d["w"], idx)
    rows = np.r_[0:4, 2047:2051, 4092:4096]
    ref = O.gemm_mxfp4_f64(c_ref, s_ref, bc, bsc, rows=rows)
    err = normalized_gemm_error(to_bits(y)[rows], ref, row_norms(d["x"][rows]), row_norms(d["w"]))
    assert err <= GEMM_TOL, err
