"""GPU parity of the channel reorder (calibration order, reordered activation quantizer, reordered
weight packer, and the block-scaled GEMM on reordered operands) against the CPU oracle.

Orders and codes/scale bytes (canonical form) must match bit for bit; GEMM outputs within the
usual 2e-3 of the oracle's FP64 GEMM, normalised by ||x_m|| ||w_n||.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import (GEMM_TOL, assert_codes_equal, gpu_codes, gpu_sf_canonical, gpu_sf_swizzled,
                            normalized_gemm_error, row_norms, to_bits, to_dev)

pytestmark = pytest.mark.gpu


def gpu_order(x_bits):
    perm = arc.calibrate_order(to_dev(x_bits))
    torch.cuda.synchronize()
    got = perm.cpu().numpy()
    np.testing.assert_array_equal(got, O.calibrate_order(x_bits))
    return perm, got


def run_reordered(x_bits, r, perm=None, static=None, gain_bits=None, eps=1e-6, weights=False):
    M, K = x_bits.shape
    if perm is None:
        d_perm, perm = gpu_order(x_bits)
    else:
        perm = np.asarray(perm, np.int32)
        d_perm = torch.from_numpy(perm).cuda()
    x = to_dev(x_bits)
    if weights:
        q = arc.pack_weight_nvfp4_reordered(x, d_perm, r)
        s_ref = O.tensor_scale(O.amax(x_bits))
        c_ref, sf_ref = O.pack_weight_reordered(x_bits, perm, r, s_ref)
    else:
        st = None if static is None else torch.tensor([static], dtype=torch.float32, device="cuda")
        g = None if gain_bits is None else to_dev(gain_bits)
        q = arc.quantize_act_nvfp4_reordered(x, d_perm, r, rms_gain=g, eps=eps, static_scale=st)
        eps32 = float(np.float32(eps))
        if static is not None:
            s_ref = float(np.float32(static))
        elif gain_bits is not None:
            s_ref = O.tensor_scale(O.amax(O.rmsnorm(x_bits, gain_bits, eps32)))
        else:
            s_ref = O.tensor_scale(O.amax(x_bits))
        c_ref, sf_ref = O.quantize_act_reordered(x_bits, perm, r, s_ref, rms_gain=gain_bits, eps=eps32)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    assert q.scale.item() == np.float32(s_ref), (q.scale.item(), s_ref)
    assert_codes_equal(gpu_codes(q, M), c_ref, "codes")
    assert_codes_equal(gpu_sf_canonical(q, M), sf_ref, "scale bytes")
    np.testing.assert_array_equal(gpu_sf_swizzled(q, M), O.sf_swizzle(sf_ref))
    return q, perm, (c_ref, sf_ref, s_ref)


def test_order_tiny_and_ties():
    d = W.tiny()
    gpu_order(d["x"])
    x = W.matrix_bf16(5, 1, 40, 96, 1.0)
    x[:, 10] = x[:, 3]
    x[:, 50] = x[:, 3]  # three equal columns: ordered by index
    gpu_order(x)


@pytest.mark.parametrize("proj,rows", [("qkv", 64), ("down", 32)])
def test_order_llama_shapes(proj, rows):
    d = W.llama8b(proj, rows=rows, with_w=False)
    gpu_order(d["x"])


def test_order_wide_k():
    # several ranking tiles: K = 28672 (the 70B down projection's input)
    d = W.mlp70b("down", rows=16, with_w=False)
    gpu_order(d["x"])


def test_tiny_config():
    d = W.tiny()
    run_reordered(d["x"], 16)


@pytest.mark.parametrize("proj,rows", [("qkv", 300), ("down", 130), ("gateup", 129)])
def test_llama_shapes_ragged_rows(proj, rows):
    d = W.llama8b(proj, rows=rows, with_w=False)
    run_reordered(d["x"], 128)


@pytest.mark.parametrize("K,r,M", [(272, 16, 40), (208, 48, 7), (64, 0, 1), (4160, 64, 131), (16, 16, 3)])
def test_k_not_multiple_of_64_and_tiny_rows(K, r, M):
    x = W.matrix_bf16(9, 1, M, K, 1.0, col_mult=W.outlier_multipliers(9, 0, K, max(1, K // 50), 10.0, 60.0))
    run_reordered(x, r)


def test_arbitrary_permutation():
    # any permutation, not only a calibration order: gathers from every position of the row
    x = W.matrix_bf16(11, 1, 77, 1024, 1.0, col_mult=W.outlier_multipliers(11, 0, 1024, 12, 5.0, 50.0))
    perm = np.random.default_rng(11).permutation(1024).astype(np.int32)
    run_reordered(x, 64, perm=perm)
    run_reordered(x, 0, perm=np.arange(1024, dtype=np.int32))


@pytest.mark.parametrize("static", [0.01, 1e-6])
def test_static_scale(static):
    d = W.llama8b("o", rows=64, with_w=False)
    run_reordered(d["x"], 32, static=static)


def test_rmsnorm_prologue():
    d = W.recurrent(S=200, d=2048, ffn=256)
    run_reordered(d["h"], 64, gain_bits=d["layers"][0]["gain"])
    h = W.matrix_bf16(21, 1, 96, 512, 3.0)
    g = W.matrix_bf16(21, 2, 1, 512, 1.0).reshape(-1)
    run_reordered(h, 32, gain_bits=g)
    run_reordered(h, 32, gain_bits=g, static=0.002)


@pytest.mark.parametrize("which", ["tiny", "qkv"])
def test_weight_pack(which):
    if which == "tiny":
        d = W.tiny()
        perm = O.calibrate_order(d["x"])
        run_reordered(d["w"], 16, perm=perm, weights=True)
    else:
        d = W.llama8b("qkv", rows=64, w_rows=512)
        perm = O.calibrate_order(d["x"])
        run_reordered(d["w"], 128, perm=perm, weights=True)


@pytest.mark.parametrize("which", ["tiny", "qkv"])
def test_gemm_on_reordered_operands(which):
    if which == "tiny":
        d = W.tiny()
        x_bits, w_bits, r = d["x"], d["w"], d["r"]
    else:
        d = W.llama8b("qkv", rows=300, w_rows=512)
        x_bits, w_bits, r = d["x"], d["w"], 128
    A, perm, (ac, asf, sa) = run_reordered(x_bits, r)
    B, _, (bc, bsf, sw) = run_reordered(w_bits, r, perm=perm, weights=True)
    y = arc.gemm_nvfp4(A, B)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    ref = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw)
    err = normalized_gemm_error(to_bits(y), ref, row_norms(x_bits), row_norms(w_bits))
    assert err <= GEMM_TOL, err


def test_rejects_too_wide_rows():
    x = torch.zeros(4, 51216, dtype=torch.bfloat16, device="cuda")
    perm = torch.arange(51216, dtype=torch.int32, device="cuda")
    with pytest.raises(arc.ArcError):
        arc.quantize_act_nvfp4_reordered(x, perm, 16)


@pytest.mark.slow
@pytest.mark.parametrize("proj", ["qkv", "down"])
def test_llama8b_full_size_reordered(proj):
    d = W.llama8b(proj)
    x_bits, w_bits = d["x"], d["w"]
    A, perm, (ac, asf, sa) = run_reordered(x_bits, 128)
    B, _, (bc, bsf, sw) = run_reordered(w_bits, 128, perm=perm, weights=True)
    y = arc.gemm_nvfp4(A, B)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    rows = np.r_[0, 1, 777, 2048, 4095]
    ref = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw, rows=rows)
    yb = to_bits(y[torch.from_numpy(rows).cuda()])
    err = normalized_gemm_error(yb, ref, row_norms(x_bits[rows]), row_norms(w_bits))
    assert err <= GEMM_TOL, err
