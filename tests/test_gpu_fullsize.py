"""GPU parity at the workloads' full sizes, in the launch configuration the benchmark times.

Per linear layer: outlier calibration (indices bit-exact), the dynamic-scale activation
quantizer and the weight packer (every code and scale byte bit-exact, tensor scales equal),
then the block-scaled GEMM of depth K + r checked on sampled output rows against the oracle's
FP64 GEMM over all N outputs. The sampled rows are seeded random rows plus, for every outlier
channel, the row holding its largest |x|, and the first and last rows (ragged-tile edges).
Rule: max |Y_gpu - Y_ref| / (||x_m|| ||w_n||) <= 2e-3.
"""
import numpy as np
import pytest
import torch

import nvfp4_block_scaled_arc_b200 as arc
import oracle as O
import workloads as W
from tests._helpers import (GEMM_TOL, assert_codes_equal, gpu_codes, gpu_sf_canonical, normalized_gemm_error,
                            row_norms, to_bits, to_dev)

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_rows(x_bits: np.ndarray, outliers, n_random: int, seed: int) -> np.ndarray:
    M = x_bits.shape[0]
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(M, size=min(n_random, M), replace=False).tolist())
    rows.update([0, M - 1])
    for c in np.asarray(outliers)[:64]:
        col = (x_bits[:, c] & 0x7FFF).astype(np.int32)  # |bf16| orders like its bit pattern
        rows.add(int(np.argmax(col)))
    return np.array(sorted(rows), np.int64)


def check_layer(x_bits, w_bits, r, outliers, n_random=24, seed=0):
    M, K = x_bits.shape
    N = w_bits.shape[0]
    x, w = to_dev(x_bits), to_dev(w_bits)
    # calibration
    idx = O.calibrate(x_bits, r) if r else np.zeros(0, np.int32)
    d_idx = None
    if r:
        d_idx = arc.calibrate_outliers(x, r)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(d_idx.cpu().numpy(), idx)
    # quantizer and weight packer, whole tensors
    A = arc.quantize_act_nvfp4(x, d_idx)
    B = arc.pack_weight_nvfp4(w, d_idx)
    y = arc.gemm_nvfp4(A, B)
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    sa = O.tensor_scale(O.amax(x_bits))
    sw = O.tensor_scale(O.amax(w_bits))
    assert A.scale.item() == np.float32(sa)
    assert B.scale.item() == np.float32(sw)
    ac, asf = O.quantize_act(x_bits, idx, sa)
    assert_codes_equal(gpu_codes(A, M), ac, "activation codes")
    assert_codes_equal(gpu_sf_canonical(A, M), asf, "activation scale bytes")
    del x
    bc, bsf = O.pack_weight(w_bits, idx, sw)
    assert_codes_equal(gpu_codes(B, N), bc, "weight codes")
    assert_codes_equal(gpu_sf_canonical(B, N), bsf, "weight scale bytes")
    del w
    # GEMM on sampled rows, every output column
    rows = sample_rows(x_bits, outliers, n_random, seed)
    ref = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw, rows=rows)
    yb = to_bits(y[torch.from_numpy(rows).cuda()])
    err = normalized_gemm_error(yb, ref, row_norms(x_bits[rows]), row_norms(w_bits))
    assert err <= GEMM_TOL, err
    return err


@pytest.mark.parametrize("proj", ["qkv", "o", "gateup", "down"])
def test_llama8b_projection_full_size(proj):
    d = W.llama8b(proj)
    check_layer(d["x"], d["w"], d["r"], d["outliers"], seed=1)


@pytest.mark.parametrize("frac", [0.0, 0.001, 0.01, 0.05])
def test_outlier_stress_full_size(frac):
    d = W.stress(frac)
    for r in (0, 32, 128, 256):
        check_layer(d["x"], d["w"], r, d["outliers"], n_random=8, seed=2)


@pytest.mark.parametrize("proj", ["gateup", "down"])
def test_mlp70b_projection_full_size(proj):
    d = W.mlp70b(proj)
    check_layer(d["x"], d["w"], d["r"], d["outliers"], n_random=12, seed=4)


def test_bf16_gemm_full_size():
    # the BF16 switch at a recurrent-block shape (gate|up of d = 2048, ffn = 8192, 4096 tokens)
    x = W.matrix_bf16(3, 1, 4096, 2048, 1.0)
    w = W.matrix_bf16(3, 2, 16384, 2048, 0.005)
    y = arc.gemm_bf16(to_dev(x), to_dev(w))
    torch.cuda.synchronize()
    assert arc.last_device_status() == 0
    rows = np.r_[0:4, 1000:1004, 4092:4096]
    ref = O.gemm_bf16_f64(x, w, rows=rows)
    err = normalized_gemm_error(to_bits(y)[rows], ref, row_norms(x[rows]), row_norms(w))
    assert err <= GEMM_TOL, err


def test_gemm_is_reproducible():
    # the MMA issue order is fixed, so repeated calls give identical bits
    d = W.llama8b("qkv")
    x, w = to_dev(d["x"]), to_dev(d["w"])
    idx = arc.calibrate_outliers(x, d["r"])
    A = arc.quantize_act_nvfp4(x, idx)
    B = arc.pack_weight_nvfp4(w, idx)
    y0 = arc.gemm_nvfp4(A, B)
    y1 = arc.gemm_nvfp4(A, B)
    b0 = arc.gemm_bf16(x, w)
    b1 = arc.gemm_bf16(x, w)
    torch.cuda.synchronize()
    assert torch.equal(y0, y1)
    assert torch.equal(b0, b1)
