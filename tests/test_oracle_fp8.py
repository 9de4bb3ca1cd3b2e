"""Pins of the oracle's FP8 W8A8 path (RAMP's low-precision format: FP8 weights and activations,
read here with one per-tensor scale s = amax / 448 each).

The signed E4M3 encoder is checked against PyTorch's CPU float8_e4m3fn cast (round to nearest
even) wherever that cast is defined, saturation and signed zeros by hand; the quantizer by a
round trip of exactly representable tensors; the GEMM against a textbook FP64 matmul of the
original values on such tensors.
"""
import numpy as np
import torch

import oracle as O
import workloads as W


def _bits(a):
    return (np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32) >> 16).astype(np.uint16)


def test_signed_e4m3_matches_torch_cast():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.uniform(-447.0, 447.0, 4000), rng.normal(0, 1e-2, 2000),
                        rng.normal(0, 1e-3, 2000)]).astype(np.float32)
    # every E4M3 grid point and the midpoints between neighbours (the ties)
    grid = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)
    v = np.concatenate([v, grid.astype(np.float32), mids, -mids]).astype(np.float32)
    got = O.e4m3_encode_signed(v)
    want = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got, want)


def test_signed_e4m3_saturation_and_zeros():
    got = O.e4m3_encode_signed([448.0, 449.0, 1e6, -448.0, -1e6, 0.0, -0.0, -1e-12, 2.0 ** -10, 2.0 ** -10 * 1.5])
    assert [int(c) for c in got] == [0x7E, 0x7E, 0x7E, 0xFE, 0xFE, 0x00, 0x80, 0x80, 0x00, 0x01]


def test_fp8_scale():
    assert O.fp8_scale(448.0) == 1.0
    assert O.fp8_scale(0.0) == 1.0
    assert O.fp8_scale(896.0) == 2.0


def test_round_trip_of_representable_tensors():
    rng = np.random.default_rng(1)
    s = 0.03125  # a power of two: x = E4M3 value * s is exact in bf16 when the value has <= 4 bits
    codes = rng.integers(0, 0x7F, size=(12, 64)).astype(np.uint8) | (rng.integers(0, 2, size=(12, 64)) << 7).astype(np.uint8)
    vals = O.e4m3_decode(codes).astype(np.float32) * np.float32(s)
    x = _bits(vals)
    assert np.array_equal(O.bf16_bits_to_f32(x), vals)  # exactly representable
    got = O.quantize_fp8(x, s)
    # +0 and -0 codes both encode back as signed zeros of their value
    np.testing.assert_array_equal(O.e4m3_decode(got) * np.float32(s), vals)
    np.testing.assert_array_equal(got[codes % 0x80 != 0], codes[codes % 0x80 != 0])


def test_gemm_equals_textbook_matmul_on_representable_inputs():
    rng = np.random.default_rng(2)
    sa, sw = 0.5, 0.0078125
    ca = rng.integers(0, 0x7F, size=(9, 96)).astype(np.uint8) | (rng.integers(0, 2, size=(9, 96)) << 7).astype(np.uint8)
    cw = rng.integers(0, 0x7F, size=(7, 96)).astype(np.uint8) | (rng.integers(0, 2, size=(7, 96)) << 7).astype(np.uint8)
    xa = O.e4m3_decode(ca).astype(np.float32) * np.float32(sa)
    xw = O.e4m3_decode(cw).astype(np.float32) * np.float32(sw)
    qa, qw = O.quantize_fp8(_bits(xa), sa), O.quantize_fp8(_bits(xw), sw)
    y = O.gemm_fp8_f64(qa, sa, qw, sw)
    ref = xa.astype(np.float64) @ xw.astype(np.float64).T
    np.testing.assert_allclose(y, ref, rtol=1e-13, atol=1e-300)


def test_dynamic_scale_maps_amax_to_the_top_code():
    d = W.tiny()
    x = d["x"]
    s = O.fp8_scale(O.amax(x))
    c = O.quantize_fp8(x, s)
    assert (c & 0x7F).max() == 0x7E
