"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU).

Each test checks the oracle against something other than itself: a format definition written
out independently, a library routine (PyTorch's float8_e4m3fn cast), exact rational arithmetic,
brute force, closed forms, provable invariants, or a value the pages print.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------------------------------
# Independent restatements of the two number formats (from their bit-field definitions)
# ------------------------------------------------------------------------------------------

def e2m1_value_from_bits(code: int) -> float:
    """E2M1: sign | 2-bit exponent (bias 1) | 1-bit mantissa; exponent 0 is subnormal."""
    s = -1.0 if code & 8 else 1.0
    e = (code >> 1) & 3
    m = code & 1
    mag = (m * 0.5) if e == 0 else (2.0 ** (e - 1)) * (1.0 + m / 2.0)
    return s * mag


def e2m1_encode_by_thresholds(v: np.ndarray) -> np.ndarray:
    """Round to nearest E2M1 by decision thresholds (midpoints), ties to the even code."""
    v = np.asarray(v, dtype=np.float32)
    a = np.abs(v.astype(np.float64))
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    c = np.searchsorted(mids, a, side="left")  # number of midpoints strictly below a
    cc = np.minimum(c, 6)
    tie = (c < 7) & (a == mids[cc])
    c = np.where(tie & (c % 2 == 1), c + 1, c)
    c = np.minimum(c, 7)
    return (c | (np.signbit(v).astype(np.int64) << 3)).astype(np.uint8)


def e4m3_value_from_bits(code: int) -> float:
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0:
        return m * 2.0 ** -9
    return (1 + m / 8) * 2.0 ** (e - 7)


def all_finite_bf16_as_f32() -> np.ndarray:
    bits = np.arange(65536, dtype=np.uint32)
    f = (bits << 16).view(np.float32)
    return f[np.isfinite(f)]


# ------------------------------------------------------------------------------------------
# E2M1
# ------------------------------------------------------------------------------------------

def test_e2m1_decode_matches_bit_definition():
    for c in range(16):
        assert O.e2m1_decode([c])[0] == e2m1_value_from_bits(c)


def test_e2m1_encode_all_bf16_against_threshold_rounding():
    f = all_finite_bf16_as_f32()
    for scale in (1.0, 0.5, 3.0, 0.37, 7.25):
        with np.errstate(over="ignore"):
            v = (f * np.float32(scale)).astype(np.float32)
        v = v[np.isfinite(v)]
        np.testing.assert_array_equal(O.e2m1_encode(v), e2m1_encode_by_thresholds(v))


def test_e2m1_encode_next_to_every_midpoint():
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0], np.float32)
    vals = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 10)]).astype(np.float32)
    vals = np.concatenate([vals, -vals])
    np.testing.assert_array_equal(O.e2m1_encode(vals), e2m1_encode_by_thresholds(vals))


def test_e2m1_tie_table_and_sign_of_zero():
    # round half to even on the E2M1 grid: value -> expected code
    table = {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6, 6.0: 7, 100.0: 7, 0.0: 0}
    for v, c in table.items():
        assert O.e2m1_encode([v])[0] == c, v
        assert O.e2m1_encode([-v])[0] == c | 8, -v
    assert O.e2m1_encode([-0.1])[0] == 0x8  # sign kept when the magnitude rounds to zero


def test_e2m1_of_quotient_hits_ties_exactly():
    # d = 0.75 (an E4M3 value) is not a power of two, so x*(1/d) would round differently from x/d
    d = np.float32(0.75)
    for q, c in {0.25: 0, 0.75: 2, 1.25: 2, 1.75: 4, 2.5: 4, 3.5: 6, 5.0: 6}.items():
        x = np.float32(q * 0.75)
        assert float(x) == q * 0.75
        assert O.e2m1_of_quotient([x], d)[0] == c, q


# ------------------------------------------------------------------------------------------
# E4M3
# ------------------------------------------------------------------------------------------

def test_e4m3_decode_matches_bit_definition():
    for c in range(0x7F):
        assert O.e4m3_decode([c])[0] == np.float32(e4m3_value_from_bits(c))


def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(v, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_cast_in_range():
    f = all_finite_bf16_as_f32()
    f = f[(f >= 0) & (f <= 448)]
    rng = np.random.default_rng(0)
    rnd = rng.uniform(0, 448, 200000).astype(np.float32)
    small = (rng.uniform(0, 1, 50000) * 2.0 ** -6).astype(np.float32)
    vals = np.array([e4m3_value_from_bits(c) for c in range(0x7F)])
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    near = np.concatenate([mids, np.nextafter(mids, 0), np.nextafter(mids, 1000)]).astype(np.float32)
    v = np.concatenate([f, rnd, small, near])
    v = v[(v >= 0) & (v <= 448) & ~np.signbit(v)]  # scale inputs are non-negative (no -0.0)
    np.testing.assert_array_equal(O.e4m3_encode(v), _torch_e4m3(v))


def test_e4m3_saturation_and_underflow_by_hand():
    cases = {448.0: 0x7E, 449.0: 0x7E, 464.0: 0x7E, 1e9: 0x7E, 2.0 ** -10: 0x00,
             2.0 ** -10 * 1.001: 0x01, 2.0 ** -9: 0x01, 0.0: 0x00, 3 * 2.0 ** -10: 0x02}
    for v, c in cases.items():
        assert O.e4m3_encode([v])[0] == c, v


def test_e4m3_code_roundtrip():
    for c in range(0x7F):
        v = O.e4m3_decode([c])[0]
        assert O.e4m3_encode([v])[0] == c


# ------------------------------------------------------------------------------------------
# Tensor scale: golden values from the Day 0 page's scale rule
# ------------------------------------------------------------------------------------------

def test_tensor_scale_golden():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "day0_tensor_scale.txt")) if l.strip() and l[0] != "#"]
    for amax, want in rows:
        assert O.tensor_scale(float(amax)) == float(want)


# ------------------------------------------------------------------------------------------
# Block code: exact round trip of representable inputs
# ------------------------------------------------------------------------------------------

def representable_matrix(rows: int, K: int, seed: int, sf_lo: int = 0x20, sf_hi: int = 0x60):
    """bf16 rows built as E2M1 value * E4M3 scale with one +-6 per block (so amax/6 == sf)."""
    rng = np.random.default_rng(seed)
    codes = rng.integers(0, 16, size=(rows, K)).astype(np.uint8)
    sf = rng.integers(sf_lo, sf_hi, size=(rows, K // 16)).astype(np.uint8)
    pos = rng.integers(0, 16, size=(rows, K // 16))
    for m in range(rows):
        for b in range(K // 16):
            codes[m, 16 * b + pos[m, b]] = 7 | (codes[m, 16 * b + pos[m, b]] & 8)
    val = np.array([e2m1_value_from_bits(c) for c in range(16)])[codes] * \
        np.repeat(np.array([e4m3_value_from_bits(c) for c in range(128)])[sf], 16, axis=1)
    f = val.astype(np.float32)
    bits = (f.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal((bits.astype(np.uint32) << 16).view(np.float32), f)  # exact in bf16
    return bits, codes, sf


def test_block_roundtrip_representable():
    bits, codes, sf = representable_matrix(8, 128, 1)
    idx = np.array(list(range(5, 21)), np.int32)
    c, s, res = O.quantize_act(bits, idx, 1.0, want_residual=True)
    K = 128
    got = np.zeros((8, K), np.uint8)
    got[:, 0::2] = c[:, : K // 2] & 0xF
    got[:, 1::2] = c[:, : K // 2] >> 4
    # a +-0 input may come back with either sign bit only when its value is zero
    zero = (codes & 7) == 0
    np.testing.assert_array_equal(got[~zero], codes[~zero])
    np.testing.assert_array_equal(s[:, : K // 16], sf)
    assert np.all(res == 0.0)
    assert np.all(c[:, K // 2:] == 0) and np.all(s[:, K // 16:] == 0)
    deq = O.dequant(c, s)[:, :K]
    np.testing.assert_array_equal(deq, (bits.astype(np.uint32) << 16).view(np.float32))


def test_zero_blocks_give_zero_scale_and_codes():
    x = np.zeros((3, 64), np.uint16)
    x[1, :] = 0x8000  # -0.0
    c, s = O.quantize_act(x, np.arange(16, dtype=np.int32), 1.0)
    assert np.all(c == 0) and np.all(s == 0)


def test_main_segment_independent_of_r_and_r0_is_plain():
    d = W.tiny()
    st = O.tensor_scale(O.amax(d["x"]))
    c0, s0 = O.quantize_act(d["x"], np.zeros(0, np.int32), st)
    idx = O.calibrate(d["x"], 16)
    c1, s1 = O.quantize_act(d["x"], idx, st)
    K = d["K"]
    np.testing.assert_array_equal(c0[:, : K // 2], c1[:, : K // 2])
    np.testing.assert_array_equal(s0[:, : K // 16], s1[:, : K // 16])
    assert c0.shape[1] * 2 == 256 and np.all(s0.shape[1] == 16)


# ------------------------------------------------------------------------------------------
# Residual stage: provable error invariant on outlier channels
# ------------------------------------------------------------------------------------------

@pytest.mark.parametrize("which", ["tiny", "llama_rows"])
def test_residual_never_increases_error(which):
    if which == "tiny":
        d = W.tiny()
        x, r = d["x"], 16
    else:
        d = W.llama8b("qkv", rows=64, with_w=False)
        x, r = d["x"], 128
    st = O.tensor_scale(O.amax(x))
    idx = O.calibrate(x, r)
    c, s, res = O.quantize_act(x, idx, st, want_residual=True)
    K = x.shape[1]
    deq = O.dequant(c, s).astype(np.float64) * st
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    main = deq[:, idx]
    corr = deq[:, K: K + r]
    res = res.astype(np.float64)
    # the residual is x minus its primary dequantized value, up to one fp32 rounding each
    assert np.all(np.abs(res - (xf[:, idx] - main)) <= 2.0 ** -23 * (np.abs(xf[:, idx]) + np.abs(main)))
    # nearest rounding onto a grid that contains 0 never moves further than |res| away
    e_plain = np.abs(res)
    e_arc = np.abs(res - corr)
    assert np.all(e_arc <= e_plain)
    if np.any(c[:, K // 2: (K + r) // 2] != 0):
        assert np.sum(e_arc ** 2) < np.sum(e_plain ** 2)


# ------------------------------------------------------------------------------------------
# GEMM: linearity (main + correction), FP64 vs exact integers, brute force, textbook matmul
# ------------------------------------------------------------------------------------------

def _packed_tiny():
    d = W.tiny()
    idx = O.calibrate(d["x"], d["r"])
    sa = O.tensor_scale(O.amax(d["x"]))
    sw = O.tensor_scale(O.amax(d["w"]))
    ac, asf = O.quantize_act(d["x"], idx, sa)
    bc, bsf = O.pack_weight(d["w"], idx, sw)
    return d, idx, sa, sw, ac, asf, bc, bsf


def test_gemm_linearity_exact():
    d, idx, sa, sw, ac, asf, bc, bsf = _packed_tiny()
    K, kp = d["K"], ac.shape[1] * 2
    full = O.gemm_nvfp4_i64(ac, asf, bc, bsf)
    main = O.gemm_nvfp4_i64(ac, asf, bc, bsf, k_range=(0, K))
    corr = O.gemm_nvfp4_i64(ac, asf, bc, bsf, k_range=(K, kp))
    np.testing.assert_array_equal(full, main + corr)
    assert np.any(corr != 0)
    y = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw)
    yi = full.astype(np.float64) * 2.0 ** -20 * np.float64(np.float32(sa)) * np.float64(np.float32(sw))
    np.testing.assert_allclose(y, yi, rtol=1e-12, atol=1e-300)


def test_gemm_matmul_form_equals_scalar_loop():
    d, idx, sa, sw, ac, asf, bc, bsf = _packed_tiny()
    y1 = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw)
    y2 = O.gemm_nvfp4_f64_matmul(ac, asf, sa, bc, bsf, sw, rows=np.arange(16))
    np.testing.assert_allclose(y2, y1, rtol=1e-12, atol=1e-300)


def test_gemm_bruteforce_tiny():
    d, idx, sa, sw, ac, asf, bc, bsf = _packed_tiny()
    kp = ac.shape[1] * 2
    e2 = [e2m1_value_from_bits(c) for c in range(16)]
    e4 = [e4m3_value_from_bits(c) for c in range(128)]

    def deq_row(codes, sf, m):
        out = []
        for k in range(kp):
            b = int(codes[m, k // 2])
            c = (b >> 4) if k & 1 else (b & 15)
            out.append(e2[c] * e4[int(sf[m, k // 16])])
        return out

    A = [deq_row(ac, asf, m) for m in range(4)]
    B = [deq_row(bc, bsf, n) for n in range(0, 256, 37)]
    y = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw, rows=[0, 1, 2, 3])
    for i in range(4):
        for j, n in enumerate(range(0, 256, 37)):
            ref = float(np.float32(sa)) * float(np.float32(sw)) * sum(a * b for a, b in zip(A[i], B[j]))
            assert abs(y[i, n] - ref) <= 1e-12 * max(1.0, abs(ref))


def test_weight_duplicates_columns():
    d, idx, sa, sw, ac, asf, bc, bsf = _packed_tiny()
    # the appended weight columns are W[:, idx] re-blocked; quantizing W[:, idx] alone gives them
    sub = np.ascontiguousarray(d["w"][:, idx])
    c2, s2 = O.pack_weight(sub, np.zeros(0, np.int32), sw)
    K, r = d["K"], d["r"]
    np.testing.assert_array_equal(bc[:, K // 2: (K + r) // 2], c2[:, : r // 2])
    np.testing.assert_array_equal(bsf[:, K // 16: (K + r) // 16], s2[:, : r // 16])


def test_gemm_representable_equals_textbook_matmul():
    xa, _, _ = representable_matrix(16, 256, 2, 0x30, 0x40)
    wb, _, _ = representable_matrix(24, 256, 3, 0x30, 0x40)
    ac, asf = O.quantize_act(xa, np.zeros(0, np.int32), 1.0)
    bc, bsf = O.pack_weight(wb, np.zeros(0, np.int32), 1.0)
    y = O.gemm_nvfp4_f64(ac, asf, 1.0, bc, bsf, 1.0)
    X = O.bf16_bits_to_f32(xa).astype(np.float64)
    Wm = O.bf16_bits_to_f32(wb).astype(np.float64)
    np.testing.assert_allclose(y, X @ Wm.T, rtol=1e-13, atol=1e-13)


def test_gemm_bf16_bruteforce():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((5, 40)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    w = (rng.standard_normal((7, 40)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    y = O.gemm_bf16_f64(x, w)
    X = [[float(v) for v in row] for row in O.bf16_bits_to_f32(x)]
    Wm = [[float(v) for v in row] for row in O.bf16_bits_to_f32(w)]
    for i in range(5):
        for j in range(7):
            ref = math.fsum(a * b for a, b in zip(X[i], Wm[j]))
            assert abs(y[i, j] - ref) <= 1e-12 * max(1.0, abs(ref))


# ------------------------------------------------------------------------------------------
# Scale-factor layout
# ------------------------------------------------------------------------------------------

def test_sf_swizzle_positions_by_hand():
    rows, nsf = 256, 8
    canon = np.zeros((rows, nsf), np.uint8)
    marks = {(0, 0): 0, (1, 0): 16, (32, 0): 4, (64, 0): 8, (96, 0): 12, (0, 1): 1, (0, 3): 3,
             (0, 4): 512, (31, 7): 512 + 31 * 16 + 3, (128, 0): 1024, (255, 5): 1024 + 512 + 31 * 16 + 12 + 1}
    for i, (mk, off) in enumerate(marks.items()):
        canon[mk] = i + 1
    swz = O.sf_swizzle(canon)
    assert swz.size == 2 * 2 * 512
    for i, (mk, off) in enumerate(marks.items()):
        assert swz[off] == i + 1, (mk, off)
    np.testing.assert_array_equal(O.sf_unswizzle(swz, rows, nsf), canon)


def test_sf_swizzle_pads_rows_with_zero():
    canon = np.full((16, 20), 0x55, np.uint8)
    swz = O.sf_swizzle(canon)
    assert swz.size == 1 * 5 * 512
    assert np.count_nonzero(swz) == 16 * 20


# ------------------------------------------------------------------------------------------
# Calibration
# ------------------------------------------------------------------------------------------

def test_top_channels_ties_by_index():
    x = np.zeros((2, 6), np.float32)
    x[0] = [3, -5, 5, 1, 0, 5]
    x[1] = [1, 1, 1, 1, -7, 0]
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    assert list(O.calibrate(bits, 4)) == [4, 1, 2, 5]


def test_tiny_calibration_finds_planted_outliers():
    idx = O.calibrate(W.tiny()["x"], 16)
    assert list(idx[:2]) == [7, 131] or list(idx[:2]) == [131, 7]
    assert len(set(idx.tolist())) == 16


# ------------------------------------------------------------------------------------------
# RMSNorm and SwiGLU pieces
# ------------------------------------------------------------------------------------------

def test_row_sumsq_is_exact_then_rounded():
    rng = np.random.default_rng(5)
    for trial in range(40):
        n = int(rng.integers(1, 300))
        span = [0, 4, 20, 40][trial % 4]
        v = rng.standard_normal(n) * 2.0 ** rng.integers(-span, span + 1, n)
        bits = (v.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
        f = O.bf16_bits_to_f32(bits)
        exact = sum((Fraction(float(a)) ** 2 for a in f), Fraction(0))
        assert O.row_sumsq(bits) == float(exact)


def test_rmsnorm_closed_forms():
    c = np.float32(1.5)
    row = np.full((1, 64), (np.array([c]).view(np.uint32) >> 16)[0], np.uint16)
    out = O.bf16_bits_to_f32(O.rmsnorm(row, eps=0.0))
    assert np.all(out == 1.0)
    h = W.matrix_bf16(7, 1, 8, 2048)
    n = O.bf16_bits_to_f32(O.rmsnorm(h)).astype(np.float64)
    np.testing.assert_allclose(np.sqrt(np.mean(n * n, axis=1)), 1.0, rtol=3e-3)
    z = np.zeros((1, 32), np.uint16)
    assert np.all(O.rmsnorm(z) == 0)


def test_silu_mul_closed_forms():
    g = np.array([0.0, 1.0, 20.0, -20.0, 2.0], np.float32)
    u = np.array([3.0, 1.0, 0.5, 4.0, -1.0], np.float32)
    gu = (np.concatenate([g, u]).view(np.uint32) >> 16).astype(np.uint16)[None, :]
    a = O.bf16_bits_to_f32(O.silu_mul(gu))[0]
    want = [0.0, 1 / (1 + math.exp(-1)), 20.0 * 0.5 / (1 + math.exp(-20)), -20.0 * 4 / (1 + math.exp(20)),
            -2 / (1 + math.exp(-2))]
    for got, w in zip(a, want):
        assert abs(got - w) <= 2 ** -8 * abs(w) + 1e-30


# ------------------------------------------------------------------------------------------
# Page-printed numbers used by the benchmark's recurrent report
# ------------------------------------------------------------------------------------------

def test_ramp_ratio_formulas_reproduce_page_numbers():
    line = [l for l in open(os.path.join(GOLDEN, "ramp_prefill_latency.txt")) if l.strip() and l[0] != "#"][0]
    bf16_ms, ramp_ms, speedup, red = map(float, line.split())
    assert round(bf16_ms / ramp_ms, 4) == speedup
    assert round(100 * (1 - ramp_ms / bf16_ms), 1) == red
