"""Pins of the oracle's MXFP4 reading (ARCQuant's "extends to MXFP4", read as the OCP microscaling
format: 32-value blocks, one power-of-two scale X = 2^(floor(log2 amax) - 2) stored as E8M0,
E2M1 elements). The E2M1 element codec is pinned elsewhere; these pin the scale rule, the exact
power-of-two scaling, and the GEMM.
"""
import numpy as np

import oracle as O

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _bits(a):
    return (np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32) >> 16).astype(np.uint16)


def test_scale_byte_by_hand():
    # floor(log2 6) = 2 -> X = 1; floor(log2 0.75) = -1 -> X = 2^-3; clamps at both ends
    cases = {6.0: 127, 7.0: 127, 7.99: 127, 8.0: 128, 0.75: 124, 1.0: 125, 0.0: 0, 2.0 ** -130: 0,
             3.0e38: 252}
    for a, want in cases.items():
        assert O.mxfp4_scale_byte(a) == want, (a, O.mxfp4_scale_byte(a))


def test_scaled_block_maximum_lies_in_4_to_8():
    # the defining property of X = 2^(floor(log2 amax) - 2): amax / X in [4, 8)
    rng = np.random.default_rng(0)
    x = _bits(rng.standard_normal((64, 256)) * np.exp(rng.uniform(-20, 20, size=(64, 1))))
    codes, sc = O.quantize_mxfp4(x)
    v = O.bf16_bits_to_f32(x).astype(np.float64).reshape(64, 8, 32)
    amax = np.abs(v).max(axis=2)
    ratio = amax / np.ldexp(1.0, sc.astype(np.int64) - 127)
    assert np.all((ratio >= 4) & (ratio < 8)), ratio.min()


def test_round_trip_of_representable_blocks():
    # each block: E2M1 magnitudes times 2^e with the block maximum 6 * 2^e (so the scale is 2^e)
    rng = np.random.default_rng(1)
    M, nb = 6, 4
    e = rng.integers(-20, 20, size=(M, nb))
    mags = E2M1[rng.integers(0, 8, size=(M, nb, 32))]
    mags[:, :, 0] = 6.0
    signs = np.where(rng.integers(0, 2, size=mags.shape) == 1, -1.0, 1.0)
    vals = (signs * mags * np.ldexp(1.0, e)[:, :, None]).reshape(M, nb * 32).astype(np.float32)
    x = _bits(vals)
    assert np.array_equal(O.bf16_bits_to_f32(x), vals)
    codes, sc = O.quantize_mxfp4(x)
    np.testing.assert_array_equal(sc, (e + 127).astype(np.uint8))
    lo, hi = codes & 15, codes >> 4
    c = np.stack([lo, hi], axis=2).reshape(M, nb * 32)
    deq = np.where(c & 8, -1.0, 1.0) * E2M1[c & 7] * np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=1))
    np.testing.assert_array_equal(np.abs(deq), np.abs(vals.astype(np.float64)))
    nz = vals != 0
    np.testing.assert_array_equal(np.sign(deq[nz]), np.sign(vals[nz]))


def test_error_within_one_scale_and_zero_blocks():
    rng = np.random.default_rng(2)
    v = rng.standard_normal((16, 128)).astype(np.float32)
    v[3, 32:64] = 0.0
    x = _bits(v)
    codes, sc = O.quantize_mxfp4(x)
    assert sc[3, 1] == 0 and not codes[3, 16:32].any()
    lo, hi = codes & 15, codes >> 4
    c = np.stack([lo, hi], axis=2).reshape(16, 128)
    X = np.ldexp(1.0, np.repeat(sc.astype(np.int64) - 127, 32, axis=1))
    deq = np.where(c & 8, -1.0, 1.0) * E2M1[c & 7] * X
    xv = O.bf16_bits_to_f32(x).astype(np.float64)
    # below saturation every element is within half of E2M1's widest step (4 -> 6), one X; the
    # scale rule lets a block maximum reach up to 8 X, and values above 6 X saturate to +-6 X
    unsat = np.abs(xv) <= 6 * X
    assert np.all(np.abs(xv - deq)[unsat] <= X[unsat])
    assert np.all(np.abs(deq[~unsat]) == 6 * X[~unsat]) and np.any(~unsat)


def test_gemm_equals_textbook_matmul_on_representable_inputs():
    rng = np.random.default_rng(3)

    def rep(M, K):
        mags = E2M1[rng.integers(0, 8, size=(M, K))]
        mags[:, ::32] = 6.0
        e = np.repeat(rng.integers(-6, 6, size=(M, K // 32)), 32, axis=1)
        s = np.where(rng.integers(0, 2, size=(M, K)) == 1, -1.0, 1.0)
        return (s * mags * np.ldexp(1.0, e)).astype(np.float32)

    xa, xw = rep(9, 128), rep(7, 128)
    ac, asc = O.quantize_mxfp4(_bits(xa))
    bc, bsc = O.quantize_mxfp4(_bits(xw))
    y = O.gemm_mxfp4_f64(ac, asc, bc, bsc)
    np.testing.assert_allclose(y, xa.astype(np.float64) @ xw.astype(np.float64).T, rtol=1e-14, atol=0)
