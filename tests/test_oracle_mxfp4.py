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


# ---------------------------------------------------------------------------------------------
# MXFP4 with augmented residual channels (ARCQuant, Resultaten / Generaliseerbaarheid: the
# approach extends to MXFP4): the dual-stage code with 32-value MXFP4 blocks. Each pin below is
# built without the C code's block routine, so a slip in it (a wrong block, a dropped residual
# term, the wrong scale of the deducted value) fails one of them.
# ---------------------------------------------------------------------------------------------

MIDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def _np_e2m1(v):
    """Independent E2M1 encoder: nearest grid magnitude, ties to the even code, saturation at
    6, sign bit from the sign of v (also for values that round to zero)."""
    v = np.asarray(v, np.float64)
    m = np.abs(v)
    code = np.searchsorted(MIDS, m, side="left")  # number of midpoints strictly below m
    tie = np.isin(m, MIDS)
    code = np.where(tie & (code % 2 == 1), code + 1, code)  # on a midpoint, take the even neighbour
    code = np.minimum(code, 7)
    return (code | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def _np_mxfp4_blocks(vals):
    """Independent MXFP4 of fp32 rows (K % 32 == 0): codes [M, K] (one per element) and scale
    bytes [M, K/32], the scale exponent from frexp."""
    v = np.asarray(vals, np.float32)
    M, K = v.shape
    blk = v.reshape(M, K // 32, 32)
    amax = np.abs(blk).max(axis=2).astype(np.float64)
    _, e2 = np.frexp(amax)
    sb = np.where(amax > 0, np.clip(e2 - 1 - 2 + 127, 0, 254), 0).astype(np.int64)
    scaled = np.ldexp(blk, (127 - sb)[:, :, None].astype(np.int32)).astype(np.float32)
    codes = np.where((amax > 0)[:, :, None], _np_e2m1(scaled), 0).astype(np.uint8)
    return codes.reshape(M, K), sb.astype(np.uint8)


def _unpack(codes):
    lo, hi = codes & 15, codes >> 4
    return np.stack([lo, hi], axis=2).reshape(codes.shape[0], -1)


def _deq(c, sb):
    X = np.ldexp(1.0, np.repeat(sb.astype(np.int64) - 127, 32, axis=1))
    return np.where(c & 8, -1.0, 1.0) * E2M1[c & 7] * X


def test_np_encoder_agrees_with_the_plain_oracle_block():
    rng = np.random.default_rng(10)
    v = (rng.standard_t(3, size=(20, 256)) * np.exp(rng.uniform(-8, 8, size=(20, 1)))).astype(np.float32)
    x = _bits(v)
    codes, sc = O.quantize_mxfp4(x)
    c_np, sb_np = _np_mxfp4_blocks(O.bf16_bits_to_f32(x))
    np.testing.assert_array_equal(sc, sb_np)
    np.testing.assert_array_equal(_unpack(codes), c_np)


def test_arc_without_channels_is_plain_mxfp4():
    rng = np.random.default_rng(11)
    x = _bits(rng.standard_normal((33, 512)))
    c0, s0 = O.quantize_mxfp4(x)
    c1, s1 = O.quantize_act_mxfp4(x, np.zeros(0, np.int32))
    np.testing.assert_array_equal(c0, c1)
    np.testing.assert_array_equal(s0, s1)


def test_weight_pack_equals_mxfp4_of_the_explicit_augmented_matrix():
    rng = np.random.default_rng(12)
    N, K, r = 24, 320, 64  # K + r = 384: no padding; also check a padded case below
    for K, r in ((320, 64), (256, 32)):
        w = _bits(rng.standard_normal((N, K)) * 0.02)
        idx = rng.choice(K, size=r, replace=False).astype(np.int32)
        kp = (K + r + 63) // 64 * 64
        waug = np.zeros((N, kp), np.uint16)
        waug[:, :K] = w
        waug[:, K:K + r] = w[:, idx]
        c_ref, s_ref = O.quantize_mxfp4(waug)
        c, s = O.pack_weight_mxfp4(w, idx)
        np.testing.assert_array_equal(c, c_ref)
        np.testing.assert_array_equal(s, s_ref)


def test_activation_residual_blocks_against_an_independent_construction():
    rng = np.random.default_rng(13)
    M, K, r = 40, 512, 64
    v = rng.standard_normal((M, K)).astype(np.float32)
    hot = rng.choice(K, size=12, replace=False)
    v[:, hot] *= rng.uniform(20, 80, size=12).astype(np.float32)
    x = _bits(v)
    xf = O.bf16_bits_to_f32(x)
    idx = np.argsort(-np.abs(xf).max(axis=0), kind="stable")[:r].astype(np.int32)
    codes, sc, res = O.quantize_act_mxfp4(x, idx, want_residual=True)
    # primary part: plain MXFP4 of X
    cp, sp = O.quantize_mxfp4(x)
    np.testing.assert_array_equal(codes[:, :K // 2], cp)
    np.testing.assert_array_equal(sc[:, :K // 32], sp)
    # residual of each outlier channel: x - E2M1(code) * X in fp32 (the product is exact)
    deq = _deq(_unpack(cp), sp).astype(np.float32)
    R = (xf[:, idx] - deq[:, idx]).astype(np.float32)
    np.testing.assert_array_equal(res, R)
    c_np, sb_np = _np_mxfp4_blocks(R)
    np.testing.assert_array_equal(_unpack(codes)[:, K:K + r], c_np)
    np.testing.assert_array_equal(sc[:, K // 32:(K + r) // 32], sb_np)
    # padding to K_pad is zero
    assert not _unpack(codes)[:, K + r:].any() and not sc[:, (K + r) // 32:].any()


def test_residual_never_increases_the_error_and_vanishes_on_representable_rows():
    rng = np.random.default_rng(14)
    M, K, r = 30, 256, 32
    x = _bits(rng.standard_t(3, size=(M, K)) * 3)
    xf = O.bf16_bits_to_f32(x).astype(np.float64)
    idx = rng.choice(K, size=r, replace=False).astype(np.int32)
    codes, sc = O.quantize_act_mxfp4(x, idx)
    c = _unpack(codes)
    deq_main = _deq(c[:, :K], sc[:, :K // 32])[:, idx]
    deq_res = _deq(c[:, K:K + r], sc[:, K // 32:(K + r) // 32])
    e_plain = np.abs(xf[:, idx] - deq_main)
    e_arc = np.abs(xf[:, idx] - deq_main - deq_res)
    assert np.all(e_arc <= e_plain)
    assert e_arc.sum() < e_plain.sum()
    # representable rows leave zero residuals: appended codes and scale bytes all zero
    mags = E2M1[rng.integers(0, 8, size=(M, K))]
    mags[:, ::32] = 6.0
    rep = (mags * np.ldexp(1.0, np.repeat(rng.integers(-5, 5, size=(M, K // 32)), 32, axis=1))).astype(np.float32)
    c2, s2 = O.quantize_act_mxfp4(_bits(rep), idx)
    assert not c2[:, K // 2:].any() and not s2[:, K // 32:].any()


def test_augmented_gemm_is_main_plus_correction():
    rng = np.random.default_rng(15)
    M, N, K, r = 12, 10, 256, 64
    x = _bits(rng.standard_normal((M, K)))
    w = _bits(rng.standard_normal((N, K)) * 0.02)
    idx = rng.choice(K, size=r, replace=False).astype(np.int32)
    ac, asc = O.quantize_act_mxfp4(x, idx)
    bc, bsc = O.pack_weight_mxfp4(w, idx)
    y = O.gemm_mxfp4_f64(ac, asc, bc, bsc)
    a = _deq(_unpack(ac), asc)
    b = _deq(_unpack(bc), bsc)
    main = a[:, :K] @ b[:, :K].T
    corr = a[:, K:K + r] @ b[:, K:K + r].T
    np.testing.assert_allclose(y, main + corr, rtol=1e-12, atol=1e-30)
    # the correction pairs each residual with its duplicated weight column
    np.testing.assert_allclose(corr, a[:, K:K + r] @ _deq(_unpack(O.quantize_mxfp4(w[:, idx])[0]),
                                                         O.quantize_mxfp4(w[:, idx])[1]).T, rtol=1e-12)
