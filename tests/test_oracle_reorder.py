"""Pins of the oracle's channel reorder (ARCQuant, Methodologie: adaptive outlier identification
reorders the channels by their absolute maxima; the primary stage quantizes the reordered
activation; the weights are reordered alike and their outlier columns duplicated).

The order is checked against an independent integer sort, and the reordered encodings against
properties the reorder must give: block scales that cannot increase along the row of the
calibration tensor, appended weight blocks identical to the first primary blocks, the residual
invariant, and a worked example where grouping the outliers saves the small channels.
"""
import numpy as np
import pytest

import oracle as O
import workloads as W


def _bits(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32).__rshift__(16).astype(np.uint16)


def test_order_matches_integer_sort():
    # |bf16| orders like its 15 magnitude bits, so a stable sort of those integers (descending,
    # ties by ascending channel) is the order the pages' reordering by abs-max defines
    for seed, (M, K) in enumerate([(16, 256), (7, 96), (33, 512)]):
        rng = np.random.default_rng(seed)
        x = _bits(rng.standard_normal((M, K)) * rng.choice([1.0, 30.0], size=K, p=[0.9, 0.1]))
        x[:, 5] = x[:, 9]  # a tie
        key = (x & 0x7FFF).max(axis=0).astype(np.int64)
        want = np.lexsort((np.arange(K), -key))
        got = O.calibrate_order(x)
        np.testing.assert_array_equal(got, want)
        assert sorted(got.tolist()) == list(range(K))
        for r in (16, 32, 64):
            np.testing.assert_array_equal(got[:r], O.calibrate(x, r))


def test_reordered_block_scales_do_not_increase():
    # on the calibration tensor itself, the largest block amax over rows of primary block b is
    # the abs-max of its first (largest) channel, which cannot increase with b; E4M3 rounding is
    # monotone, so neither can the largest scale byte
    d = W.tiny()
    x, r = d["x"], d["r"]
    perm = O.calibrate_order(x)
    s = O.tensor_scale(O.amax(x))
    codes, sf = O.quantize_act_reordered(x, perm, r, s)
    K = x.shape[1]
    top = sf[:, : K // 16].max(axis=0).astype(int)
    assert np.all(np.diff(top) <= 0), top
    # without the reorder the outlier channels 7 and 131 sit in blocks 0 and 8
    _, sf0 = O.quantize_act(x, O.calibrate(x, r), s)
    top0 = sf0[:, : K // 16].max(axis=0).astype(int)
    assert np.any(np.diff(top0) > 0)


def test_reordered_weight_appends_copies_of_first_blocks():
    # W_aug = [W[:, perm] | W[:, perm[:r]]]: the duplicated channels are the first r reordered
    # columns, blocked the same way under the same tensor scale, so the appended blocks repeat
    # primary blocks 0 .. r/16 - 1 exactly
    d = W.tiny()
    w = d["w"]
    K = w.shape[1]
    perm = O.calibrate_order(d["x"])
    for r in (16, 48):
        s_w = O.tensor_scale(O.amax(w))
        codes, sf = O.pack_weight_reordered(w, perm, r, s_w)
        np.testing.assert_array_equal(codes[:, K // 2: (K + r) // 2], codes[:, : r // 2])
        np.testing.assert_array_equal(sf[:, K // 16: (K + r) // 16], sf[:, : r // 16])
        assert not codes[:, (K + r) // 2:].any() and not sf[:, (K + r) // 16:].any()


def test_identity_order_is_the_plain_path():
    d = W.tiny()
    x = d["x"]
    K = x.shape[1]
    s = O.tensor_scale(O.amax(x))
    a = O.quantize_act_reordered(x, np.arange(K), 32, s)
    b = O.quantize_act(x, np.arange(32, dtype=np.int32), s)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


def test_reordered_residual_invariant():
    # the residual stage never makes an outlier channel worse: |x - deq - deq_res| <= |x - deq|
    d = W.tiny()
    x, r = d["x"], d["r"]
    perm = O.calibrate_order(x)
    s = O.tensor_scale(O.amax(x))
    codes, sf = O.quantize_act_reordered(x, perm, r, s)
    K = x.shape[1]
    deq = O.dequant(codes, sf).astype(np.float64) * s
    xv = O.bf16_bits_to_f32(x).astype(np.float64)[:, perm[:r]]
    prim = deq[:, :r]
    both = prim + deq[:, K: K + r]
    assert np.all(np.abs(xv - both) <= np.abs(xv - prim) + 1e-30)
    assert np.linalg.norm(xv - both) < np.linalg.norm(xv - prim)


def test_worked_example_grouping_saves_small_channels():
    # one row, 32 channels: two outliers (x40) at channels 3 and 20, the rest 0.1 .. 0.41. In
    # the natural order both blocks carry an outlier, the block scale is ~40/6 and every small
    # value codes to 0; reordered, both outliers and the 14 largest small values share block 0,
    # and block 1 holds the 16 smallest values only, which it codes with a scale of their own
    vals = np.array([0.1 + 0.01 * i for i in range(32)], np.float32)
    vals[3], vals[20] = 40.0, -40.0
    x = _bits(vals[None, :])
    s = O.tensor_scale(O.amax(x))
    perm = O.calibrate_order(x)
    assert set(perm[:2].tolist()) == {3, 20}
    c0, f0 = O.quantize_act(x, np.zeros(0, np.int32), s)
    c1, f1 = O.quantize_act_reordered(x, perm, 0, s)
    xv = O.bf16_bits_to_f32(x).astype(np.float64)[0]
    e0 = np.abs(xv - O.dequant(c0, f0)[0, :32] * s)
    e1 = np.abs(xv[perm] - O.dequant(c1, f1)[0, :32] * s)
    small0 = np.delete(e0, [3, 20])
    small1 = e1[2:]
    assert np.all(O.dequant(c0, f0)[0, np.r_[0:3, 4:20, 21:32]] == 0)  # natural order: all lost
    assert np.all(O.dequant(c1, f1)[0, 16:32] != 0)  # reordered block 1: none lost
    # within half of E2M1's widest step (4 -> 6, i.e. one decode scale d) of block 1's own scale
    d1 = float(O.e4m3_decode(np.array([f1[0, 1]], np.uint8))[0]) * s
    assert d1 < 0.05 and np.all(e1[16:32] <= d1)
    assert np.linalg.norm(small1) < np.linalg.norm(small0)


@pytest.mark.parametrize("r", [0, 16])
def test_reordered_gemm_is_the_permuted_dot_product(r):
    # the reordered augmented GEMM sums the same products in another order: equal to the
    # FP64 GEMM of the dequantized operands mapped back to the natural channel order
    d = W.tiny()
    x, w = d["x"], d["w"]
    K = x.shape[1]
    perm = O.calibrate_order(x)
    sa, sw = O.tensor_scale(O.amax(x)), O.tensor_scale(O.amax(w))
    ac, asf = O.quantize_act_reordered(x, perm, r, sa)
    bc, bsf = O.pack_weight_reordered(w, perm, r, sw)
    y = O.gemm_nvfp4_f64(ac, asf, sa, bc, bsf, sw)
    A = O.dequant(ac, asf).astype(np.float64) * sa
    B = O.dequant(bc, bsf).astype(np.float64) * sw
    An = np.zeros((x.shape[0], K)); Bn = np.zeros((w.shape[0], K))
    An[:, perm] = A[:, :K]; Bn[:, perm] = B[:, :K]
    ref = An @ Bn.T + A[:, K: K + r] @ B[:, K: K + r].T
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-12)
