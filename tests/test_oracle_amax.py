"""Pins of the oracle's tensor abs-max and tensor scale (CPU).

The dynamic tensor scale is s = amax(|x|) / 2688 with s = 1 for an all-zero tensor ("Day 0 LLM
Inference Support…", section V: scale = amax / FMT_MAX with an all-zero guard; 2688 = 6 * 448 is
the largest magnitude of the two-level NVFP4 code). The abs-max is a plain definition, so it is
pinned against numpy's max of |x| over the decoded bf16 values, on inputs built so that the
plausible slips fail: a signed max instead of |x| (the extreme is negative), a dropped last row or
column (the extreme sits there), the row pitch taken for the row length (the padding between rows
holds larger values that must be ignored), the row split of the threaded wrapper (many row counts).
"""
import ctypes

import numpy as np
import pytest

import oracle as O


def _bf16(f32: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _numpy_amax(bits: np.ndarray) -> float:
    if bits.size == 0:
        return 0.0
    return float(np.max(np.abs(O.bf16_bits_to_f32(bits))))


def _c_amax(bits_padded: np.ndarray, rows: int, cols: int) -> float:
    """The C function on a row-major buffer whose row pitch is bits_padded.shape[1]."""
    a = np.ascontiguousarray(bits_padded)
    return float(O.lib().oracle_amax_bf16(a.ctypes.data_as(ctypes.c_void_p), rows, cols, a.shape[1]))


@pytest.mark.parametrize("rows,cols,pad", [(1, 16, 0), (7, 33, 5), (64, 256, 16), (130, 1000, 24), (513, 48, 1)])
@pytest.mark.parametrize("where", ["last_row_last_col", "first", "middle"])
def test_amax_matches_numpy_with_negative_extremes_and_row_pitch(rows, cols, pad, where):
    rng = np.random.default_rng(rows * 1000 + cols + pad)
    x = rng.standard_normal((rows, cols + pad)).astype(np.float32)
    # the padding columns hold larger magnitudes than any real entry: reading them is a bug
    x[:, cols:] = 1.0e4
    i, k = {"last_row_last_col": (rows - 1, cols - 1), "first": (0, 0), "middle": (rows // 2, cols // 2)}[where]
    x[i, k] = -37.5  # the extreme is negative: a signed max would miss it
    bits = _bf16(x)
    want = _numpy_amax(bits[:, :cols])
    assert want == 37.5
    assert _c_amax(bits, rows, cols) == want
    # the threaded wrapper (contiguous rows, split across threads)
    assert O.amax(np.ascontiguousarray(bits[:, :cols])) == want


def test_amax_of_random_tensors_equals_numpy():
    rng = np.random.default_rng(11)
    for rows in (1, 2, 63, 64, 65, 127, 1000, 4099):
        cols = int(rng.integers(1, 300))
        x = (rng.standard_t(3, size=(rows, cols)) * rng.uniform(0.01, 100)).astype(np.float32)
        bits = _bf16(x)
        assert O.amax(bits) == _numpy_amax(bits), rows


def test_amax_special_values():
    # signed zeros, subnormal bf16 values, the largest finite bf16 magnitude
    z = np.array([[0x8000, 0x0000, 0x8000]], np.uint16)
    assert O.amax(z) == 0.0
    sub = np.array([[0x0001, 0x8003, 0x0002]], np.uint16)  # bf16 subnormals: 3 * 2^-133 is the largest
    assert O.amax(sub) == float(np.float32(3.0) * np.float32(2.0) ** -133)
    big = np.array([[0x3F80, 0xFF7F, 0x7F7E]], np.uint16)  # 1, -max finite, slightly smaller positive
    assert O.amax(big) == float(O.bf16_bits_to_f32(np.array([0x7F7F], np.uint16))[0])


def test_tensor_scale_of_the_amax():
    # s = fp32(amax / 2688), divide form; an all-zero tensor gives 1
    rng = np.random.default_rng(5)
    for _ in range(200):
        a = np.float32(rng.uniform(1e-3, 1e3))
        assert O.tensor_scale(float(a)) == float(np.float32(a) / np.float32(2688.0))
    assert O.tensor_scale(0.0) == 1.0
    assert O.tensor_scale(2688.0) == 1.0
