"""The seeded input generator: determinism, slice independence and the recipes' structure."""
import numpy as np

import workloads as W


def test_deterministic_and_sliceable():
    a = W.matrix_bf16(11, 1, 64, 96, 1.0)
    b = W.matrix_bf16(11, 1, 64, 96, 1.0, threads=1)
    np.testing.assert_array_equal(a, b)
    c = W.matrix_bf16(11, 1, 20, 96, 1.0, row0=30)
    np.testing.assert_array_equal(a[30:50], c)
    d = W.matrix_bf16(12, 1, 64, 96, 1.0)
    assert not np.array_equal(a, d)


def test_normal_and_t3_moments():
    x = (W.matrix_bf16(1, 1, 512, 512, 1.0).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1) < 0.01
    t = (W.matrix_bf16(1, 1, 512, 512, 1.0, dist="t3").astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    # Student-t(3): variance 3, heavy tails
    assert abs(np.median(np.abs(t)) - 0.765) < 0.02 and np.abs(t).max() > 20


def test_tiny_recipe_plants_outliers():
    d = W.tiny()
    x = (d["x"].astype(np.uint32) << 16).view(np.float32)
    colmax = np.abs(x).max(axis=0)
    assert set(np.argsort(-colmax)[:2].tolist()) == {7, 131}
    assert d["x"].shape == (16, 256) and d["w"].shape == (256, 256)


def test_outlier_channels_distinct_and_counted():
    d = W.llama8b("down", rows=8, with_w=False)
    assert len(d["outliers"]) == round(0.01 * 14336)
    m = W.outlier_multipliers(1, 3, 14336, 143, 20.0, 80.0)
    assert np.all((m[m != 1] >= 20) & (m[m != 1] <= 80))
