"""The seeded generators: determinism and the stated outlier structure."""

import numpy as np

from bit_gemm_w4_b200 import synth


def test_weight_deterministic_and_outlier_count():
    a = synth.weight(64, 256, std=0.02, outlier_frac=0.01, seed=5)
    b = synth.weight(64, 256, std=0.02, outlier_frac=0.01, seed=5)
    assert a.dtype == np.float32 and np.array_equal(a, b)
    assert np.abs(a).max() > 0.1
    assert abs(float(a[np.abs(a) < 0.1].std()) - 0.02) < 0.002


def test_clustered_outlier_columns():
    W = synth.weight(200, 1024, std=0.015, outlier_frac=0.01, outlier_cols=8, seed=3)
    heavy = (np.abs(W) > 0.1).mean(axis=0)
    assert (heavy > 0.3).sum() == 8          # the 8 whole outlier columns
    rows = synth.weight(200, 1024, std=0.015, outlier_frac=0.01, outlier_cols=8,
                        seed=3, rows=[5, 150])
    assert np.array_equal(rows, W[[5, 150]])


def test_activation_channels():
    X = synth.activations(4, 512, seed=1, channels=4, mult=20.0).float().numpy()
    big = np.abs(X).max(axis=0) > 8
    assert big.sum() >= 3


def test_sweep_decomposition_structure():
    d = synth.sweep_decomposition(50, 4096, 41, seed=2)
    assert d["row_ptr"][-1] == 50 * 41
    cols = d["col"].reshape(50, 41)
    assert np.all(np.diff(cols, axis=1) > 0)
    assert np.all(d["qr"] != 0) and d["qr"].min() >= -8 and d["qr"].max() <= 7
    assert abs(d["clustered_frac"] - 29 / 41) < 1e-12
