"""Pin the oracle's product Y = X * W_hat^T (MosaicQuant, "Methodology" 3.:
the dense GEMM and the sparse residual end in one reduction-add).

Pins: density 0 reduces to a plain W4 GEMM (checked with torch.matmul); a
full-density unquantized residual reproduces W bit-exactly; the brute-force
triple loop; row and K-group permutations; the hand-derived example.
"""

import numpy as np
import torch

from oracle import decompose, dequant_base, w_hat, linear, linear_brute
from bit_gemm_w4_b200 import synth


def test_density_zero_is_plain_w4_gemm():
    W = synth.weight(64, 512, std=0.02, outlier_frac=0.01, seed=3)
    X = synth.activations(5, 512, seed=4, channels=4, mult=20.0)
    d = decompose(W, 0.0)
    assert d.nnz == 0
    ref = torch.matmul(X.double(), torch.from_numpy(dequant_base(d)).T).numpy()
    np.testing.assert_allclose(linear(X, d), ref, rtol=1e-12, atol=1e-12)


def test_full_density_exact_residual_reproduces_w():
    W = synth.weight(16, 256, std=0.02, outlier_frac=0.02, seed=8)
    d = decompose(W, 1.0, exact_residual=True)
    assert d.nnz == W.size
    assert np.array_equal(w_hat(d), W.astype(np.float64))
    X = synth.activations(3, 256, seed=9)
    ref = X.double().numpy() @ W.astype(np.float64).T
    np.testing.assert_allclose(linear(X, d), ref, rtol=1e-12, atol=1e-12)


def test_brute_force_8x8_and_8x128():
    rng = np.random.default_rng(1)
    W = (rng.standard_normal((8, 8)) * 0.02).astype(np.float32)
    W[3, 5] = 0.7
    d = decompose(W, 0.25, group=8)
    X = rng.standard_normal((2, 8))
    np.testing.assert_allclose(linear(X, d), linear_brute(X, d), rtol=1e-12, atol=1e-13)
    W = synth.weight(8, 128, std=0.02, outlier_frac=0.03, seed=2)
    d = decompose(W, 0.05)
    X = synth.activations(3, 128, seed=5)
    np.testing.assert_allclose(linear(X, d), linear_brute(X, d), rtol=1e-12, atol=1e-13)


def test_row_permutation_permutes_outputs():
    W = synth.weight(32, 256, std=0.02, outlier_frac=0.01, seed=12)
    X = synth.activations(4, 256, seed=13)
    perm = np.random.default_rng(0).permutation(32)
    Y = linear(X, decompose(W, 0.02))
    Yp = linear(X, decompose(np.ascontiguousarray(W[perm]), 0.02))
    np.testing.assert_allclose(Yp, Y[:, perm], rtol=1e-12, atol=1e-12)


def test_group_permutation_with_x_columns_is_invariant():
    W = synth.weight(16, 512, std=0.02, outlier_frac=0.01, seed=21)
    X = synth.activations(3, 512, seed=22)
    gp = np.array([2, 0, 3, 1])
    cols = (gp[:, None] * 128 + np.arange(128)).reshape(-1)
    d = decompose(W, 0.02)
    dp = decompose(np.ascontiguousarray(W[:, cols]), 0.02)
    np.testing.assert_array_equal(dp.s, d.s[:, gp])
    np.testing.assert_array_equal(dp.q, d.q[:, cols])
    np.testing.assert_allclose(linear(X[:, cols], dp), linear(X, d), rtol=1e-11, atol=1e-12)


def test_rows_subset_matches_full():
    W = synth.weight(40, 256, std=0.02, outlier_frac=0.01, seed=30)
    X = synth.activations(2, 256, seed=31)
    d = decompose(W, 0.03)
    rows = np.array([39, 0, 17])
    np.testing.assert_allclose(linear(X, d, rows=rows), linear(X, d)[:, rows], rtol=0, atol=0)


def test_hand_derived_example(golden):
    f = golden("hand_group8.txt")
    v = np.array([float(x) for x in f["v"]], np.float32).reshape(1, -1)
    d = decompose(v, float(f["rho"][0]), group=int(f["group"][0]))
    x = np.array([[float(a) for a in f["x"]]])
    assert linear(x, d)[0, 0] == float(f["y"][0])
    assert linear_brute(x, d)[0, 0] == float(f["y"][0])
