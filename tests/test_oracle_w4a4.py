"""Pin the oracle's W4A4 variant (MosaicQuant, "Methodology" 3.: the
pipeline's quantization stage ahead of the fused GEMM; "Experimental
Results": W4A4).

Pins: every activation code is the nearest int4 value of x / s_x (brute
force over the 16 codes, ties to even); the per-token scale; ties; zero
tokens; power-of-two scaling; activations already on the int4 grid give the
W4A16 oracle's result exactly; in general the result equals the W4A16
oracle on the dequantized activations, and the brute-force triple loop.
"""

import numpy as np
import pytest
import torch

from oracle import decompose, linear, linear_brute
from oracle.w4a4 import quantize_activations, dequantized_activations, linear_w4a4
from bit_gemm_w4_b200 import synth


def _nearest_code(v: np.float32) -> int:
    """The int4 code nearest to v, ties to the even code (brute force)."""
    best, bd = None, None
    for c in range(-8, 8):
        dist = abs(float(v) - c)
        if bd is None or dist < bd - 1e-12 or (abs(dist - bd) <= 1e-12 and c % 2 == 0):
            best, bd = c, dist
    return best


def test_codes_are_nearest_brute_force():
    X = synth.activations(4, 256, seed=61, channels=3, mult=25.0)
    c, s = quantize_activations(X)
    Xf = X.float().numpy()
    for m in range(4):
        for k in range(0, 256, 7):
            v = np.float32(Xf[m, k]) / s[m]        # the fp32 quotient the reading fixes
            assert c[m, k] == _nearest_code(np.float32(v)), (m, k)


def test_scale_is_max_over_seven():
    X = synth.activations(6, 512, seed=62, channels=2, mult=30.0)
    c, s = quantize_activations(X)
    a = X.float().abs().max(dim=1).values.numpy()
    assert s.dtype == np.float32
    np.testing.assert_array_equal(s, (a / np.float32(7)).astype(np.float32))
    # the largest magnitude maps to +-7, no code reaches -8
    assert np.all(np.abs(c).max(axis=1) == 7)
    assert c.min() >= -7 and c.max() <= 7


def test_ties_go_to_even():
    x = torch.tensor([[7.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5]]).to(torch.bfloat16)
    c, s = quantize_activations(x)
    assert s[0] == np.float32(1.0)
    assert c[0].tolist() == [7, 2, 4, -2, -4, 0, 0, 2]


def test_zero_token_has_unit_scale_and_zero_output():
    W = synth.weight(32, 256, std=0.02, outlier_frac=0.01, seed=63)
    d = decompose(W, 0.02)
    X = synth.activations(3, 256, seed=64)
    X[1] = 0
    c, s = quantize_activations(X)
    assert s[1] == np.float32(1.0) and not c[1].any()
    Y = linear_w4a4(X, d)
    assert np.all(Y[1] == 0.0)


def test_power_of_two_scaling():
    W = synth.weight(48, 384, std=0.02, outlier_frac=0.01, seed=65)
    d = decompose(W, 0.02)
    X = synth.activations(4, 384, seed=66, channels=2, mult=10.0)
    c1, s1 = quantize_activations(X)
    c2, s2 = quantize_activations(X * 4)           # exact in bf16
    assert np.array_equal(c1, c2) and np.array_equal(s2, s1 * 4)
    np.testing.assert_array_equal(linear_w4a4(X * 4, d), 4 * linear_w4a4(X, d))


def test_grid_activations_give_the_w4a16_result():
    # integer activations in [-7, 7] with a 7 in every token: s_x = 1 and
    # the quantization is the identity
    rng = np.random.default_rng(67)
    W = synth.weight(40, 512, std=0.02, outlier_frac=0.01, seed=68)
    d = decompose(W, 0.03)
    Xi = rng.integers(-7, 8, size=(5, 512)).astype(np.float32)
    Xi[:, 0] = 7
    X = torch.from_numpy(Xi).to(torch.bfloat16)
    c, s = quantize_activations(X)
    assert np.all(s == 1.0) and np.array_equal(c.astype(np.float32), Xi)
    np.testing.assert_allclose(linear_w4a4(X, d), linear(Xi.astype(np.float64), d),
                               rtol=1e-13, atol=1e-13)


def test_equals_w4a16_of_dequantized_activations():
    W = synth.weight(64, 1024, std=0.02, outlier_frac=0.005, seed=69)
    d = decompose(W, 0.01)
    X = synth.activations(7, 1024, seed=70, channels=4, mult=20.0)
    np.testing.assert_allclose(linear_w4a4(X, d), linear(dequantized_activations(X), d),
                               rtol=1e-11, atol=1e-12)
    rows = np.array([0, 17, 63])
    np.testing.assert_allclose(linear_w4a4(X, d, rows=rows), linear_w4a4(X, d)[:, rows],
                               rtol=0, atol=0)


@pytest.mark.parametrize("K,group", [(8, 8), (128, 128)])
def test_brute_force_tiny(K, group):
    rng = np.random.default_rng(71)
    W = (rng.standard_normal((8, K)) * 0.02).astype(np.float32)
    W[2, 3] = 0.6
    d = decompose(W, 0.25, group=group)
    X = torch.from_numpy(rng.standard_normal((3, K)).astype(np.float32)).to(torch.bfloat16)
    np.testing.assert_allclose(linear_w4a4(X, d), linear_brute(dequantized_activations(X), d),
                               rtol=1e-12, atol=1e-12)
