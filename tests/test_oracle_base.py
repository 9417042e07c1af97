"""Pin the oracle's dense 4-bit base (step D1) without re-typing its formula.

MosaicQuant, "Methodology" 1.: the dense 4-bit base Q(W) captures the
inliers of every group. Pins: brute force over the 16 codes and over all fp16
scales, the half-step error bound, special groups, and a hand-derived
example (tests/golden/hand_group8.txt).
"""

import numpy as np
import pytest

from oracle import quantize_base, decompose

_FP16 = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)


def _nearest_fp16(x):
    i = np.searchsorted(_FP16, x)
    c = [j for j in (i - 1, i) if 0 <= j < _FP16.size]
    return _FP16[min(c, key=lambda j: (abs(_FP16[j] - x), j & 1))]


def _brute_group(v):
    """Choose s, z, q by search: s the fp16 nearest to the range / 15, z the
    integer code nearest to -lo/s, each q the code whose grid point is
    nearest to v (ties to an even offset from z)."""
    v = v.astype(np.float64)
    lo, hi = min(v.min(), 0.0), max(v.max(), 0.0)
    if hi == lo:
        s = 1.0
    else:
        s = _nearest_fp16((hi - lo) / 15.0)
        if s == 0.0:
            s = 2.0 ** -24
    zs = np.arange(16, dtype=np.float64)
    zd = np.abs(zs - (-lo / s))
    z = min(range(16), key=lambda c: (zd[c], c & 1))
    q = []
    for x in v:
        d = [abs(x - (c - z) * s) for c in range(16)]
        q.append(min(range(16), key=lambda c: (d[c], (c - z) & 1)))
    return s, z, np.array(q)


@pytest.mark.parametrize("seed", range(6))
def test_brute_force_random_groups(seed):
    rng = np.random.default_rng(seed)
    g = 8 if seed < 3 else 128
    W = (rng.standard_normal((8, 4 * g)) * 0.02).astype(np.float32)
    W.reshape(-1)[rng.choice(W.size, W.size // 50, replace=False)] = (
        0.2 * rng.standard_t(3, W.size // 50)).astype(np.float32)
    q, s, z, deq = quantize_base(W, g)
    for n in range(W.shape[0]):
        for j in range(W.shape[1] // g):
            v = W[n, j * g:(j + 1) * g]
            bs, bz, bq = _brute_group(v)
            assert float(s[n, j]) == bs
            assert float(z[n, j]) == bz
            np.testing.assert_array_equal(q[n, j * g:(j + 1) * g], bq)


def test_half_step_bound_unless_clamped():
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((16, 1024)) * 0.02).astype(np.float32)
    q, s, z, deq = quantize_base(W, 128)
    s64 = np.repeat(s.astype(np.float64), 128, axis=1)
    z64 = np.repeat(z.astype(np.float64), 128, axis=1)
    err = np.abs(W.astype(np.float64) - deq)
    raw = np.rint(W / s64) + z64
    unclamped = (raw >= 0) & (raw <= 15)
    assert np.all(err[unclamped] <= s64[unclamped] / 2)
    assert unclamped.mean() > 0.99


def test_zero_and_constant_groups():
    W = np.zeros((2, 256), np.float32)
    W[1, 128:] = 0.3
    q, s, z, deq = quantize_base(W, 128)
    assert s[0, 0] == 1.0 and z[0, 0] == 0 and np.all(q[0] == 0)
    assert np.all(deq[0] == 0)
    # constant positive group: range [0, 0.3], code 15 at the constant
    assert z[1, 1] == 0 and np.all(q[1, 128:] == 15)
    assert np.allclose(deq[1, 128:], 0.3, atol=float(s[1, 1]) / 2)


def test_single_outlier_is_an_endpoint():
    rng = np.random.default_rng(3)
    v = (rng.standard_normal(128) * 0.01).astype(np.float32)
    v[37] = 1.0
    q, s, z, deq = quantize_base(v.reshape(1, 128), 128)
    assert q[0, 37] == 15
    assert abs(deq[0, 37] - 1.0) <= float(s[0, 0]) / 2


def test_tiny_range_scale_floor():
    W = np.zeros((1, 128), np.float32)
    W[0, 0] = np.float32(1e-9)      # (hi-lo)/15 rounds to fp16 zero
    q, s, z, deq = quantize_base(W, 128)
    assert float(s[0, 0]) == 2.0 ** -24


def test_overflow_and_nonfinite_rejected():
    W = np.zeros((1, 128), np.float32)
    W[0, 0] = 1e6
    with pytest.raises(ValueError):
        quantize_base(W, 128)
    W[0, 0] = np.nan
    with pytest.raises(ValueError):
        quantize_base(W, 128)


def test_hand_derived_example(golden):
    f = golden("hand_group8.txt")
    v = np.array([float(x) for x in f["v"]], np.float32).reshape(1, -1)
    d = decompose(v, float(f["rho"][0]), group=int(f["group"][0]))
    np.testing.assert_array_equal(d.q[0], [int(x) for x in f["q"]])
    assert d.s.view(np.uint16)[0, 0] == int(f["s_bits"][0], 16)
    assert d.z.view(np.uint16)[0, 0] == int(f["z_bits"][0], 16)


def test_zero_point_encoding_is_canonical():
    W = np.abs(np.random.default_rng(4).standard_normal((1, 128))).astype(np.float32)
    q, s, z, deq = quantize_base(W, 128)
    assert z.view(np.uint16)[0, 0] == 0x0000      # +0, never -0
