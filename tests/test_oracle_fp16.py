"""Pin the oracle's fp64 -> fp16 rounding against enumeration of every fp16.

The scales of the disaggregated form are fp16 values rounded once from fp64
(the encoding of MosaicQuant's dense 4-bit base and sparse residual this
library fixes). Brute force: the nearest finite fp16, ties to the even bit
pattern, overflow to inf at or above 65520.
"""

import numpy as np

from oracle import fp16_rne

_ALL = np.arange(0, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)  # +0 .. max finite


def _brute(x: float) -> np.float16:
    ax = abs(x)
    if ax >= 65520.0:
        return np.float16(np.inf if x > 0 else -np.inf)
    i = np.searchsorted(_ALL, ax)
    cands = [j for j in (i - 1, i) if 0 <= j < _ALL.size]
    best = min(cands, key=lambda j: (abs(_ALL[j] - ax), j & 1))
    r = np.uint16(best).view(np.float16)
    return -r if x < 0 else r


def _check(xs):
    got = fp16_rne(np.array(xs))
    for x, g in zip(xs, got):
        want = _brute(float(x))
        assert np.uint16(g.view(np.uint16)) == np.uint16(want.view(np.uint16)) or (
            g == 0 and want == 0), (x, g, want)


def test_random_normal_range():
    rng = np.random.default_rng(1)
    _check(list(rng.standard_normal(2000) * 0.05) + list(rng.standard_normal(500) * 300))


def test_midpoints_and_neighbours():
    rng = np.random.default_rng(2)
    idx = rng.integers(1, 0x7BFF, 400)
    xs = []
    for i in idx:
        lo, hi = _ALL[i], _ALL[i + 1]
        mid = (lo + hi) / 2.0
        xs += [mid, np.nextafter(mid, 0.0), np.nextafter(mid, np.inf)]
    _check(xs)


def test_subnormals_and_underflow():
    xs = [2.0 ** -24, 2.0 ** -25, 2.0 ** -25 * 1.0000001, 2.0 ** -26, 3 * 2.0 ** -25,
          6.1e-5, 6.0e-5, 1e-7, 2.0 ** -14, 2.0 ** -14 - 2.0 ** -25]
    _check(xs)


def test_overflow_boundary():
    _check([65504.0, 65519.99, 65520.0, 70000.0, -65520.0])
