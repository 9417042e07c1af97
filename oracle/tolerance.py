"""Oracle: parity metrics for a bf16 output against the fp64 product.

Test infrastructure (see oracle/__init__.py).

Two bounds accept an output y against the fp64 value y64:
  T1 normalized error  (|y - y64| - ulp(y64) / 2) / (||x_m|| * ||w_hat_n||) <= 2e-3
  T2 relative error    |y - y64| / |y64| <= 1e-2 wherever |y64| > 1e-3

Reading of T1: the outputs are bf16, whose unit roundoff is 2^-8 (3.9e-3)
relative. Rounding even the exact y64 to bf16 can exceed 2e-3 * ||x|| * ||w||
whenever |y64| is more than about half of ||x|| * ||w|| (x and the weight row
nearly parallel), so the normalized bound is applied to the error in excess
of half a bf16 ulp at y64: the most that rounding y64 to the nearest point of
the output grid can add. T2 needs no such allowance (1e-2 is above the bf16
roundoff). The report also gives t1_raw, the normalized error with no
allowance.
"""

from __future__ import annotations

import numpy as np

T1_MAX = 2e-3
T2_MAX = 1e-2
T2_FLOOR = 1e-3


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 grid at |y| (8 significant bits; normal range)."""
    a = np.abs(np.asarray(y, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126.0)
    return np.where(a > 0, np.exp2(e - 7.0), np.exp2(-133.0))


def parity_report(Y, Y64: np.ndarray, X64: np.ndarray,
                  w_rows_norm: np.ndarray) -> dict:
    """Y (any float array, e.g. bf16 widened), Y64 fp64 [M,N], X64 [M,K],
    w_rows_norm [N] = ||w_hat_n||. Returns the worst T1/T2 and pass flags."""
    Y = np.asarray(Y, dtype=np.float64)
    diff = np.abs(Y - Y64)
    xn = np.linalg.norm(X64, axis=1)[:, None]
    denom = xn * np.asarray(w_rows_norm, np.float64)[None, :]
    excess = np.maximum(diff - 0.5 * bf16_ulp(Y64), 0.0)
    t1 = np.where(denom > 0, excess / np.where(denom > 0, denom, 1.0), excess)
    t1_raw = np.where(denom > 0, diff / np.where(denom > 0, denom, 1.0), diff)
    big = np.abs(Y64) > T2_FLOOR
    t2 = np.where(big, diff / np.where(big, np.abs(Y64), 1.0), 0.0)
    finite = bool(np.all(np.isfinite(Y)))
    t1max = float(t1.max()) if t1.size else 0.0
    t2max = float(t2.max()) if t2.size else 0.0
    return dict(t1=t1max, t1_raw=float(t1_raw.max()) if t1_raw.size else 0.0, t2=t2max,
                finite=finite, n_t2_fail=int((t2 > T2_MAX).sum()),
                ok=finite and t1max <= T1_MAX and t2max <= T2_MAX)
