"""Oracle: the product Y = X * W_hat^T in fp64.

Test infrastructure (see oracle/__init__.py): never imported by the product.

Passage: MosaicQuant, "Methodology" 3. ZipperEngine: the sparse residual is
integrated into the dense 4-bit GEMM, and its pipeline ends in a
reduction-add of the dense and sparse parts. Read plainly, the fused layer
computes Y = X * deq(Q)^T + X * R^T = X * W_hat^T, which is what both forms
here compute:

  linear        - numpy fp64 matmul with the dequantized base, then one CSR
                  pass that adds each residual entry (form 1);
  linear_brute  - an explicit triple loop over a dense W_hat (form 2, tiny
                  inputs only).
"""

from __future__ import annotations

import numpy as np

from .decompose import Decomposition


def dequant_base(d: Decomposition) -> np.ndarray:
    """deq[n][k] = (q - z) * s in fp64 (exact: at most 16 significant bits)."""
    G, g = d.G, d.group
    q = d.q.astype(np.float64).reshape(d.N, G, g)
    z = d.z.astype(np.float64)[..., None]
    s = d.s.astype(np.float64)[..., None]
    return ((q - z) * s).reshape(d.N, d.K)


def w_hat(d: Decomposition) -> np.ndarray:
    """W_hat = deq + scatter(residual) in fp64."""
    W = dequant_base(d)
    rows = np.repeat(np.arange(d.N), np.diff(d.row_ptr))
    np.add.at(W, (rows, d.col), d.residual_values())
    return W


def _as_f64(X) -> np.ndarray:
    try:
        import torch
        if isinstance(X, torch.Tensor):
            return X.detach().to("cpu").double().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(X, dtype=np.float64)


def linear(X, d: Decomposition, rows: np.ndarray | None = None) -> np.ndarray:
    """Y[M][N] = X * W_hat^T in fp64 (form 1). X is bf16 (widened exactly)
    or fp64. ``rows`` restricts the output to those output features."""
    X64 = _as_f64(X)
    if X64.shape[1] != d.K:
        raise ValueError("X has the wrong number of columns")
    sel = np.arange(d.N) if rows is None else np.asarray(rows)
    deq = dequant_base(d)[sel]
    Y = X64 @ deq.T
    vals = d.residual_values()
    for j, n in enumerate(sel):
        a, b = int(d.row_ptr[n]), int(d.row_ptr[n + 1])
        if b > a:
            Y[:, j] += X64[:, d.col[a:b]] @ vals[a:b]
    return Y


def linear_brute(X, d: Decomposition) -> np.ndarray:
    """Y[m][n] = sum_k X[m][k] * W_hat[n][k] by explicit loops (form 2)."""
    X64 = _as_f64(X)
    W = w_hat(d)
    M, K = X64.shape
    Y = np.zeros((M, d.N))
    for m in range(M):
        for n in range(d.N):
            acc = 0.0
            for k in range(K):
                acc += X64[m, k] * W[n, k]
            Y[m, n] = acc
    return Y
