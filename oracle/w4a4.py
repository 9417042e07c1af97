"""Oracle: the W4A4 variant of the product (weights and activations 4-bit).

Test infrastructure (see oracle/__init__.py): never imported by the product.

Passages (MosaicQuant, gist.science/paper/2606.15652): "Methodology" 3.
ZipperEngine, whose pipeline begins with a quantization stage ahead of the
dense computation, the sparse compensation and the reduction-add; and
"Experimental Results", which evaluates the method as W4A4, activations
4-bit like the weights. The pages give no activation format. The readings
taken here:

  A1 scale:   per token m, a = max_k |x[m,k]| over its bf16 values (exact in
              fp32); s_x[m] = fp32(a / 7), one IEEE fp32 division; s_x = 1
              when a = 0.
  A2 codes:   c[m,k] = clamp(rne(fp32(x[m,k] / s_x[m])), -8, 7), the division
              again one IEEE fp32 step. A float decides an integer here, so
              the oracle takes that decision in the precision the kernel uses
              (fp32); everything after it is fp64.
  P product:  Y[m,n] = s_x[m] * ( sum_g s[n,g] * sum_{k in g} (q[n,k] - z[n,g]) * c[m,k]
                                  + s_r[n] * sum_{entries e of row n} q_r[e] * c[m, col(e)] ),
              with the integer sums exact. In real arithmetic this is
              Xhat * W_hat^T with Xhat = c * s_x, the W4A16 product of the
              dequantized activations.
"""

from __future__ import annotations

import numpy as np

from .decompose import Decomposition


def _bf16_as_f32(X) -> np.ndarray:
    try:
        import torch
        if isinstance(X, torch.Tensor):
            return X.detach().to("cpu").float().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(X, dtype=np.float32)


def quantize_activations(X):
    """A1, A2 on bf16 X [M, K] (a torch bf16 tensor, or values already on the
    bf16 grid as float32). Returns (codes int8 [M, K], s_x float32 [M])."""
    Xf = _bf16_as_f32(X)
    a = np.abs(Xf).max(axis=1) if Xf.shape[1] else np.zeros(Xf.shape[0], np.float32)
    s = (a.astype(np.float32) / np.float32(7.0)).astype(np.float32)
    s = np.where(a == 0, np.float32(1.0), s).astype(np.float32)
    v = (Xf / s[:, None]).astype(np.float32)          # one fp32 division per element
    c = np.clip(np.rint(v), -8, 7).astype(np.int8)    # rint: round half to even
    return c, s


def dequantized_activations(X) -> np.ndarray:
    """Xhat = c * s_x in fp64 (exact: a 4-bit code times an fp32 scale)."""
    c, s = quantize_activations(X)
    return c.astype(np.float64) * s.astype(np.float64)[:, None]


def linear_w4a4(X, d: Decomposition, rows: np.ndarray | None = None) -> np.ndarray:
    """P: Y [M, N] in fp64 from exact integer group sums, then the scales.
    ``rows`` restricts the output to those output features."""
    c, sx = quantize_activations(X)
    if c.shape[1] != d.K:
        raise ValueError("X has the wrong number of columns")
    sel = np.arange(d.N) if rows is None else np.asarray(rows)
    M, G, g = c.shape[0], d.G, d.group
    ci = c.astype(np.int64).reshape(M, G, g)
    qz = d.q[sel].astype(np.int64).reshape(len(sel), G, g) - d.z[sel].astype(np.int64)[..., None]
    # exact integer sums per (token, row, group)
    isum = np.einsum("mgk,ngk->mng", ci, qz)
    dense = (isum.astype(np.float64) * d.s[sel].astype(np.float64)[None, :, :]).sum(axis=2)
    Y = dense
    for j, n in enumerate(sel):
        a, b = int(d.row_ptr[n]), int(d.row_ptr[n + 1])
        if b > a:
            r = (c[:, d.col[a:b]].astype(np.int64) * d.qr[a:b].astype(np.int64)[None, :]).sum(axis=1)
            Y[:, j] += float(d.sr[n]) * r.astype(np.float64)
    return Y * sx.astype(np.float64)[:, None]
