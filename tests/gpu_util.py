"""Helpers for the GPU parity tests: compare a library output with the oracle."""

import numpy as np
import torch

import oracle
from oracle.tolerance import parity_report


def oracle_check(Y: torch.Tensor, X: torch.Tensor, d):
    """Parity of a bf16 GPU output Y [M, d.N] against the fp64 oracle (the
    normalized and relative bounds of oracle/tolerance.py)."""
    X64 = X.detach().cpu().double().numpy()
    Y64 = oracle.linear(X64, d)
    wn = np.linalg.norm(oracle.w_hat(d), axis=1)
    Yg = Y.detach().float().cpu().double().numpy()
    return parity_report(Yg, Y64, X64, wn)


def oracle_check_w4a4(Y: torch.Tensor, X: torch.Tensor, d, rows=None):
    """Parity of a bf16 W4A4 output Y against the fp64 W4A4 oracle; the
    normalized bound uses the norms of the dequantized activations, the
    input the W4A4 product is defined on. ``rows`` restricts both sides."""
    from oracle.w4a4 import linear_w4a4, dequantized_activations
    Y64 = linear_w4a4(X, d, rows=rows)
    Xh = dequantized_activations(X)
    wh = oracle.w_hat(d)
    wn = np.linalg.norm(wh if rows is None else wh[np.asarray(rows)], axis=1)
    Yg = Y.detach().float().cpu().double().numpy()
    if rows is not None:
        Yg = Yg[:, np.asarray(rows)]
    return parity_report(Yg, Y64, Xh, wn)
