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
