"""Seeded synthetic inputs for the fused W4 + sparse-residual linear.

This module is shared by the CUDA path's tests/bench and by the CPU oracle's
tests. It holds random draws and their shaping only: no quantization, no
packing and no product arithmetic of the method lives here.

The pages measure on LLaMA3 / Qwen3 layers (MosaicQuant, "Experimental
Results"); no model weights exist here, so these generators stand in for
those layers with the shapes and outlier structure of the named workloads.

Draw order inside one generator call is fixed: W values, outlier mask,
Student-t outlier values (weights); X values, then outlier channel picks
(activations).
"""

from __future__ import annotations

import numpy as np

GROUP = 128

# Named workloads. Shapes are (N, K): N output features (rows of W), K inputs.
WORKLOADS = {
    # 1 token, one 512x512 layer, 1 % of weights replaced by 0.2 * t(3).
    "tiny": dict(
        M=1, shapes=[(512, 512)], w_std=0.02, w_outlier_frac=0.01,
        w_outlier_cols=0, x_channels=0, x_mult=1.0, rho=0.01),
    # 7B-shaped decode: q/k/v/o, gate/up, down at one token.
    "7b_decode": dict(
        M=1, shapes=[(4096, 4096), (11008, 4096), (4096, 11008)], w_std=0.02,
        w_outlier_frac=0.005, w_outlier_cols=0, x_channels=4, x_mult=20.0,
        rho=0.005),
    # 70B MLP batched decode: 32 whole outlier input columns plus a scattered
    # remainder, 1 % outliers in total.
    "70b_mlp": dict(
        M=16, shapes=[(28672, 8192)], w_std=0.015, w_outlier_frac=0.01,
        w_outlier_cols=32, x_channels=0, x_mult=1.0, rho=0.01),
    # Prefill: 2048 tokens through one 14336x4096 projection.
    "prefill": dict(
        M=2048, shapes=[(14336, 4096)], w_std=0.02, w_outlier_frac=0.005,
        w_outlier_cols=0, x_channels=8, x_mult=30.0, rho=0.005),
}

# Llama-7B block linears used by the density sweep.
SWEEP_SHAPES = {"qkvo": (4096, 4096), "gateup": (11008, 4096), "down": (4096, 11008)}
SWEEP_M = (1, 8, 64, 512, 4096)
SWEEP_RHO = (0.0, 0.0025, 0.01, 0.04)


def weight(N: int, K: int, *, std: float, outlier_frac: float, seed: int,
           outlier_scale: float = 0.2, outlier_cols: int = 0,
           rows: np.ndarray | None = None) -> np.ndarray:
    """fp32 W[N][K] ~ N(0, std) with round(outlier_frac*N*K) entries replaced
    by outlier_scale * t(3).

    With outlier_cols > 0, that many seeded input columns are outliers in
    every row and the rest of the outlier budget is scattered uniformly over
    the other columns. ``rows`` (optional) returns only those rows of the same
    matrix, for samples of matrices too large to hold.
    """
    rng = np.random.default_rng(seed)
    W = rng.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(std)
    n_out = int(round(outlier_frac * N * K))
    if outlier_cols > 0:
        cols = np.sort(rng.choice(K, outlier_cols, replace=False))
        n_col = N * outlier_cols
        n_rest = max(n_out - n_col, 0)
        other = np.setdiff1d(np.arange(K), cols)
        flat = rng.choice(N * other.size, n_rest, replace=False)
        t_col = rng.standard_t(3, size=n_col) * outlier_scale
        t_rest = rng.standard_t(3, size=n_rest) * outlier_scale
        W[:, cols] = t_col.reshape(N, outlier_cols).astype(np.float32)
        r, c = np.divmod(flat, other.size)
        W[r, other[c]] = t_rest.astype(np.float32)
    else:
        flat = rng.choice(N * K, n_out, replace=False)
        t = rng.standard_t(3, size=n_out) * outlier_scale
        W.reshape(-1)[flat] = t.astype(np.float32)
    if rows is not None:
        return np.ascontiguousarray(W[np.asarray(rows)])
    return W


def activations(M: int, K: int, *, seed: int, channels: int = 0,
                mult: float = 1.0, channel_seed: int | None = None):
    """bf16 X[M][K] ~ N(0, 1) with ``channels`` seeded input channels scaled
    by ``mult``. Returned as a CPU torch.bfloat16 tensor (RNE from fp32).

    The outlier channels are drawn after X from the same generator, unless
    ``channel_seed`` is given: then they come from a generator of their own,
    so that several draws of X (calibration and evaluation tokens of one
    layer) share the same outlier channels."""
    import torch
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((M, K), dtype=np.float32)
    if channels > 0:
        crng = rng if channel_seed is None else np.random.default_rng(channel_seed)
        ch = crng.choice(K, channels, replace=False)
        X[:, ch] *= np.float32(mult)
    return torch.from_numpy(X).to(torch.bfloat16)


def workload_inputs(name: str, shape_index: int = 0, *, rows=None,
                    M: int | None = None):
    """(W fp32, X bf16, rho) for one shape of a named workload.

    Seeds: W uses 1000 * (shape_index + 1); X uses 7 + shape_index.
    """
    cfg = WORKLOADS[name]
    N, K = cfg["shapes"][shape_index]
    W = weight(N, K, std=cfg["w_std"], outlier_frac=cfg["w_outlier_frac"],
               outlier_cols=cfg["w_outlier_cols"], seed=1000 * (shape_index + 1),
               rows=rows)
    X = activations(cfg["M"] if M is None else M, K, seed=7 + shape_index,
                    channels=cfg["x_channels"], mult=cfg["x_mult"])
    return W, X, cfg["rho"]


def sweep_decomposition(N: int, K: int, k_n: int, *, seed: int,
                        cluster_frac: float = 0.7, n_channels: int = 8):
    """A synthetic decomposition for the density sweep, drawn directly.

    Base codes are uniform in 0..15 with one scale fp16(0.02*6/15) and zero
    point 8 everywhere. Each row gets k_n residual entries: round(0.7*k_n) of
    them uniform without replacement in the 128-wide K-groups that hold
    ``n_channels`` seeded channels, the rest uniform over the other columns.
    Residual codes are uniform in [-8, 7] without 0; one scale fp16(0.004).

    Returns a dict of numpy arrays: q u8 [N,K], s f16 [N,G], z f16 [N,G],
    row_ptr i64 [N+1], col i64 [nnz], qr i8 [nnz], sr f16 [N].
    """
    rng = np.random.default_rng(seed)
    G = K // GROUP
    q = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    s = np.full((N, G), np.float16(0.02 * 6 / 15), dtype=np.float16)
    z = np.full((N, G), np.float16(8.0), dtype=np.float16)
    channels = rng.choice(K, n_channels, replace=False)
    groups = np.unique(channels // GROUP)
    cl_cols = (groups[:, None] * GROUP + np.arange(GROUP)[None, :]).reshape(-1)
    other = np.setdiff1d(np.arange(K), cl_cols)
    n_cl = min(int(round(cluster_frac * k_n)), cl_cols.size)
    if other.size == 0:                 # the clustered groups cover all of K
        n_cl = k_n
    n_ot = k_n - n_cl
    cols = np.empty((N, k_n), dtype=np.int64)
    for n in range(N):
        a = rng.choice(cl_cols, n_cl, replace=False)
        b = rng.choice(other, n_ot, replace=False) if n_ot else other[:0]
        cols[n] = np.sort(np.concatenate([a, b]))
    vals = rng.integers(-8, 7, size=(N, k_n), dtype=np.int8)
    vals[vals >= 0] += 1                       # uniform over [-8,7] \ {0}
    row_ptr = np.arange(N + 1, dtype=np.int64) * k_n
    sr = np.full(N, np.float16(0.004), dtype=np.float16)
    return dict(N=N, K=K, group=GROUP, q=q, s=s, z=z, row_ptr=row_ptr,
                col=cols.reshape(-1), qr=vals.reshape(-1), sr=sr,
                clustered_frac=(n_cl / k_n) if k_n else 0.0)
