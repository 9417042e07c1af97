"""Oracle: inlier-outlier disaggregation W_hat ~= Q(W_hat) + R in fp64.

Test infrastructure (see oracle/__init__.py): never imported by the product.

Passages followed (MosaicQuant, gist.science/paper/2606.15652):
  * "Methodology" 1. Inlier-Outlier Disaggregation: W_hat ~= Q(W_hat) + R,
    a dense 4-bit base that captures inliers and a sparse 4-bit residual R
    that compensates the quantization error the outliers leave; both parts
    are 4-bit.
  * "Methodology" 2. Block-Wise Residual Allocation and the abstract (OpenAlex
    record): the residual goes to the most error-critical weights.

The pages fix no encoding. The readings used here (the dense base is int4
asymmetric with group 128 along K and one fp16 scale and zero per group and
row; the residual is a per-row CSR of int4 values with one fp16 scale per
row; the residual of each row holds its k_n largest |error| entries) are the
encoding this library implements, step by step:

  D1 base:   lo = min(min v, 0), hi = max(max v, 0);
             s = fp16_rne((hi - lo) / 15)  (fp64 divide, direct fp64->fp16);
             s = 1 if hi == lo; s = 2^-24 if it rounds to 0 while hi > lo;
             an fp16 overflow is an error;
             z = clamp(rne(-lo / s), 0, 15); q = clamp(rne(v / s) + z, 0, 15);
             deq = (q - z) * s.
  D2 error:  E = v - deq.
  D3 select: k_n = floor(rho * K + 0.5) entries per row, ranked by |E|
             descending, ties to the smaller column; stored by ascending
             column; kept even when their code is 0.
  D4 resid:  a = max |E| over the selected entries; s_r = fp16_rne(a / 7),
             1 if that is 0; q_r = clamp(rne(E / s_r), -8, 7).
  D5:        W_hat = deq + scatter(q_r * s_r).

rne is round-half-to-even (numpy.rint).

Block mode ("Methodology" 2, Block-Wise Residual Allocation, with its
Hessian-guided delta score) replaces D3: W is cut into 16-row x 64-column
blocks; each block's score is its residual error weighted by the activation
sensitivity of the input channels, delta(b) = sum (E * E) * h over the block
(h = a diagonal Hessian estimate, e.g. sum over calibration tokens of x_k^2;
all ones without one), summed in fp64 row by row and column by column; the
floor(fraction * blocks + 0.5) largest scores (ties to the smaller block
index, row-block major) carry a residual on every entry. D4 then quantizes
each row's residual entries with one scale per row, as above.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def fp16_rne(x) -> np.ndarray:
    """fp64 -> fp16 with one round-to-nearest-even step (numpy's direct
    double->half conversion; pinned against enumeration of all fp16 values in
    tests/test_oracle_fp16.py)."""
    with np.errstate(over="ignore"):
        return np.asarray(x, dtype=np.float64).astype(np.float16)


def residual_count(K: int, rho: float) -> int:
    """k_n = floor(rho * K + 0.5), the same for every row."""
    return int(np.floor(float(rho) * K + 0.5))


@dataclass
class Decomposition:
    """One weight matrix in its disaggregated form.

    q   uint8   [N, K]   base codes 0..15
    s   float16 [N, G]   group scales
    z   float16 [N, G]   group zero points (integers 0..15)
    row_ptr int64 [N+1]  CSR row offsets of the residual
    col int64   [nnz]    residual columns, ascending within a row
    qr  int8    [nnz]    residual codes in [-8, 7]
    sr  float16 [N]      residual scale per row
    exact float64 [nnz]  only in the unquantized-residual test mode: the
                         residual values themselves (qr/sr unused)
    """
    N: int
    K: int
    group: int
    q: np.ndarray
    s: np.ndarray
    z: np.ndarray
    row_ptr: np.ndarray
    col: np.ndarray
    qr: np.ndarray
    sr: np.ndarray
    exact: np.ndarray | None = None

    @property
    def G(self) -> int:
        return self.K // self.group

    @property
    def nnz(self) -> int:
        return int(self.row_ptr[-1])

    def residual_values(self) -> np.ndarray:
        """fp64 value of every residual entry (q_r * s_r, or the exact one)."""
        if self.exact is not None:
            return self.exact
        rows = np.repeat(np.arange(self.N), np.diff(self.row_ptr))
        return self.qr.astype(np.float64) * self.sr.astype(np.float64)[rows]


def quantize_base(W: np.ndarray, group: int):
    """D1 for every (row, group): returns q u8 [N,K], s f16 [N,G], z f16
    [N,G] and deq f64 [N,K]."""
    W = np.asarray(W)
    if W.dtype != np.float32:
        raise TypeError("W must be float32")
    N, K = W.shape
    if K % group:
        raise ValueError("K must be a multiple of the group size")
    if not np.all(np.isfinite(W)):
        raise ValueError("W holds NaN or Inf")
    G = K // group
    v = W.astype(np.float64).reshape(N, G, group)
    lo = np.minimum(v.min(axis=2), 0.0)
    hi = np.maximum(v.max(axis=2), 0.0)
    s = fp16_rne((hi - lo) / 15.0)
    if np.any(np.isinf(s)):
        raise ValueError("a group scale overflows fp16")
    s = np.where(hi == lo, np.float16(1.0), s)
    s = np.where((s == 0) & (hi > lo), np.float16(2.0 ** -24), s)
    s64 = s.astype(np.float64)
    # z is an integer code 0..15; "+ 0.0" keeps its fp16 encoding canonical
    # (+0, not the -0 that -lo/s gives when lo = 0)
    z = np.clip(np.rint(-lo / s64), 0.0, 15.0) + 0.0
    q = np.clip(np.rint(v / s64[..., None]) + z[..., None], 0.0, 15.0)
    deq = (q - z[..., None]) * s64[..., None]
    return (q.astype(np.uint8).reshape(N, K), s.astype(np.float16),
            z.astype(np.float16), deq.reshape(N, K))


def select_residual(E: np.ndarray, k_n: int) -> np.ndarray:
    """D3: per row, the columns of the k_n largest |E| (ties to the smaller
    column), ascending. Returns int64 [N, k_n]."""
    N, K = E.shape
    if not 0 <= k_n <= K:
        raise ValueError("k_n out of range")
    order = np.argsort(-np.abs(E), axis=1, kind="stable")
    return np.sort(order[:, :k_n], axis=1)


def quantize_residual(Esel: np.ndarray):
    """D4 on the selected errors of each row (Esel f64 [N, k_n]): returns
    q_r int8 [N, k_n] and s_r f16 [N]."""
    N = Esel.shape[0]
    if Esel.shape[1] == 0:
        return np.zeros((N, 0), np.int8), np.ones(N, np.float16)
    a = np.abs(Esel).max(axis=1)
    sr = fp16_rne(a / 7.0)
    if np.any(np.isinf(sr)):
        raise ValueError("a residual scale overflows fp16")
    sr = np.where(sr == 0, np.float16(1.0), sr).astype(np.float16)
    qr = np.clip(np.rint(Esel / sr.astype(np.float64)[:, None]), -8.0, 7.0)
    return qr.astype(np.int8), sr


def decompose(W: np.ndarray, rho: float, group: int = 128,
              exact_residual: bool = False) -> Decomposition:
    """D1-D5 on a fp32 weight matrix W[N][K].

    exact_residual=True keeps the selected errors unquantized (a test mode:
    at rho = 1 the decomposition then reproduces W exactly)."""
    q, s, z, deq = quantize_base(W, group)
    N, K = q.shape
    E = W.astype(np.float64) - deq
    k_n = residual_count(K, rho)
    cols = select_residual(E, k_n)
    Esel = np.take_along_axis(E, cols, axis=1)
    row_ptr = np.arange(N + 1, dtype=np.int64) * k_n
    if exact_residual:
        return Decomposition(N, K, group, q, s, z, row_ptr, cols.reshape(-1),
                             np.zeros(N * k_n, np.int8), np.ones(N, np.float16),
                             exact=Esel.reshape(-1).copy())
    qr, sr = quantize_residual(Esel)
    return Decomposition(N, K, group, q, s, z, row_ptr, cols.reshape(-1),
                         qr.reshape(-1), sr)


BLOCK_ROWS, BLOCK_COLS = 16, 64


def blocks_selected(N: int, K: int, fraction: float) -> int:
    """floor(fraction * blocks + 0.5) with blocks = (N/16) * (K/64)."""
    return int(np.floor(float(fraction) * ((N // BLOCK_ROWS) * (K // BLOCK_COLS)) + 0.5))


def block_scores(E: np.ndarray, h=None) -> np.ndarray:
    """The delta score of every 16 x 64 block (block index rb * (K/64) + cb):
    sum over the block of (E * E) * h[k], accumulated in fp64 in row-major
    order (cumsum is a sequential sum). h: K channel weights (float32) or
    None for all ones."""
    N, K = E.shape
    nbr, nbc = N // BLOCK_ROWS, K // BLOCK_COLS
    w = np.ones(K) if h is None else np.asarray(h, np.float32).astype(np.float64)
    T = (E * E) * w[None, :]
    T = T.reshape(nbr, BLOCK_ROWS, nbc, BLOCK_COLS).transpose(0, 2, 1, 3)
    T = T.reshape(nbr * nbc, BLOCK_ROWS * BLOCK_COLS)
    if T.shape[1] == 0 or T.shape[0] == 0:
        return np.zeros(nbr * nbc)
    return np.cumsum(T, axis=1)[:, -1]


def select_blocks(score: np.ndarray, n_sel: int) -> np.ndarray:
    """The n_sel largest scores, ties to the smaller index: bool mask."""
    order = np.argsort(-score, kind="stable")
    sel = np.zeros(score.size, dtype=bool)
    sel[order[:n_sel]] = True
    return sel


def decompose_blocks(W: np.ndarray, block_fraction: float, h=None, group: int = 128,
                     exact_residual: bool = False) -> Decomposition:
    """D1, D2, block selection, D4, D5 on fp32 W[N][K] (N % 16 == 0)."""
    q, s, z, deq = quantize_base(W, group)
    N, K = q.shape
    if N % BLOCK_ROWS or K % BLOCK_COLS:
        raise ValueError("block mode needs N % 16 == 0 and K % 64 == 0")
    if not 0.0 <= block_fraction <= 1.0:
        raise ValueError("block_fraction must be in [0, 1]")
    if h is not None:
        hv = np.asarray(h, np.float32)
        if hv.shape != (K,) or not np.all(np.isfinite(hv)) or np.any(hv < 0):
            raise ValueError("channel weights must be K finite values >= 0")
    E = W.astype(np.float64) - deq
    nbr, nbc = N // BLOCK_ROWS, K // BLOCK_COLS
    sel = select_blocks(block_scores(E, h), blocks_selected(N, K, block_fraction)).reshape(nbr, nbc)
    counts = np.repeat(sel.sum(axis=1) * BLOCK_COLS, BLOCK_ROWS)
    row_ptr = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    cols, qrs, exact = [], [], []
    sr = np.ones(N, np.float16)
    for rb in range(nbr):
        cb = np.nonzero(sel[rb])[0]
        if cb.size == 0:
            continue
        c = (cb[:, None] * BLOCK_COLS + np.arange(BLOCK_COLS)[None, :]).reshape(-1)
        Esel = E[rb * BLOCK_ROWS:(rb + 1) * BLOCK_ROWS][:, c]
        cols.append(np.tile(c, BLOCK_ROWS))
        if exact_residual:
            exact.append(Esel.reshape(-1))
            continue
        qr, s_r = quantize_residual(Esel)
        qrs.append(qr.reshape(-1))
        sr[rb * BLOCK_ROWS:(rb + 1) * BLOCK_ROWS] = s_r
    col = np.concatenate(cols).astype(np.int64) if cols else np.zeros(0, np.int64)
    if exact_residual:
        ex = np.concatenate(exact) if exact else np.zeros(0)
        return Decomposition(N, K, group, q, s, z, row_ptr, col, np.zeros(col.size, np.int8),
                             np.ones(N, np.float16), exact=ex)
    qr = np.concatenate(qrs).astype(np.int8) if qrs else np.zeros(0, np.int8)
    return Decomposition(N, K, group, q, s, z, row_ptr, col, qr, sr)


def from_arrays(d: dict) -> Decomposition:
    """A Decomposition from a dict of arrays (e.g. a synthetic sweep draw)."""
    return Decomposition(int(d["N"]), int(d["K"]), int(d.get("group", 128)),
                         np.asarray(d["q"], np.uint8),
                         np.asarray(d["s"], np.float16),
                         np.asarray(d["z"], np.float16),
                         np.asarray(d["row_ptr"], np.int64),
                         np.asarray(d["col"], np.int64),
                         np.asarray(d["qr"], np.int8),
                         np.asarray(d["sr"], np.float16))
