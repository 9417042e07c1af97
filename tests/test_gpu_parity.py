"""GPU parity: the CUDA path against the fp64 oracle on the same seeded
inputs, through the C ABI. Bounds (oracle/tolerance.py): normalized error
<= 2e-3 and relative error <= 1e-2 where |y| > 1e-3; packed bytes bit-exact.

MosaicQuant "Methodology" 1. (W ~= Q(W) + R, both 4-bit) and 3. (the fused
dense + sparse pass ending in one reduction-add)."""

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_w4_b200 import synth
from gpu_util import oracle_check

pytestmark = pytest.mark.gpu


def _run(mq, W, X, rho, path="auto"):
    w = mq.Weight.pack(W, rho)
    Y = w.linear(X.cuda(), path=path)
    torch.cuda.synchronize()
    assert w.device_error() == 0
    return w, Y


def _bytes_equal(got, want):
    for k in ("qweight", "sz", "row_ptr", "col", "val", "rscale"):
        a, b = np.asarray(got[k]), np.ascontiguousarray(want[k])
        assert a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8)), k


def test_tiny_workload(mq, cuda):
    W, X, rho = synth.workload_inputs("tiny")
    w, Y = _run(mq, W, X, rho)
    d = oracle.decompose(W, rho)
    _bytes_equal(w.export(), oracle.pack(d))
    r = oracle_check(Y, X, d)
    assert r["ok"], r


@pytest.mark.parametrize("shape", [0, 1, 2])
def test_7b_decode_workload(mq, cuda, shape):
    W, X, rho = synth.workload_inputs("7b_decode", shape)
    w, Y = _run(mq, W, X, rho)
    d = oracle.decompose(W, rho)
    _bytes_equal(w.export(), oracle.pack(d))
    r = oracle_check(Y, X, d)
    assert r["ok"], r


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 12, 16])
def test_decode_token_counts_ragged_rows(mq, cuda, M):
    W = synth.weight(200, 1024, std=0.02, outlier_frac=0.01, seed=M)
    X = synth.activations(M, 1024, seed=100 + M, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, 0.02, path="decode")
    r = oracle_check(Y, X, oracle.decompose(W, 0.02))
    assert r["ok"], r


@pytest.mark.parametrize("M", [17, 40, 129])
def test_prefill_token_counts(mq, cuda, M):
    W = synth.weight(136, 512, std=0.02, outlier_frac=0.01, seed=M)
    X = synth.activations(M, 512, seed=200 + M, channels=8, mult=30.0)
    w, Y = _run(mq, W, X, 0.01, path="prefill")
    r = oracle_check(Y, X, oracle.decompose(W, 0.01))
    assert r["ok"], r


@pytest.mark.parametrize("path", ["decode", "prefill", "unfused"])
@pytest.mark.parametrize("M", [1, 16])
def test_every_path_small(mq, cuda, path, M):
    W = synth.weight(264, 896, std=0.02, outlier_frac=0.01, seed=3)
    X = synth.activations(M, 896, seed=4, channels=4, mult=20.0)
    if path == "unfused":
        w = mq.Weight.pack(W, 0.01)
        Y = w.linear_unfused(X.cuda())
        torch.cuda.synchronize()
    else:
        w, Y = _run(mq, W, X, 0.01, path=path)
    r = oracle_check(Y, X, oracle.decompose(W, 0.01))
    assert r["ok"], (path, r)


@pytest.mark.parametrize("M", [1, 8, 40])
def test_unfused_matches_fused(mq, cuda, M):
    W = synth.weight(300, 1024, std=0.02, outlier_frac=0.01, seed=M)
    X = synth.activations(M, 1024, seed=9, channels=4, mult=20.0).cuda()
    w = mq.Weight.pack(W, 0.03)
    Yf = w.linear(X)
    Yu = w.linear_unfused(X)
    torch.cuda.synchronize()
    r = oracle_check(Yu, X.cpu(), oracle.decompose(W, 0.03))
    assert r["ok"], r
    # both round an fp32 result once; they may differ by one bf16 ulp
    diff = (Yf.float() - Yu.float()).abs()
    assert float((diff / Yf.float().abs().clamp_min(1e-3)).max()) < 2 ** -7


@pytest.mark.parametrize("rho", [0.0, 0.04])
def test_density_zero_and_dense_residual(mq, cuda, rho):
    W = synth.weight(128, 4096, std=0.02, outlier_frac=0.005, seed=5)
    X = synth.activations(8, 4096, seed=6, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, rho)
    r = oracle_check(Y, X, oracle.decompose(W, rho))
    assert r["ok"], r


def test_single_group_and_tiny_n(mq, cuda):
    W = synth.weight(8, 128, std=0.02, outlier_frac=0.02, seed=7)
    X = synth.activations(3, 128, seed=8)
    w, Y = _run(mq, W, X, 0.05)
    r = oracle_check(Y, X, oracle.decompose(W, 0.05))
    assert r["ok"], r


@pytest.mark.parametrize("M", [1, 8])
def test_sweep_decomposition_dense_clustered(mq, cuda, M):
    dd = synth.sweep_decomposition(256, 4096, 164, seed=11)
    w = mq.Weight.pack_decomposed(dd)
    X = synth.activations(M, 4096, seed=12)
    Y = w.linear(X.cuda())
    torch.cuda.synchronize()
    d = oracle.from_arrays(dd)
    _bytes_equal(w.export(), oracle.pack(d))
    r = oracle_check(Y, X, d)
    assert r["ok"], r


def test_argument_errors(mq, cuda):
    W = synth.weight(16, 128, std=0.02, outlier_frac=0.0, seed=1)
    w = mq.Weight.pack(W, 0.01)
    X = torch.zeros((2, 128), dtype=torch.bfloat16, device=cuda)
    Y = torch.zeros((2, 16), dtype=torch.bfloat16, device=cuda)
    w.linear_raw(X.data_ptr(), 0, Y.data_ptr())                      # M = 0: no-op
    with pytest.raises(mq.MQError) as e:
        w.linear_raw(X.data_ptr() + 2, 2, Y.data_ptr())              # misaligned X
    assert e.value.status == mq.INVALID_ARG
    with pytest.raises(mq.MQError) as e:
        w.linear_raw(X.data_ptr(), -1, Y.data_ptr())
    assert e.value.status == mq.INVALID_ARG
    with pytest.raises(mq.MQError):
        w.linear_raw(0, 2, Y.data_ptr())
    small = torch.zeros(4, dtype=torch.float32, device=cuda)
    with pytest.raises(mq.MQError) as e:
        w.linear_unfused(X, Y, small)                                # workspace too small
    assert e.value.status == mq.INVALID_ARG


def test_70b_mlp_full_size_sampled_rows(mq, cuda):
    cfg = synth.WORKLOADS["70b_mlp"]
    N, K = cfg["shapes"][0]
    W, X, rho = synth.workload_inputs("70b_mlp")
    w, Y = _run(mq, W, X, rho)
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(N - 24, N),
                                     np.random.default_rng(0).choice(N, 64, replace=False)]))
    d = oracle.decompose(np.ascontiguousarray(W[rows]), rho)
    ex = w.export()
    want = oracle.pack(d)
    assert np.array_equal(ex["qweight"][rows], want["qweight"])
    assert np.array_equal(ex["sz"][rows], want["sz"])
    assert np.array_equal(ex["rscale"][rows], want["rscale"])
    r = oracle_check(Y[:, rows], X, d)
    assert r["ok"], r


def test_prefill_full_size_sampled_rows(mq, cuda):
    cfg = synth.WORKLOADS["prefill"]
    N, K = cfg["shapes"][0]
    W, X, rho = synth.workload_inputs("prefill")
    w, Y = _run(mq, W, X, rho)
    rows = np.unique(np.concatenate([np.arange(0, 32), np.arange(N - 16, N),
                                     np.random.default_rng(1).choice(N, 48, replace=False)]))
    d = oracle.decompose(np.ascontiguousarray(W[rows]), rho)
    r = oracle_check(Y[:, rows], X, d)
    assert r["ok"], r


@pytest.mark.parametrize("N,K,M,rho", [
    (200, 128, 130, 0.02),      # one group, ragged rows and tokens
    (136, 11008, 40, 0.005),    # 86 groups (padded scale rows), ragged rows
    (300, 4096, 256, 0.01),     # two token tiles, three row tiles
    (128, 512, 17, 0.0),        # no residual
    (130, 32768, 20, 0.002),    # longest K: scale/zero words read from global memory
])
def test_prefill_kernel_shapes(mq, cuda, N, K, M, rho):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=N + K)
    X = synth.activations(M, K, seed=M, channels=8, mult=30.0)
    w, Y = _run(mq, W, X, rho, path="prefill")
    r = oracle_check(Y, X, oracle.decompose(W, rho))
    assert r["ok"], r


def test_prefill_kernel_dense_residual(mq, cuda):
    dd = synth.sweep_decomposition(256, 4096, 164, seed=21)
    w = mq.Weight.pack_decomposed(dd)
    X = synth.activations(200, 4096, seed=22)
    Y = w.linear(X.cuda(), path="prefill")
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check(Y, X, oracle.from_arrays(dd))
    assert r["ok"], r


def _row_subset(dd: dict, rows: np.ndarray) -> dict:
    """The decomposition restricted to the given rows (arrays re-indexed)."""
    rp = np.asarray(dd["row_ptr"], np.int64)
    idx = np.concatenate([np.arange(rp[r], rp[r + 1]) for r in rows]) if len(rows) else np.zeros(0, np.int64)
    counts = rp[rows + 1] - rp[rows]
    return dict(N=len(rows), K=dd["K"], q=dd["q"][rows], s=dd["s"][rows], z=dd["z"][rows],
                row_ptr=np.concatenate([[0], np.cumsum(counts)]).astype(np.int64),
                col=np.asarray(dd["col"])[idx], qr=np.asarray(dd["qr"])[idx], sr=dd["sr"][rows])


@pytest.mark.parametrize("rho", synth.SWEEP_RHO)
@pytest.mark.parametrize("shape", sorted(synth.SWEEP_SHAPES))
def test_sweep_grid(mq, cuda, shape, rho):
    """The density sweep: Llama-7B block linears at every M of the sweep
    (decode and prefill kernels) and every density, on clustered synthetic
    decompositions; packed rows byte-exact and outputs within the bounds on
    48 sampled rows (first, last and random)."""
    N, K = synth.SWEEP_SHAPES[shape]
    k_n = int(np.floor(rho * K + 0.5))
    dd = synth.sweep_decomposition(N, K, k_n, seed=N + K + k_n)
    w = mq.Weight.pack_decomposed(dd)
    rows = np.unique(np.concatenate([np.arange(0, 16), np.arange(N - 16, N),
                                     np.random.default_rng(k_n).choice(N, 16, replace=False)]))
    sub = _row_subset(dd, rows)
    d = oracle.from_arrays(sub)
    ex, want = w.export(), oracle.pack(d)
    for key in ("qweight", "sz", "rscale"):
        assert np.array_equal(ex[key][rows], want[key]), key
    for M in synth.SWEEP_M:
        X = synth.activations(M, K, seed=M + k_n)
        Y = w.linear(X.cuda())
        torch.cuda.synchronize()
        assert w.device_error() == 0
        r = oracle_check(Y[:, rows], X, d)
        assert r["ok"], (M, r)


@pytest.mark.parametrize("M", [1, 16, 300])
def test_block_mode_parity(mq, cuda, M):
    # "Methodology" 2: the block-allocated residual through both kernels
    W = synth.weight(512, 4096, std=0.02, outlier_frac=0.005, seed=41)
    Xc = synth.activations(64, 4096, seed=42, channels=4, mult=20.0).double().numpy()
    h = (Xc * Xc).sum(0).astype(np.float32)
    w = mq.Weight.pack(W, block_fraction=0.1, channel_weight=h)
    d = oracle.decompose_blocks(W, 0.1, h)
    _bytes_equal(w.export(), oracle.pack(d))
    X = synth.activations(M, 4096, seed=M, channels=8, mult=30.0)
    Y = w.linear(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check(Y, X, d)
    assert r["ok"], r
    Yu = w.linear_unfused(X.cuda())
    torch.cuda.synchronize()
    r = oracle_check(Yu, X, d)
    assert r["ok"], r


@pytest.mark.parametrize("N,K,M", [(4096, 4096, 1), (4096, 4096, 8), (2048, 11008, 3)])
def test_block_tiles_decode(mq, cuda, N, K, M):
    # a block-allocated residual held as block tiles (byte-exact with the
    # oracle's layout) and run as tensor-core passes by the streaming decode
    # kernel, several tiles per CTA
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=N + M)
    w = mq.Weight.pack(W, block_fraction=0.1)
    d = oracle.decompose_blocks(W, 0.1)
    want = oracle.pack_blocks(d)
    got = w.export_blocks()
    for k in ("blk_ptr", "blk_col", "blk_q"):
        assert np.array_equal(np.asarray(got[k]).view(np.uint8), np.asarray(want[k]).view(np.uint8)), k
    X = synth.activations(M, K, seed=50 + M, channels=4, mult=20.0)
    Y = w.linear(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check(Y, X, d)
    assert r["ok"], r


def test_block_tiles_absent_for_row_residuals(mq, cuda):
    w = mq.Weight.pack(synth.weight(64, 256, std=0.02, outlier_frac=0.005, seed=1), 0.05)
    with pytest.raises(mq.MQError) as e:
        w.export_blocks()
    assert e.value.status == mq.UNSUPPORTED


def test_block_mode_long_rows(mq, cuda):
    # 10 % of the 16 x 64 blocks of a 1024 x 11008 projection carry a residual
    N, K = 1024, 11008
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=43)
    w = mq.Weight.pack(W, block_fraction=0.1)
    d = oracle.decompose_blocks(W, 0.1)
    _bytes_equal(w.export(), oracle.pack(d))
    X = synth.activations(64, K, seed=44)
    for M in (1, 64):
        Y = w.linear(X[:M].cuda())
        torch.cuda.synchronize()
        assert w.device_error() == 0
        r = oracle_check(Y, X[:M], d)
        assert r["ok"], (M, r)


@pytest.mark.parametrize("M", [1, 5, 16])
@pytest.mark.parametrize("mode", ["rows", "blocks"])
def test_long_residual_rows(mq, cuda, M, mode):
    # Residual rows far longer than a tile's shared-memory slice: the decode
    # walk reads them from global memory; M = 16 at K = 8192 also splits K
    # over a cluster, so each rank walks only its column range.
    N, K = 128, 8192
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=47)
    if mode == "rows":
        w = mq.Weight.pack(W, 0.3)
        d = oracle.decompose(W, 0.3)
    else:
        w = mq.Weight.pack(W, block_fraction=0.6)
        d = oracle.decompose_blocks(W, 0.6)
    _bytes_equal(w.export(), oracle.pack(d))
    X = synth.activations(M, K, seed=48 + M, channels=4, mult=20.0)
    for path in ("auto", "unfused"):
        Y = w.linear(X.cuda()) if path == "auto" else w.linear_unfused(X.cuda())
        torch.cuda.synchronize()
        assert w.device_error() == 0
        r = oracle_check(Y, X, d)
        assert r["ok"], (path, r)


@pytest.mark.parametrize("M", [9, 13, 16])
def test_wide_decode_ragged(mq, cuda, M):
    # 9..16 tokens on a layer tall enough for the wide decode kernel (149
    # 128-row blocks, the last one ragged) with a last 256-column stage that
    # holds one group (K = 384), fused and unfused
    W = synth.weight(19000, 384, std=0.02, outlier_frac=0.01, seed=53)
    X = synth.activations(M, 384, seed=54 + M, channels=2, mult=20.0)
    w, Y = _run(mq, W, X, 0.05)
    d = oracle.decompose(W, 0.05)
    r = oracle_check(Y, X, d)
    assert r["ok"], r
    Yu = w.linear_unfused(X.cuda())
    torch.cuda.synchronize()
    r = oracle_check(Yu, X, d)
    assert r["ok"], r


@pytest.mark.parametrize("M", [1, 5, 16])
def test_linear_prefetch_matches_linear(mq, cuda, M):
    # bringing the next layer's weight into L2 changes nothing in the result
    W1 = synth.weight(384, 4096, std=0.02, outlier_frac=0.005, seed=95)
    W2 = synth.weight(1024, 384, std=0.02, outlier_frac=0.005, seed=96)
    w1, w2 = mq.Weight.pack(W1, 0.01), mq.Weight.pack(W2, 0.01)
    X = synth.activations(M, 4096, seed=97).cuda()
    Y0 = w1.linear(X)
    Y1 = torch.empty_like(Y0)
    w1.linear_raw(X.data_ptr(), M, Y1.data_ptr(), next_weight=w2)
    torch.cuda.synchronize()
    assert torch.equal(Y0, Y1)
    assert w1.device_error() == 0


@pytest.mark.parametrize("M", [1, 8, 16])
def test_longest_k_decode(mq, cuda, M):
    # K = 65536 (the u16 column limit): at 16 tokens X's slice no longer fits
    # the narrow kernel even split over 8 CTAs, and the wide kernel takes it
    N, K = 64, 65536
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=98)
    X = synth.activations(M, K, seed=99, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, 0.002)
    r = oracle_check(Y, X, oracle.decompose(W, 0.002))
    assert r["ok"], r


@pytest.mark.parametrize("M,K,rho", [(9, 2176, 0.01), (16, 2176, 0.04), (16, 1024, 0.01), (12, 640, 0.0)])
def test_tall_layer_decode(mq, cuda, M, K, rho):
    # 9-16 tokens on a layer tall enough for the wide kernel (19000 rows: the
    # last 16-row tile ragged); K = 2176 ends in a half stage
    N = 19000
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=M + K)
    X = synth.activations(M, K, seed=31 + M, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, rho)
    d = oracle.decompose(W, rho)
    r = oracle_check(Y, X, d)
    assert r["ok"], r
    Yu = w.linear_unfused(X.cuda())      # the split execution's dense half without residual
    torch.cuda.synchronize()
    ru = oracle_check(Yu, X, d)
    assert ru["ok"], ru


@pytest.mark.parametrize("rho", [0.01, 0.04])
def test_tall_kernel_sampled_rows(mq, cuda, rho):
    # 2-16 tokens on a layer tall enough for the tall-layer kernel (19000
    # rows, the last 16-row tile ragged) whose X (K = 8192) does not fit the
    # streaming kernel's shared memory; at rho = 4 % a CTA's residual lists
    # exceed their budget and the wide and register kernels take the call.
    # Fused and unfused, checked on sampled rows.
    N, K = 19000, 8192
    W = synth.weight(N, K, std=0.015, outlier_frac=0.01, outlier_cols=32, seed=71)
    w = mq.Weight.pack(W, rho)
    rows = np.unique(np.concatenate([np.arange(0, 40), np.arange(N - 24, N),
                                     np.random.default_rng(1).choice(N, 64, replace=False)]))
    d = oracle.decompose(np.ascontiguousarray(W[rows]), rho)
    del W
    for M in (2, 5, 8, 12, 16):
        X = synth.activations(M, K, seed=72 + M, channels=4, mult=20.0)
        Y = w.linear(X.cuda())
        Yu = w.linear_unfused(X.cuda())
        torch.cuda.synchronize()
        assert w.device_error() == 0
        r = oracle_check(Y[:, rows], X, d)
        assert r["ok"], (M, r)
        r = oracle_check(Yu[:, rows], X, d)
        assert r["ok"], (M, "unfused", r)


@pytest.mark.parametrize("M", [17, 40, 64])
def test_decode_token_slices(mq, cuda, M):
    # the decode path past 16 tokens: 16-token slices of X and Y, each a
    # decode launch (ragged rows, a last slice shorter than 16)
    W = synth.weight(1000, 1024, std=0.02, outlier_frac=0.01, seed=M + 5)
    X = synth.activations(M, 1024, seed=M + 6, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, 0.02, path="decode")
    r = oracle_check(Y, X, oracle.decompose(W, 0.02))
    assert r["ok"], r


@pytest.mark.parametrize("M", [17, 40, 64])
def test_auto_token_counts_17_to_64(mq, cuda, M):
    # mq_linear at 17-64 tokens: decode slices on a short layer (the
    # estimate favours them), the prefill kernel on an 11008 x 4096 layer at
    # 32 or more tokens (it favours prefill there), checked on sampled rows
    W = synth.weight(136, 512, std=0.02, outlier_frac=0.01, seed=M + 40)
    X = synth.activations(M, 512, seed=M + 41, channels=8, mult=30.0)
    w, Y = _run(mq, W, X, 0.01)
    r = oracle_check(Y, X, oracle.decompose(W, 0.01))
    assert r["ok"], r
    if M >= 32:
        N, K = 11008, 4096
        W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=M + 42)
        X = synth.activations(M, K, seed=M + 43, channels=4, mult=20.0)
        w, Y = _run(mq, W, X, 0.005)
        rows = np.unique(np.concatenate([np.arange(0, 24), np.arange(N - 24, N),
                                         np.random.default_rng(M).choice(N, 48, replace=False)]))
        r = oracle_check(Y[:, rows], X, oracle.decompose(np.ascontiguousarray(W[rows]), 0.005))
        assert r["ok"], r


@pytest.mark.parametrize("M", [17, 40])
def test_longest_k_prefill(mq, cuda, M):
    # K = 65536 at more than 16 tokens: the prefill kernel reads 512 scale
    # words per row (beyond the 256 of its first design)
    N, K = 160, 65536
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=96)
    X = synth.activations(M, K, seed=97, channels=4, mult=20.0)
    w, Y = _run(mq, W, X, 0.002, path="prefill")
    r = oracle_check(Y, X, oracle.decompose(W, 0.002))
    assert r["ok"], r


def test_bounded_wait_gives_up(mq, cuda):
    # a wait on a barrier phase nobody completes ends after its limit with
    # its code in the error word, and the wait after it returns at once
    assert mq.selftest_bounded_wait(1 << 20) == [1, 0, 0, 2]


@pytest.mark.parametrize("N,K,M,path", [
    (200, 384, 1, "auto"),        # narrow decode, ragged tile
    (200, 384, 13, "auto"),       # narrow decode, 16-token layout
    (19000, 384, 16, "auto"),     # wide decode kernel
    (200, 384, 77, "prefill"),    # prefill, ragged tiles
    (200, 384, 5, "w4a4"),        # W4A4
    (19000, 384, 12, "w4a4"),     # W4A4 through the wide kernel
    (200, 512, 77, "w4a4"),       # W4A4 through the prefill kernel, ragged tiles
])
def test_outputs_stay_inside_y(mq, cuda, N, K, M, path):
    # Y lives inside a canary-filled buffer; only its M x N elements may change
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=107)
    w = mq.Weight.pack(W, 0.05)
    X = synth.activations(M, K, seed=108).cuda()
    pad = 4096
    canary = torch.full((pad + M * N + pad,), -7.5, dtype=torch.bfloat16, device="cuda")
    Y = canary[pad:pad + M * N].view(M, N)
    if path == "w4a4":
        w.linear_w4a4(X, Y)
    else:
        w.linear(X, Y, path=path)
    torch.cuda.synchronize()
    assert torch.all(canary[:pad] == -7.5) and torch.all(canary[pad + M * N:] == -7.5)
    fresh = w.linear_w4a4(X) if path == "w4a4" else w.linear(X, path=path)
    torch.cuda.synchronize()
    assert torch.equal(Y, fresh)
