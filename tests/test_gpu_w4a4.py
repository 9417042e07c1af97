"""GPU parity of the W4A4 variant (MosaicQuant "Methodology" 3.: the
pipeline's quantization stage; "Experimental Results": W4A4) against the
fp64 W4A4 oracle, through the C ABI: the activation codes and scales
bit-exact, outputs within the normalized and relative bounds."""

import numpy as np
import pytest
import torch

import oracle
from oracle.w4a4 import quantize_activations as oracle_quantize
from bit_gemm_w4_b200 import synth
from gpu_util import oracle_check_w4a4

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,K", [(1, 128), (5, 4096), (16, 11008), (64, 4096)])
def test_quantization_bit_exact(mq, cuda, M, K):
    X = synth.activations(M, K, seed=80 + M, channels=4, mult=25.0)
    if M > 2:
        X[2] = 0                                  # a zero token: scale 1, codes 0
    codes, scales = mq.quantize_activations(X.cuda())
    torch.cuda.synchronize()
    c_ref, s_ref = oracle_quantize(X)
    assert np.array_equal(codes.cpu().numpy(), c_ref)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_quantization_ties(mq, cuda):
    x = torch.tensor([[7.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5]]).to(torch.bfloat16)
    codes, scales = mq.quantize_activations(x.cuda())
    torch.cuda.synchronize()
    assert codes.cpu().tolist() == [[7, 2, 4, -2, -4, 0, 0, 2]]
    assert float(scales[0]) == 1.0


@pytest.mark.parametrize("N,K,M,rho", [
    (512, 4096, 1, 0.005),       # M = 1 layout
    (512, 4096, 5, 0.04),        # M <= 8 layout, dense residual
    (512, 4096, 16, 0.01),       # M = 16 layout
    (200, 384, 13, 0.05),        # ragged rows, odd group count
    (256, 8192, 16, 0.01),       # K split over a cluster of 2
    (128, 11008, 16, 0.005),     # cluster of 2, uneven group split
    (64, 32768, 16, 0.002),      # cluster of 8
    (300, 4096, 9, 0.0),         # density 0
])
def test_w4a4_parity(mq, cuda, N, K, M, rho):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=N + K + M)
    X = synth.activations(M, K, seed=M + 3, channels=4, mult=20.0)
    w = mq.Weight.pack(W, rho)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check_w4a4(Y, X, oracle.decompose(W, rho))
    assert r["ok"], r


@pytest.mark.parametrize("M", [1, 16])
def test_w4a4_block_residual(mq, cuda, M):
    # block mode: long residual rows read from global memory by the walk
    W = synth.weight(256, 4096, std=0.02, outlier_frac=0.005, seed=91)
    w = mq.Weight.pack(W, block_fraction=0.25)
    X = synth.activations(M, 4096, seed=92, channels=4, mult=20.0)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    r = oracle_check_w4a4(Y, X, oracle.decompose_blocks(W, 0.25))
    assert r["ok"], r


def test_w4a4_7b_shapes_sampled_rows(mq, cuda):
    # the three 7B decode shapes at M = 1, 48 rows each against the oracle
    from bit_gemm_w4_b200.synth import WORKLOADS
    cfg = WORKLOADS["7b_decode"]
    for i, (N, K) in enumerate(cfg["shapes"]):
        W, X, rho = synth.workload_inputs("7b_decode", i)
        w = mq.Weight.pack(W, rho)
        Y = w.linear_w4a4(X.cuda())
        torch.cuda.synchronize()
        rows = np.unique(np.concatenate([np.arange(16), np.arange(N - 16, N),
                                         np.random.default_rng(i).choice(N, 16, replace=False)]))
        d = oracle.decompose(W[rows], rho)
        sub = Y[:, torch.from_numpy(rows).cuda()]
        r = oracle_check_w4a4(sub, X, d)
        assert r["ok"], (N, K, r)


def test_w4a4_errors(mq, cuda):
    W = synth.weight(64, 384, std=0.02, outlier_frac=0.01, seed=93)
    w = mq.Weight.pack(W, 0.02)
    X = synth.activations(17, 384, seed=94).cuda()
    with pytest.raises(mq.MQError) as e:      # the prefill form needs K % 256 == 0
        w.linear_w4a4(X)
    assert e.value.status == mq.UNSUPPORTED
    ws = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(mq.MQError) as e:
        w.linear_w4a4(X[:4], workspace=ws)
    assert e.value.status == mq.INVALID_ARG


@pytest.mark.parametrize("M,mode", [(9, "rows"), (16, "rows"), (16, "blocks")])
def test_w4a4_wide_kernel(mq, cuda, M, mode):
    # a layer tall enough for the wide kernel's W4A4 form (150 128-row
    # blocks, K = 384: a last stage holding one group)
    N, K = 19200, 384
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=101)
    X = synth.activations(M, K, seed=102 + M, channels=2, mult=20.0)
    if mode == "rows":
        w = mq.Weight.pack(W, 0.05)
        d = oracle.decompose(W, 0.05)
    else:
        w = mq.Weight.pack(W, block_fraction=0.2)
        d = oracle.decompose_blocks(W, 0.2)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check_w4a4(Y, X, d)
    assert r["ok"], r


def test_w4a4_70b_mlp_sampled_rows(mq, cuda):
    # the 70B MLP at M = 16 through the wide kernel's W4A4 form
    N, K = synth.WORKLOADS["70b_mlp"]["shapes"][0]
    W, X, rho = synth.workload_inputs("70b_mlp")
    w = mq.Weight.pack(W, rho)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    rows = np.unique(np.concatenate([np.arange(0, 24), np.arange(N - 24, N),
                                     np.random.default_rng(1).choice(N, 48, replace=False)]))
    d = oracle.decompose(np.ascontiguousarray(W[rows]), rho)
    r = oracle_check_w4a4(Y[:, torch.from_numpy(rows).cuda()], X, d)
    assert r["ok"], r


# ---------------------------------------------------------------- M > 16: the tcgen05 prefill kernel (kind::i8)
@pytest.mark.parametrize("N,K,M,rho", [
    (512, 4096, 17, 0.005),      # one partial token tile
    (300, 1024, 200, 0.02),      # ragged rows and tokens, two token tiles
    (256, 2048, 256, 0.0),       # no residual: eight operand slots
    (384, 512, 130, 0.05),       # dense residual, a 2-token last tile
    (128, 8192, 64, 0.01),       # long K
    (1000, 768, 129, 0.005),     # 6 groups, ragged rows
])
def test_w4a4_prefill_parity(mq, cuda, N, K, M, rho):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=N + K + M)
    X = synth.activations(M, K, seed=M + 7, channels=4, mult=20.0)
    X[M // 2] = 0                                 # a zero token: scale 1, output 0
    w = mq.Weight.pack(W, rho)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    assert not Y[M // 2].any()
    r = oracle_check_w4a4(Y, X, oracle.decompose(W, rho))
    assert r["ok"], r


def test_w4a4_prefill_block_residual(mq, cuda):
    W = synth.weight(256, 4096, std=0.02, outlier_frac=0.005, seed=95)
    w = mq.Weight.pack(W, block_fraction=0.25)
    X = synth.activations(100, 4096, seed=96, channels=4, mult=20.0)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    r = oracle_check_w4a4(Y, X, oracle.decompose_blocks(W, 0.25))
    assert r["ok"], r


def test_w4a4_prefill_full_size_sampled_rows(mq, cuda):
    # the prefill workload (M = 2048, 14336 x 4096, density 0.5 %) in the
    # launch configuration the bench times, 64 rows against the oracle
    W, X, rho = synth.workload_inputs("prefill")
    N = W.shape[0]
    w = mq.Weight.pack(W, rho)
    Y = w.linear_w4a4(X.cuda())
    torch.cuda.synchronize()
    assert w.device_error() == 0
    rows = np.unique(np.concatenate([np.arange(0, 16), np.arange(N - 16, N),
                                     np.random.default_rng(3).choice(N, 32, replace=False)]))
    d = oracle.decompose(np.ascontiguousarray(W[rows]), rho)
    sub = Y[:, torch.from_numpy(rows).cuda()]
    r = oracle_check_w4a4(sub, X, d)
    assert r["ok"], r
