"""The no-allocation variant of the unfused path (mq_linear_unfused_noalloc).

It exists for callers that cannot allocate device memory or pass a
workspace (fixed memory budgets, plugins that only receive their input and
output buffers, hosts that route every allocation through their own
allocator). It keeps the fp32 partial outputs in a fixed array inside the
library. This file is collected last so that a run stopping at the first
failure has already run every other test.
"""

import numpy as np
import pytest
import torch

import oracle
from bit_gemm_w4_b200 import synth
from gpu_util import oracle_check

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M", [1, 16, 40])
def test_noalloc_matches_workspace_unfused_twice(mq, cuda, M):
    W = synth.weight(264, 1024, std=0.02, outlier_frac=0.01, seed=M)
    w = mq.Weight.pack(W, 0.02)
    d = oracle.decompose(W, 0.02)
    for call in range(2):   # two calls in a row share (and reuse) the scratch
        X = synth.activations(M, 1024, seed=50 + 10 * M + call, channels=4, mult=20.0).cuda()
        Y_ref = w.linear_unfused(X)          # existing entry point, caller workspace
        Y_na = w.linear_unfused_noalloc(X)   # built-in scratch, no allocation
        torch.cuda.synchronize()
        r = oracle_check(Y_na, X.cpu(), d)
        assert r["ok"], (call, r)
        diff = (Y_na.float() - Y_ref.float()).abs()
        rel = diff / Y_ref.float().abs().clamp_min(1e-3)
        assert float(rel.max()) <= 2 ** -7, call
        assert w.device_error() == 0


@pytest.mark.parametrize("N,K,M,rows", [
    (4096, 256, 512, 48),        # M*N exactly the capacity, through the prefill kernel
    (131072, 128, 16, 48),       # M*N exactly the capacity, through a decode kernel
])
def test_noalloc_at_capacity(mq, cuda, N, K, M, rows):
    # the largest call the built-in scratch takes: every partial index up to
    # the array's end is written by the dense kernel and read by the merge
    assert M * N == mq.UNFUSED_NOALLOC_MAX_OUTPUTS
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=N + M)
    w = mq.Weight.pack(W, 0.01)
    X = synth.activations(M, K, seed=3, channels=4, mult=20.0).cuda()
    Y_ref = w.linear_unfused(X)
    Y_na = w.linear_unfused_noalloc(X)
    torch.cuda.synchronize()
    assert w.device_error() == 0
    diff = (Y_na.float() - Y_ref.float()).abs()
    assert float((diff / Y_ref.float().abs().clamp_min(1e-3)).max()) <= 2 ** -7
    # sampled rows against the oracle, including the last ones
    d = oracle.decompose(W, 0.01)
    pick = np.unique(np.concatenate([np.arange(rows - 8), np.arange(N - 8, N)]))
    Y64 = oracle.linear(X.cpu().double().numpy(), d, rows=pick)
    wn = np.linalg.norm(oracle.w_hat(d)[pick], axis=1)
    from oracle.tolerance import parity_report
    r = parity_report(Y_na.float().cpu().double().numpy()[:, pick], Y64, X.cpu().double().numpy(), wn)
    assert r["ok"], r


def test_noalloc_rejects_oversized_outputs(mq, cuda):
    N = 4096
    W = synth.weight(N, 128, std=0.02, outlier_frac=0.0, seed=1)
    w = mq.Weight.pack(W, 0.01)
    M = 2 * 1024 * 1024 // N + 1          # M*N just above the built-in capacity
    X = torch.zeros((M, 128), dtype=torch.bfloat16, device=cuda)
    with pytest.raises(mq.MQError) as e:
        w.linear_unfused_noalloc(X)
    assert e.value.status == mq.INVALID_ARG and "scratch" in str(e.value)
