"""The library's host decomposition + packing equals the oracle's, byte for
byte (MosaicQuant "Methodology" 1.: W ~= Q(W) + R, both parts 4-bit, in the
encoding this library fixes). Runs without a GPU (mq_pack_host)."""

import numpy as np
import pytest

import oracle
from bit_gemm_w4_b200 import synth


def _same(mq, W, rho):
    got = mq.pack_host(W, rho)
    want = oracle.pack(oracle.decompose(W, rho))
    for k in ("qweight", "sz", "row_ptr", "col", "val", "rscale"):
        a, b = np.asarray(got[k]), np.asarray(want[k])
        assert a.shape == b.shape, k
        assert a.dtype.itemsize == b.dtype.itemsize, k
        assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)), k


def test_tiny_workload(mq):
    W, _, rho = synth.workload_inputs("tiny")
    _same(mq, W, rho)


def test_7b_qkvo_workload(mq):
    W, _, rho = synth.workload_inputs("7b_decode", 0)
    _same(mq, W, rho)


def test_down_shape_rows(mq):
    W, _, rho = synth.workload_inputs("7b_decode", 2, rows=np.arange(0, 4096, 97))
    _same(mq, W, rho)


def test_70b_like_rows(mq):
    rng = np.random.default_rng(0)
    W = (rng.standard_normal((5, 8192)) * 0.015).astype(np.float32)
    W[:, rng.choice(8192, 32, replace=False)] = (0.2 * rng.standard_t(3, (5, 32))).astype(np.float32)
    _same(mq, W, 0.01)


@pytest.mark.parametrize("rho", [0.0, 0.25, 1.0])
def test_density_extremes(mq, rho):
    W = synth.weight(24, 256, std=0.02, outlier_frac=0.02, seed=9)
    _same(mq, W, rho)


def test_ties_zeros_and_constants(mq):
    W = np.zeros((6, 256), np.float32)
    W[1] = 0.5                                        # constant row
    W[2, ::3] = 0.25                                  # many equal errors
    W[3] = np.tile(np.float32([0.1, -0.1, 0.3, 0.0]), 64)
    W[4, 0] = 1e-9                                    # scale floor 2^-24
    W[5] = np.abs(np.random.default_rng(1).standard_normal(256)).astype(np.float32)
    _same(mq, W, 0.05)


def test_subnormal_scales(mq):
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((8, 128)) * 1e-5).astype(np.float32)
    _same(mq, W, 0.03)


def _same_blocks(mq, W, fraction, h=None):
    got = mq.pack_host(W, 0.0, block_fraction=fraction, channel_weight=h)
    want = oracle.pack(oracle.decompose_blocks(W, fraction, h))
    for k in ("qweight", "sz", "row_ptr", "col", "val", "rscale"):
        a, b = np.asarray(got[k]), np.asarray(want[k])
        assert a.shape == b.shape, k
        assert np.array_equal(a.view(np.uint8), np.ascontiguousarray(b).view(np.uint8)), k


@pytest.mark.parametrize("fraction", [0.0, 0.05, 0.1, 0.3, 1.0])
def test_block_mode_matches_oracle(mq, fraction):
    # "Methodology" 2: 16x64 blocks ranked by the delta score, no weights
    W = synth.weight(256, 1024, std=0.02, outlier_frac=0.005, seed=31)
    _same_blocks(mq, W, fraction)


def test_block_mode_with_calibration_weights(mq):
    # delta score weighted by a diagonal Hessian estimate from calibration X
    W, _, _ = synth.workload_inputs("7b_decode", 0, rows=np.arange(512))
    Xc = synth.activations(64, 4096, seed=5, channels=4, mult=20.0).double().numpy()
    h = (Xc * Xc).sum(0).astype(np.float32)
    _same_blocks(mq, W, 0.1, h)


def test_block_mode_clustered_columns(mq):
    # whole outlier columns: the selection concentrates on their blocks
    W = synth.weight(128, 2048, std=0.015, outlier_frac=0.01, seed=33, outlier_cols=8)
    _same_blocks(mq, W, 0.1)


def test_block_mode_counts_and_errors(mq):
    assert mq.residual_nnz(256, 1024, 0.0, block_fraction=0.1) == 26 * 1024  # 256 blocks
    W = np.zeros((24, 256), np.float32)
    with pytest.raises(mq.MQError) as e:
        mq.pack_host(W, 0.0, block_fraction=0.1)                 # N % 16 != 0
    assert e.value.status == 1
    W = np.zeros((32, 256), np.float32)
    with pytest.raises(mq.MQError) as e:
        mq.pack_host(W, 0.0, block_fraction=0.1, channel_weight=-np.ones(256, np.float32))
    assert e.value.status == 1
    with pytest.raises(mq.MQError) as e:
        mq.pack_host(W, 0.0, block_fraction=2.0)
    assert e.value.status == 1


def _arrays(d):
    return dict(N=d.N, K=d.K, q=d.q, s=d.s, z=d.z, row_ptr=d.row_ptr, col=d.col, qr=d.qr, sr=d.sr)


@pytest.mark.parametrize("N,K,frac", [(32, 256, 0.1), (64, 512, 0.03), (48, 1024, 0.5), (16, 128, 1.0)])
def test_block_tiles_equal_oracle(mq, N, K, frac):
    # the library's block tiles of a block-allocated residual, byte for byte
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=N + K)
    d = oracle.decompose_blocks(W, frac)
    got = mq.block_tiles_host(_arrays(d))
    want = oracle.pack_blocks(d)
    for k in ("blk_ptr", "blk_col", "blk_q"):
        a, b = np.asarray(got[k]), np.asarray(want[k])
        assert a.shape == b.shape and np.array_equal(a.view(np.uint8), b.view(np.uint8)), k


def test_block_tiles_refuse_a_row_residual(mq):
    d = oracle.decompose(synth.weight(32, 256, std=0.02, outlier_frac=0.005, seed=2), 0.05)
    with pytest.raises(mq.MQError) as e:
        mq.block_tiles_host(_arrays(d))
    assert e.value.status == mq.UNSUPPORTED
