"""Pins of the oracle's block mode (MosaicQuant, "Methodology" 2: block-wise
residual allocation with the Hessian-guided delta score)."""

import itertools

import numpy as np
import pytest

import oracle
from bit_gemm_w4_b200 import synth


def _errors(W):
    q, s, z, deq = oracle.quantize_base(W, 128)
    return W.astype(np.float64) - deq


def test_one_hot_channel_weight_scores_are_column_norms():
    # with h = e_j a block's score is the squared norm of column j inside it
    W = synth.weight(48, 256, std=0.02, outlier_frac=0.01, seed=5)
    E = _errors(W)
    for j in (0, 63, 64, 200):
        h = np.zeros(256, np.float32)
        h[j] = 1.0
        sc = oracle.block_scores(E, h).reshape(3, 4)
        for rb in range(3):
            for cb in range(4):
                seg = E[16 * rb:16 * rb + 16, j]
                want = np.linalg.norm(seg) ** 2 if cb == j // 64 else 0.0
                assert sc[rb, cb] == pytest.approx(want, rel=1e-12, abs=0.0)


@pytest.mark.parametrize("n_sel", [0, 1, 3, 5, 12])
def test_selection_is_the_best_subset(n_sel):
    # exhaustive search over all subsets of 12 blocks: the selection maximizes
    # the total score; among equal totals the smallest indices win
    W = synth.weight(48, 256, std=0.02, outlier_frac=0.02, seed=7)
    sc = oracle.block_scores(_errors(W))
    sel = oracle.select_blocks(sc, n_sel)
    best = max(itertools.combinations(range(12), n_sel),
               key=lambda c: (sum(sc[list(c)]), [-i for i in c]))
    assert sorted(np.nonzero(sel)[0].tolist()) == list(best)


def test_ties_go_to_the_smaller_index():
    sel = oracle.select_blocks(np.array([1.0, 2.0, 2.0, 0.5, 2.0]), 2)
    assert np.nonzero(sel)[0].tolist() == [1, 2]


def test_selected_dominate_unselected():
    W = synth.weight(64, 512, std=0.02, outlier_frac=0.01, seed=8)
    h = synth.activations(32, 512, seed=9, channels=4, mult=20.0).double().pow(2).sum(0).numpy()
    sc = oracle.block_scores(_errors(W), h.astype(np.float32))
    sel = oracle.select_blocks(sc, 7)
    assert sc[sel].min() >= sc[~sel].max()


def test_power_of_two_weight_scale_keeps_selection():
    W = synth.weight(64, 512, std=0.02, outlier_frac=0.01, seed=10)
    h = np.random.default_rng(3).random(512).astype(np.float32)
    a = oracle.decompose_blocks(W, 0.2, h)
    b = oracle.decompose_blocks(W, 0.2, h * np.float32(4.0))
    assert np.array_equal(a.col, b.col) and np.array_equal(a.qr, b.qr)


def test_fraction_zero_is_the_plain_base_and_one_covers_everything():
    W = synth.weight(32, 256, std=0.02, outlier_frac=0.01, seed=11)
    d0 = oracle.decompose_blocks(W, 0.0)
    r0 = oracle.decompose(W, 0.0)
    assert d0.row_ptr[-1] == 0 and np.array_equal(d0.q, r0.q)
    d1 = oracle.decompose_blocks(W, 1.0)
    assert d1.row_ptr[-1] == 32 * 256
    # every entry carries a residual: |W - W_hat| <= s_r / 2 unless clamped
    E = _errors(W)
    err = np.abs(W.astype(np.float64) - oracle.w_hat(d1))
    sr = d1.sr.astype(np.float64)[:, None]
    clamped = np.abs(E) > 7.5 * sr
    assert np.all(err[~clamped] <= sr.repeat(256, 1)[~clamped] / 2 + 1e-18)


def test_exact_residual_at_full_fraction_reproduces_w():
    W = synth.weight(32, 256, std=0.02, outlier_frac=0.01, seed=12)
    d = oracle.decompose_blocks(W, 1.0, exact_residual=True)
    assert np.array_equal(oracle.w_hat(d), W.astype(np.float64))


def test_blocks_selected_rounding():
    assert oracle.blocks_selected(32, 256, 0.1) == 1      # 8 blocks * 0.1 = 0.8
    assert oracle.blocks_selected(32, 256, 0.0625) == 1   # 0.5 rounds up
    assert oracle.blocks_selected(32, 256, 0.05) == 0     # 0.4


def test_delta_score_beats_random_blocks_on_output_distortion():
    # the score is the diagonal-Hessian estimate of the output distortion a
    # block's residual removes: on calibration data with outlier channels its
    # choice removes more true output distortion than random choices do
    K = 512
    W = synth.weight(64, K, std=0.02, outlier_frac=0.005, seed=13)
    Xc = synth.activations(64, K, seed=14, channels=6, mult=20.0).double().numpy()
    h = (Xc * Xc).sum(0).astype(np.float32)
    base = oracle.decompose_blocks(W, 0.0)

    def distortion(d):
        return np.sum((Xc @ (W.astype(np.float64) - oracle.w_hat(d)).T) ** 2)

    d_base = distortion(base)
    # both sides with exact residuals, so only the choice of blocks differs
    chosen = distortion(oracle.decompose_blocks(W, 0.1, h, exact_residual=True))
    rng = np.random.default_rng(0)
    E = _errors(W)
    rand = []
    for _ in range(8):
        sel = oracle.select_blocks(rng.random((64 // 16) * (K // 64)),
                                   oracle.blocks_selected(64, K, 0.1))
        mask = np.repeat(np.repeat(sel.reshape(4, 8), 16, 0), 64, 1)
        # the error left with exact residuals on the random blocks
        rand.append(np.sum((Xc @ (E * (1 - mask)).T) ** 2))
    assert chosen < d_base
    assert chosen < min(rand)


def test_rejects_bad_input():
    W = synth.weight(24, 256, std=0.02, outlier_frac=0.0, seed=1)
    with pytest.raises(ValueError):
        oracle.decompose_blocks(W, 0.1)          # N % 16 != 0
    W = synth.weight(32, 256, std=0.02, outlier_frac=0.0, seed=1)
    with pytest.raises(ValueError):
        oracle.decompose_blocks(W, 1.5)
    with pytest.raises(ValueError):
        oracle.decompose_blocks(W, 0.1, -np.ones(256, np.float32))
