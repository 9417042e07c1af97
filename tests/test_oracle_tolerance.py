"""Pin the parity metrics: the bf16 grid spacing and the two bounds."""

import numpy as np
import torch

from oracle.tolerance import bf16_ulp, parity_report


def test_bf16_ulp_matches_torch_grid():
    rng = np.random.default_rng(0)
    y = np.concatenate([rng.standard_normal(2000) * 10 ** rng.uniform(-3, 3, 2000), [1.0, -2.0, 0.75]])
    t = torch.from_numpy(y.astype(np.float32)).to(torch.bfloat16)
    nxt = torch.nextafter(t.abs(), torch.tensor(float("inf"), dtype=torch.bfloat16))
    spacing = (nxt.double() - t.abs().double()).numpy()
    # on bf16 values the helper gives the distance to the next value up
    assert np.array_equal(bf16_ulp(t.double().numpy()), spacing)
    # and for any y the spacing of the binade holding |y|
    assert np.array_equal(bf16_ulp(y), np.exp2(np.floor(np.log2(np.abs(y))) - 7))


def test_exact_rounding_passes_and_real_errors_fail():
    rng = np.random.default_rng(1)
    X = rng.standard_normal((4, 256))
    W = rng.standard_normal((32, 256)) * 0.02
    W[3] = X[0] * 0.5                    # nearly parallel row: |y| ~ ||x|| ||w||
    Y64 = X @ W.T
    wn = np.linalg.norm(W, axis=1)
    Yb = torch.from_numpy(Y64).to(torch.bfloat16).double().numpy()
    assert parity_report(Yb, Y64, X, wn)["ok"]
    bad = Yb.copy()
    bad[1, 5] += 0.01 * np.linalg.norm(X[1]) * wn[5]      # a real error
    assert not parity_report(bad, Y64, X, wn)["ok"]
    bad = Yb.copy()
    i = np.argmax(np.abs(Y64[2]) > 0.5)
    bad[2, i] *= 1.05                                       # 5 % relative error
    assert not parity_report(bad, Y64, X, wn)["ok"]
