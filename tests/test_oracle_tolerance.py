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


def test_t1_allows_half_an_ulp_not_one():
    # a weight row exactly parallel to x, scaled so that y64 sits just above
    # a power of two: there |y64| ~ ||x|| ||w|| and one bf16 ulp is |y64|/128
    x = np.ones((1, 128))
    w = np.ones((1, 128)) * (1.01 / 128)
    Y64 = x @ w.T                                    # 1.01
    wn = np.linalg.norm(w, axis=1)
    Yb = torch.from_numpy(Y64).to(torch.bfloat16).double().numpy()
    r = parity_report(Yb, Y64, x, wn)
    assert r["ok"] and r["t1"] == 0.0                # correct rounding passes
    assert r["t1_raw"] > 2e-3                        # which alone would exceed the bound
    u = bf16_ulp(Y64)
    assert parity_report(Y64 + 0.5 * u, Y64, x, wn)["t1"] == 0.0    # half an ulp: free
    assert not parity_report(Y64 + u, Y64, x, wn)["ok"]            # one full ulp off fails
    assert not parity_report(Y64 - u, Y64, x, wn)["ok"]
