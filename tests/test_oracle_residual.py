"""Pin the oracle's sparse 4-bit residual (steps D3, D4).

MosaicQuant, "Methodology" 1.-2. and the abstract: the residual compensates
the quantization error and targets the most error-critical weights; it is
4-bit like the base. Pins: brute force over all subsets on 8x8, the
dominance invariant, the tie rule, the half-step bound of the residual codes,
and the hand-derived example.
"""

import itertools

import numpy as np

from oracle import decompose, select_residual, quantize_residual, residual_count


def _valid(absE, S):
    """S is a correct top-k set iff every chosen entry outranks every other
    (larger |E|, or equal |E| and a smaller column)."""
    rest = [j for j in range(absE.size) if j not in S]
    return all(absE[i] > absE[j] or (absE[i] == absE[j] and i < j)
               for i in S for j in rest)


def test_brute_force_subsets_8x8():
    rng = np.random.default_rng(5)
    E = rng.standard_normal((8, 8))
    E[2, :] = np.round(E[2, :])          # many ties
    E[3, :] = 0.5                        # all tied
    for k in range(0, 9):
        sel = select_residual(E, k)
        for n in range(8):
            absE = np.abs(E[n])
            valid = [S for S in itertools.combinations(range(8), k) if _valid(absE, S)]
            assert len(valid) == 1
            assert list(valid[0]) == list(sel[n])


def test_unselected_dominated():
    rng = np.random.default_rng(6)
    W = (rng.standard_normal((32, 512)) * 0.02).astype(np.float32)
    W.reshape(-1)[rng.choice(W.size, 160, replace=False)] = 0.2 * rng.standard_t(3, 160)
    d = decompose(W, 0.01)
    from oracle import dequant_base
    E = np.abs(W.astype(np.float64) - dequant_base(d))
    for n in range(32):
        a, b = d.row_ptr[n], d.row_ptr[n + 1]
        cols = d.col[a:b]
        assert np.all(np.diff(cols) > 0)
        mask = np.ones(512, bool)
        mask[cols] = False
        assert E[n, mask].max() <= E[n, cols].min()


def test_k_n_rounding():
    assert residual_count(512, 0.01) == 5
    assert residual_count(4096, 0.005) == 20
    assert residual_count(11008, 0.005) == 55
    assert residual_count(8192, 0.01) == 82
    assert residual_count(4096, 0.0025) == 10
    assert residual_count(11008, 0.0025) == 28
    assert residual_count(4096, 0.04) == 164
    assert residual_count(11008, 0.04) == 440
    assert residual_count(4096, 0.0) == 0


def test_residual_code_bound_and_peak():
    rng = np.random.default_rng(7)
    Esel = rng.standard_normal((64, 20)) * 0.01
    qr, sr = quantize_residual(Esel)
    s = sr.astype(np.float64)[:, None]
    raw = np.rint(Esel / s)
    ok = (raw >= -8) & (raw <= 7)
    assert np.all(np.abs(Esel - qr * s)[ok] <= s.repeat(20, 1)[ok] / 2)
    peak = np.argmax(np.abs(Esel), axis=1)
    assert np.all(np.abs(qr[np.arange(64), peak]) == 7)


def test_zero_residual_scale_is_one():
    qr, sr = quantize_residual(np.zeros((3, 4)))
    assert np.all(sr == 1.0) and np.all(qr == 0)
    qr, sr = quantize_residual(np.zeros((3, 0)))
    assert np.all(sr == 1.0)


def test_hand_derived_example(golden):
    f = golden("hand_group8.txt")
    v = np.array([float(x) for x in f["v"]], np.float32).reshape(1, -1)
    d = decompose(v, float(f["rho"][0]), group=int(f["group"][0]))
    np.testing.assert_array_equal(d.col, [int(x) for x in f["col"]])
    np.testing.assert_array_equal(d.qr, [int(x) for x in f["qr"]])
    assert d.sr.view(np.uint16)[0] == int(f["sr_bits"][0], 16)
