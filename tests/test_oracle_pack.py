"""Pin the oracle's packed layout: exact round trip, the nibble interleave's
extraction property, and hand-derived packed words."""

import numpy as np

from oracle import decompose, pack, unpack, from_arrays
from bit_gemm_w4_b200 import synth


def _eq(a, b):
    for f in ("q", "s", "z", "row_ptr", "col", "qr", "sr"):
        x, y = getattr(a, f), getattr(b, f)
        assert x.shape == y.shape, f
        assert np.array_equal(np.asarray(x).view(np.uint8), np.asarray(y).view(np.uint8)) or \
            np.array_equal(x, y), f


def test_round_trip_decomposition():
    W, _, rho = synth.workload_inputs("tiny")
    d = decompose(W, rho)
    _eq(unpack(pack(d), d.N, d.K), d)


def test_round_trip_odd_nnz_and_sweep_draw():
    d = from_arrays(synth.sweep_decomposition(9, 256, 3, seed=4))
    assert d.nnz % 2 == 1
    p = pack(d)
    assert p["val"].size == (d.nnz + 1) // 2
    assert (p["val"][-1] >> 4) == 0          # pad nibble
    _eq(unpack(p, d.N, d.K), d)


def test_pair_extraction_property():
    rng = np.random.default_rng(0)
    d = from_arrays(synth.sweep_decomposition(4, 128, 0, seed=1))
    d.q[:] = rng.integers(0, 16, d.q.shape, dtype=np.uint8)
    w = pack(d)["qweight"]
    for i in range(4):
        pair = (w >> np.uint32(4 * i)) & np.uint32(0x000F000F)
        np.testing.assert_array_equal(pair & 0xF, d.q.reshape(4, -1, 8)[:, :, 2 * i])
        np.testing.assert_array_equal(pair >> 16, d.q.reshape(4, -1, 8)[:, :, 2 * i + 1])


def test_hand_derived_words(golden):
    f = golden("hand_group8.txt")
    v = np.array([float(x) for x in f["v"]], np.float32).reshape(1, -1)
    d = decompose(v, float(f["rho"][0]), group=int(f["group"][0]))
    p = pack(d)
    assert int(p["qweight"][0, 0]) == int(f["qweight"][0], 16)
    assert int(p["sz"][0, 0]) == int(f["sz"][0], 16)
    assert [int(b) for b in p["val"]] == [int(x, 16) for x in f["val"]]
    assert list(p["row_ptr"]) == [0, 3]
