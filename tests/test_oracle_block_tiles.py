"""Pin the oracle's block-tile layout (P4) of a block-allocated residual:
exact round trip against the CSR it restates, the block count the selection
fixes, rejection of residuals that are not whole blocks, and hand-derived
words."""

import numpy as np
import pytest

from oracle import (Decomposition, block_structure, blocks_selected, decompose,
                    decompose_blocks, pack, pack_blocks, unpack_blocks)
from oracle.pack import PI
from bit_gemm_w4_b200 import synth


def _weight(N, K, seed):
    return synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=seed)


@pytest.mark.parametrize("frac", [0.0, 0.03, 0.1, 0.5, 1.0])
def test_round_trip_matches_the_csr(frac):
    N, K = 64, 512
    d = decompose_blocks(_weight(N, K, 3), frac)
    p = pack_blocks(d)
    assert p["blk_col"].size == blocks_selected(N, K, frac)
    row_ptr, col, qr = unpack_blocks(p, N, K)
    assert np.array_equal(row_ptr, d.row_ptr)
    assert np.array_equal(col, d.col)
    assert np.array_equal(qr, d.qr)
    # each tile word holds the codes of eight consecutive columns
    assert p["blk_q"].shape == (p["blk_col"].size, 16, 8)


def test_block_structure_rejects_row_mode_and_ragged_shapes():
    d = decompose(_weight(32, 256, 4), 0.05)       # per-row top-k entries
    assert d.nnz > 0 and block_structure(d) is None
    with pytest.raises(ValueError):
        pack_blocks(d)
    d0 = decompose(_weight(24, 256, 5), 0.0)        # N not a multiple of 16
    assert block_structure(d0) is None
    d1 = decompose(_weight(32, 256, 6), 0.0)        # no residual at all: zero blocks
    p = pack_blocks(d1)
    assert p["blk_col"].size == 0 and list(p["blk_ptr"]) == [0, 0, 0]


def test_hand_derived_tile_words():
    # one block at column-block 1 of a 16 x 128 weight; row 0 holds
    # q_r = (c - 64) % 16 - 8 on columns c = 64..127, so u = q_r + 8 runs
    # 0, 1, ..., 15, 0, ...; word 0 (columns 64..71) holds u = pi(j) in
    # nibble j, word 1 (columns 72..79) u = 8 + pi(j)
    N, K = 16, 128
    cols = np.tile(np.arange(64, 128), N)
    qr = np.tile(((np.arange(64, 128) - 64) % 16 - 8), N).astype(np.int8)
    d = Decomposition(N, K, 128, np.zeros((N, K), np.uint8), np.ones((N, 1), np.float16),
                      np.zeros((N, 1), np.float16), np.arange(N + 1, dtype=np.int64) * 64,
                      cols.astype(np.int64), qr, np.ones(N, np.float16))
    p = pack_blocks(d)
    assert list(p["blk_ptr"]) == [0, 1] and list(p["blk_col"]) == [1]
    assert int(p["blk_q"][0, 0, 0]) == 0x75316420     # nibbles 0,2,4,6,1,3,5,7
    assert int(p["blk_q"][0, 0, 1]) == 0xFDB9ECA8     # nibbles 8,10,12,14,9,11,13,15
    assert int(p["blk_q"][0, 15, 7]) == 0xFDB9ECA8    # columns 120..127: u = 8..15
    # the words hold the same codes as the CSR's two's-complement nibbles
    val = pack(d)["val"]
    assert (int(val[0]) & 0xF) == (-8 & 0xF) and (int(val[0]) >> 4) == (-7 & 0xF)


def test_pair_extraction_gives_offset_codes():
    # the base codes' pair extraction applies unchanged: (word >> 4i) &
    # 0x000F000F holds u of columns 8w + 2i and 8w + 2i + 1
    d = decompose_blocks(_weight(32, 256, 7), 0.25)
    p = pack_blocks(d)
    w = p["blk_q"]
    for b in range(w.shape[0]):
        rb = np.searchsorted(p["blk_ptr"], b, side="right") - 1
        cb = int(p["blk_col"][b])
        for r in (0, 9):
            row = 16 * rb + r
            lo, hi = d.row_ptr[row], d.row_ptr[row + 1]
            c = d.col[lo:hi]
            u = d.qr[lo:hi][(c >= 64 * cb) & (c < 64 * cb + 64)].astype(np.int32) + 8
            for i in range(4):
                pair = (w[b, r] >> np.uint32(4 * i)) & np.uint32(0x000F000F)
                assert np.array_equal(pair & 0xF, u.reshape(8, 8)[:, 2 * i])
                assert np.array_equal(pair >> 16, u.reshape(8, 8)[:, 2 * i + 1])
    assert PI == (0, 2, 4, 6, 1, 3, 5, 7)
