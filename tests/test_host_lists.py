"""The prefill kernel's residual lists, built on the host at upload, checked
on the CPU: regrouping the packed CSR by (128-row tile, 64-column stage,
32-row quadrant) must give back every entry exactly once, with its row,
column and int4 code, in (group, row, column) order (mq_prefill_lists_host
exports the lists the upload sends to the device)."""

import numpy as np
import pytest

from bit_gemm_w4_b200 import mosaicq as mq, synth


def _entries(packed):
    """(row, column, code) of every CSR entry of a host pack."""
    rp, col, val = packed["row_ptr"], packed["col"], packed["val"]
    out = []
    for n in range(len(rp) - 1):
        for e in range(rp[n], rp[n + 1]):
            nib = (int(val[e >> 1]) >> ((e & 1) * 4)) & 0xF
            out.append((n, int(col[e]), (nib ^ 8) - 8))
    return out


def _expected(N, K, packed):
    nk = K // 64
    keys = ((N + 127) // 128) * nk * 4
    groups = [[] for _ in range(keys)]
    for n, c, q in _entries(packed):
        groups[((n // 128) * nk + c // 64) * 4 + (n % 128) // 32].append((n, c, q))
    ptr = np.zeros(keys + 1, np.int64)
    ent = []
    for k, g in enumerate(groups):
        g.sort()
        ptr[k + 1] = ptr[k] + len(g)
        for n, c, q in g:
            bits = int(np.array([q], np.float32).view(np.uint32)[0]) & 0xFFFF0000
            ent.append((n % 128) | ((c % 64) << 8) | bits)
    return ptr, np.array(ent, np.uint64)


@pytest.mark.parametrize("N,K,rho,blocks", [
    (300, 512, 0.05, None),      # ragged last tile, row mode
    (128, 384, 0.1, None),       # one tile, six stages
    (256, 1024, 0.0, 0.25),      # block mode
    (64, 256, 0.0, None),        # no residual
])
def test_prefill_lists_regroup_the_csr(N, K, rho, blocks):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=N + K)
    packed = mq.pack_host(W, rho, block_fraction=blocks)
    ptr, ent = mq.prefill_lists_host(N, K, packed)
    eptr, eent = _expected(N, K, packed)
    assert np.array_equal(ptr.astype(np.int64), eptr)
    assert np.array_equal(ent.astype(np.uint64), eent)
    # every code is an exact bf16 integer in [-8, 7]
    codes = (ent.astype(np.uint32) & 0xFFFF0000).view(np.float32)
    assert np.all(codes == np.round(codes)) and codes.min(initial=0) >= -8 and codes.max(initial=0) <= 7


def test_prefill_lists_reject_bad_input():
    rp = np.array([0, 2, 1], np.int32)           # decreasing offsets
    packed = dict(row_ptr=rp, col=np.array([0, 1], np.uint16), val=np.array([0x12], np.uint8))
    with pytest.raises(mq.MQError) as e:
        mq.prefill_lists_host(2, 128, packed)
    assert e.value.status == mq.INVALID_ARG
    packed = dict(row_ptr=np.array([0, 1], np.int32), col=np.array([130], np.uint16),
                  val=np.array([0x01], np.uint8))   # a column not below K
    with pytest.raises(mq.MQError) as e:
        mq.prefill_lists_host(1, 128, packed)
    assert e.value.status == mq.INVALID_ARG


def _wide_expected(N, K, packed):
    S = (K + 255) // 256
    slices = ((N + 127) // 128) * S
    buckets = [[[] for _ in range(128)] for _ in range(slices)]
    rp, col, val = packed["row_ptr"], packed["col"], packed["val"]
    for n in range(N):
        for e in range(rp[n], rp[n + 1]):
            c = int(col[e])
            nib = (int(val[e >> 1]) >> ((e & 1) * 4)) & 0xF
            u = ((n % 128) // 16) * 16 + ((c % 256) // 128) * 8 + (c % 32) // 4
            buckets[(n // 128) * S + c // 256][u].append((n, c, (c % 256) | ((n % 16) << 8) | (nib << 12)))
    ptr = np.zeros(slices + 1, np.int64)
    off = np.zeros((slices, 136), np.int64)
    ent = []
    for k in range(slices):
        pos = 0
        for u in range(128):
            off[k, u] = pos
            b = sorted(buckets[k][u])
            ent.extend(w for _, _, w in b)
            pos += len(b)
        off[k, 128] = pos
        ptr[k + 1] = ptr[k] + pos
    return ptr, off, np.array(ent, np.int64)


@pytest.mark.parametrize("N,K,rho,blocks", [
    (300, 640, 0.05, None),      # ragged block, a half last stage (K % 256 = 128)
    (256, 1024, 0.0, 0.25),      # block mode
    (128, 256, 0.0, None),       # no residual
])
def test_wide_lists_regroup_the_csr(N, K, rho, blocks):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=2 * N + K)
    packed = mq.pack_host(W, rho, block_fraction=blocks)
    ptr, off, ent, mx = mq.wide_lists_host(N, K, packed)
    eptr, eoff, eent = _wide_expected(N, K, packed)
    assert np.array_equal(ptr.astype(np.int64), eptr)
    assert np.array_equal(off[:, :129].astype(np.int64), eoff[:, :129])
    assert np.array_equal(ent.astype(np.int64), eent)
    assert mx == int(np.diff(eptr).max(initial=0))


def _fragment_byte(r, c):
    """Byte of the code at (row r, column c) of a 16-row x 128-column group in
    the m16n8k16 bf16 A fragments of its k-step, from the fragment's
    definition: thread 4 * (row % 8) + kk % 8 / 2 holds element (row, kk) in
    register (row >= 8) + 2 * (kk >= 8), half kk % 2; under the packed
    codes' nibble interleave, k-step s of thread t covers columns 32t + 4s +
    {0, 1} as kk = 2t + {0, 1} and 32t + 4s + {2, 3} as kk = 2t + 8 + {0, 1}."""
    t, s, j = c // 32, (c % 32) // 4, c % 4
    kk = 2 * t + (j % 2) + (8 if j >= 2 else 0)
    lane = 4 * (r % 8) + (kk % 8) // 2
    reg = int(r >= 8) + 2 * int(kk >= 8)
    return s * 512 + lane * 16 + reg * 4 + (kk % 2) * 2


def _tile_expected(N, K, packed):
    G = K // 128
    keys = ((N + 15) // 16) * G
    buckets = [[] for _ in range(keys)]
    rp, col, val = packed["row_ptr"], packed["col"], packed["val"]
    for n in range(N):
        for e in range(rp[n], rp[n + 1]):
            c = int(col[e])
            nib = (int(val[e >> 1]) >> ((e & 1) * 4)) & 0xF
            key = (n // 16) * G + c // 128
            buckets[key].append(_fragment_byte(n % 16, c % 128) | (nib << 12))
    ptr = np.zeros(keys + 1, np.int64)
    for k in range(keys):
        ptr[k + 1] = ptr[k] + len(buckets[k])
    return ptr, np.array([w for b in buckets for w in b], np.int64)


@pytest.mark.parametrize("N,K,rho,blocks", [
    (300, 640, 0.05, None),      # ragged last tile, five groups
    (256, 1024, 0.0, 0.25),      # block mode
    (128, 256, 0.0, None),       # no residual
    (17, 128, 0.3, None),        # one group, a second tile of one row
    (1, 256, 0.5, None),         # one row: half its entries in the residual
])
def test_tile_lists_regroup_the_csr(N, K, rho, blocks):
    W = synth.weight(N, K, std=0.02, outlier_frac=0.01, seed=3 * N + K)
    packed = mq.pack_host(W, rho, block_fraction=blocks)
    ptr, ent = mq.tile_lists_host(N, K, packed)
    eptr, eent = _tile_expected(N, K, packed)
    assert np.array_equal(ptr.astype(np.int64), eptr)
    assert np.array_equal(ent.astype(np.int64), eent)


def test_fragment_byte_covers_each_k_step_once():
    # every (row, column) of a group lands on its own byte pair, and the
    # sixteen rows x sixteen columns of one k-step fill its 512 bytes exactly
    seen = {_fragment_byte(r, c) for r in range(16) for c in range(128)}
    assert seen == set(range(0, 4096, 2))
    for s in range(8):
        cols = [c for c in range(128) if (c % 32) // 4 == s]
        assert {_fragment_byte(r, c) for r in range(16) for c in cols} == set(range(512 * s, 512 * s + 512, 2))
