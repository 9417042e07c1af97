"""Oracle: the device byte layout of a decomposition, and its inverse.

Test infrastructure (see oracle/__init__.py): never imported by the product.
This restates the layout from its definition so the library's packer can be
compared byte for byte; it shares no code with the library.

Layout (the encoding this library fixes for MosaicQuant's dense 4-bit base
and sparse 4-bit residual, "Methodology" 1.):
  P1 qweight u32 [N][K/8]: bits [4j, 4j+4) of word w hold q[n][8w + pi(j)]
     with pi = (0, 2, 4, 6, 1, 3, 5, 7). Shifting the word right by 4i and
     masking 0x000F000F leaves the codes of columns 8w+2i (low half) and
     8w+2i+1 (high half).
  P2 sz u32 [N][K/128]: fp16 bits of s in the low half, of z in the high half.
  P3 row_ptr i32 [N+1]; col u16 [nnz] (ascending within a row); val u8
     [ceil(nnz/2)]: entry e in byte e>>1, low nibble when e is even, two's
     complement int4, a final odd pad nibble 0; rscale u16 [N]: fp16 bits of
     s_r.
  P4 block tiles, for a residual made of whole 16-row x 64-column blocks on
     the fixed block grid (the block allocation of "Methodology" 2.):
     blk_ptr i32 [N/16 + 1] offsets of each 16-row block-row's selected
     blocks; blk_col u16 [nblk] their column-block index cb (the block covers
     columns 64*cb .. 64*cb + 63), ascending within a block-row; blk_q u32
     [nblk][16][8]: word w of row r of a block holds, in bits [4j, 4j+4),
     u = q_r + 8 (offset binary, 0..15) of column 64*cb + 8w + pi(j), the
     base codes' interleave. Every entry of a selected block is present in
     the CSR (P3), so the tiles carry the same codes.
"""

from __future__ import annotations

import numpy as np

from .decompose import Decomposition

PI = (0, 2, 4, 6, 1, 3, 5, 7)


def pack(d: Decomposition) -> dict:
    """Decomposition -> dict of numpy arrays in the device layout."""
    if d.exact is not None:
        raise ValueError("the exact-residual test mode has no packed form")
    N, K = d.N, d.K
    if K % 8 or K > 65536:
        raise ValueError("K must be a multiple of 8 and at most 65536")
    q = d.q.astype(np.uint32).reshape(N, K // 8, 8)
    qweight = np.zeros((N, K // 8), dtype=np.uint32)
    for j in range(8):
        qweight |= q[:, :, PI[j]] << np.uint32(4 * j)
    sz = (d.s.view(np.uint16).astype(np.uint32)
          | (d.z.view(np.uint16).astype(np.uint32) << np.uint32(16)))
    nnz = d.nnz
    nib = (d.qr.astype(np.int16) & 0xF).astype(np.uint8)
    if nnz % 2:
        nib = np.concatenate([nib, np.zeros(1, np.uint8)])
    val = (nib[0::2] | (nib[1::2] << np.uint8(4))).astype(np.uint8)
    return dict(
        qweight=qweight,
        sz=sz.astype(np.uint32),
        row_ptr=d.row_ptr.astype(np.int32),
        col=d.col.astype(np.uint16),
        val=val,
        rscale=d.sr.view(np.uint16).copy(),
    )


def unpack(p: dict, N: int, K: int, group: int = 128) -> Decomposition:
    """Device layout -> Decomposition (the inverse of pack)."""
    qweight = np.asarray(p["qweight"], np.uint32).reshape(N, K // 8)
    q = np.zeros((N, K // 8, 8), dtype=np.uint8)
    for j in range(8):
        q[:, :, PI[j]] = ((qweight >> np.uint32(4 * j)) & np.uint32(0xF)).astype(np.uint8)
    sz = np.asarray(p["sz"], np.uint32).reshape(N, K // group)
    s = (sz & np.uint32(0xFFFF)).astype(np.uint16).view(np.float16)
    z = (sz >> np.uint32(16)).astype(np.uint16).view(np.float16)
    row_ptr = np.asarray(p["row_ptr"], np.int32).astype(np.int64)
    nnz = int(row_ptr[-1])
    val = np.asarray(p["val"], np.uint8)
    nib = np.empty(2 * val.size, dtype=np.uint8)
    nib[0::2] = val & 0xF
    nib[1::2] = val >> 4
    nib = nib[:nnz].astype(np.int16)
    qr = np.where(nib >= 8, nib - 16, nib).astype(np.int8)
    col = np.asarray(p["col"], np.uint16).astype(np.int64)
    sr = np.asarray(p["rscale"], np.uint16).view(np.float16)
    return Decomposition(N, K, group, q.reshape(N, K), s, z, row_ptr, col, qr,
                         sr.copy())


BLOCK_ROWS, BLOCK_COLS = 16, 64


def block_structure(d: Decomposition):
    """(blk_ptr, blk_col) when the residual consists of whole 16 x 64 blocks
    on the block grid: N % 16 == 0, K % 64 == 0, and in every block-row each
    of the 16 rows holds exactly the columns of the same aligned 64-column
    runs. None otherwise."""
    N, K = d.N, d.K
    if N % BLOCK_ROWS or K % BLOCK_COLS:
        return None
    ptr, cols = [0], []
    for rb in range(N // BLOCK_ROWS):
        runs = None
        for r in range(rb * BLOCK_ROWS, (rb + 1) * BLOCK_ROWS):
            c = d.col[d.row_ptr[r]:d.row_ptr[r + 1]]
            if c.size % BLOCK_COLS:
                return None
            cb = c.reshape(-1, BLOCK_COLS)
            if cb.size and (np.any(cb[:, 0] % BLOCK_COLS) or
                            np.any(cb != cb[:, :1] + np.arange(BLOCK_COLS)[None, :])):
                return None
            these = cb[:, 0] // BLOCK_COLS
            if runs is None:
                runs = these
            elif not np.array_equal(runs, these):
                return None
        cols.extend(int(x) for x in runs)
        ptr.append(len(cols))
    return np.asarray(ptr, np.int32), np.asarray(cols, np.uint16)


def pack_blocks(d: Decomposition) -> dict:
    """The P4 block tiles of a block-structured residual (ValueError
    otherwise)."""
    bs = block_structure(d)
    if bs is None:
        raise ValueError("the residual is not made of whole 16 x 64 blocks")
    blk_ptr, blk_col = bs
    nblk = blk_col.size
    tiles = np.zeros((nblk, BLOCK_ROWS, BLOCK_COLS), np.uint32)
    b = 0
    for rb in range(d.N // BLOCK_ROWS):
        nb = int(blk_ptr[rb + 1] - blk_ptr[rb])
        for r in range(BLOCK_ROWS):
            row = rb * BLOCK_ROWS + r
            codes = d.qr[d.row_ptr[row]:d.row_ptr[row + 1]].astype(np.int16) + 8
            tiles[b:b + nb, r, :] = codes.reshape(nb, BLOCK_COLS).astype(np.uint32)
        b += nb
    t = tiles.reshape(nblk, BLOCK_ROWS, BLOCK_COLS // 8, 8)
    blk_q = np.zeros((nblk, BLOCK_ROWS, BLOCK_COLS // 8), np.uint32)
    for j in range(8):
        blk_q |= t[:, :, :, PI[j]] << np.uint32(4 * j)
    return dict(blk_ptr=blk_ptr, blk_col=blk_col, blk_q=blk_q)


def unpack_blocks(p: dict, N: int, K: int):
    """P4 -> the residual's CSR codes (row_ptr int64 [N+1], col int64, qr
    int8), rows ordered by block, columns ascending: the inverse of
    pack_blocks for the residual codes."""
    blk_ptr = np.asarray(p["blk_ptr"], np.int64)
    blk_col = np.asarray(p["blk_col"], np.int64)
    q = np.asarray(p["blk_q"], np.uint32).reshape(-1, BLOCK_ROWS, BLOCK_COLS // 8)
    u = np.zeros((q.shape[0], BLOCK_ROWS, BLOCK_COLS // 8, 8), np.int16)
    for j in range(8):
        u[:, :, :, PI[j]] = ((q >> np.uint32(4 * j)) & np.uint32(0xF)).astype(np.int16)
    u = u.reshape(-1, BLOCK_ROWS, BLOCK_COLS) - 8
    row_ptr, cols, qrs = [0], [], []
    for rb in range(N // BLOCK_ROWS):
        bl = np.arange(blk_ptr[rb], blk_ptr[rb + 1])
        for r in range(BLOCK_ROWS):
            c = (blk_col[bl][:, None] * BLOCK_COLS + np.arange(BLOCK_COLS)[None, :]).reshape(-1)
            cols.append(c)
            qrs.append(u[bl, r, :].reshape(-1))
            row_ptr.append(row_ptr[-1] + c.size)
    col = np.concatenate(cols) if cols else np.zeros(0, np.int64)
    qr = np.concatenate(qrs) if qrs else np.zeros(0, np.int16)
    return np.asarray(row_ptr, np.int64), col.astype(np.int64), qr.astype(np.int8)
