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
