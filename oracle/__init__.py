"""CPU oracle for the fused W4 + sparse-residual linear (test infrastructure).

A plain, slow, fp64 restatement of what the hot path computes, written from
the MosaicQuant pages:

  * decompose.py - inlier-outlier disaggregation W ~= Q(W) + R: a dense 4-bit
    base and a sparse 4-bit residual that patches the worst-quantized entries
    (MosaicQuant, "Methodology", 1. Inlier-Outlier Disaggregation, the
    equation W_hat ~= Q(W_hat) + R; both parts 4-bit), with the residual
    allocated per row or per block ("Methodology" 2, the Hessian-guided
    delta score).
  * pack.py      - the device byte layout of that decomposition, and unpack;
                   the block-tile layout of a block-allocated residual.
  * linear.py    - the product Y = X * W_hat^T, W_hat = deq(Q) + R, as dense
    base plus a CSR loop (the "reduction-add" of ZipperEngine's pipeline) and
    as a brute-force triple loop.
  * tolerance.py - the parity metrics used to accept a bf16 GPU output.
  * w4a4.py      - the W4A4 variant: per-token int4 activation quantization
    (the pipeline's quantization stage in "Methodology" 3.) and the product
    from exact integer sums ("Experimental Results" evaluate W4A4).

This package is test infrastructure. Only tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline / reference arm may import it. The product path
(bit_gemm_w4_b200) never imports it, and it imports nothing from the product.
Every function is pinned by CPU tests against brute force, closed forms or
library routines (tests/test_oracle_*.py); none is "parity unpinned".
"""

from .decompose import (Decomposition, decompose, from_arrays, fp16_rne,
                        residual_count, quantize_base, select_residual,
                        quantize_residual, decompose_blocks, block_scores,
                        select_blocks, blocks_selected)
from .pack import pack, unpack, block_structure, pack_blocks, unpack_blocks
from .linear import dequant_base, w_hat, linear, linear_brute
from .tolerance import parity_report

__all__ = [
    "Decomposition", "decompose", "from_arrays", "fp16_rne", "residual_count",
    "quantize_base", "select_residual", "quantize_residual", "pack", "unpack",
    "block_structure", "pack_blocks", "unpack_blocks",
    "dequant_base", "w_hat", "linear", "linear_brute", "parity_report",
    "decompose_blocks", "block_scores", "select_blocks", "blocks_selected",
]
