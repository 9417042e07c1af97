"""Write tests/golden/tiny_oracle.txt from the oracle alone.

Run from the repository root: python tests/golden/make_golden.py
It calls only oracle/ and the seeded generators; nothing here touches the
CUDA library. The fixture pins the oracle's decomposition, packed bytes and
product on the tiny workload (one 512x512 layer, 1 token, rho = 1 %) so that
any later change to the oracle's arithmetic shows up as a diff.
"""

import hashlib
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from bit_gemm_w4_b200 import synth  # noqa: E402

SAMPLE = [0, 1, 7, 63, 128, 255, 300, 511]


def main():
    W, X, rho = synth.workload_inputs("tiny")
    d = oracle.decompose(W, rho)
    p = oracle.pack(d)
    Y = oracle.linear(X, d)
    lines = [
        "# Oracle regression fixture: the tiny workload (512x512 weights ~N(0,0.02)",
        "# with 1 % 0.2*t(3) outliers, one N(0,1) bf16 token, rho = 1 %).",
        "# Decomposition and product per MosaicQuant 'Methodology' 1. (W ~= Q(W) + R,",
        "# both 4-bit) and 3. (dense GEMM + sparse residual, reduction-add).",
        "# Written by tests/golden/make_golden.py from oracle/ only.",
        f"nnz: {d.nnz}",
    ]
    for k in ("qweight", "sz", "row_ptr", "col", "val", "rscale"):
        lines.append(f"sha256_{k}: {hashlib.sha256(np.ascontiguousarray(p[k]).tobytes()).hexdigest()}")
    lines.append("sample_n: " + " ".join(str(n) for n in SAMPLE))
    lines.append("sample_y: " + " ".join(repr(float(Y[0, n])) for n in SAMPLE))
    with open(os.path.join(ROOT, "tests", "golden", "tiny_oracle.txt"), "w") as f:
        f.write("\n".join(lines) + "\n")


if __name__ == "__main__":
    main()
