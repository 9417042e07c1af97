"""The oracle still reproduces its committed fixture on the tiny workload
(tests/golden/tiny_oracle.txt, written by tests/golden/make_golden.py)."""

import hashlib

import numpy as np

import oracle
from bit_gemm_w4_b200 import synth


def test_tiny_fixture(golden):
    f = golden("tiny_oracle.txt")
    W, X, rho = synth.workload_inputs("tiny")
    d = oracle.decompose(W, rho)
    assert d.nnz == int(f["nnz"][0])
    p = oracle.pack(d)
    for k in ("qweight", "sz", "row_ptr", "col", "val", "rscale"):
        assert hashlib.sha256(np.ascontiguousarray(p[k]).tobytes()).hexdigest() == f["sha256_" + k][0], k
    Y = oracle.linear(X, d)
    # the fp64 matmul's summation order may differ between BLAS builds
    for n, y in zip(f["sample_n"], f["sample_y"]):
        assert abs(Y[0, int(n)] - float(y)) <= 1e-12 * max(1.0, abs(float(y)))
