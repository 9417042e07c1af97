"""The C-ABI library loads on a machine without a GPU and exports every
function include/mosaicq.h declares; host-only calls validate arguments."""

import ctypes
import os
import re

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "mosaicq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mq_[a-z_]+)\s*\(", src)))


def test_every_declared_symbol_is_exported(mq):
    names = _declared()
    assert "mq_pack" in names and "mq_linear" in names and "mq_free" in names
    lib = ctypes.CDLL(mq.LIB_PATH)
    missing = [n for n in names if not hasattr(lib, n)]
    assert not missing, missing


def test_strerror_and_free_null(mq):
    lib = mq.lib()
    assert lib.mq_strerror(0) == b"ok"
    assert lib.mq_strerror(1) == b"invalid argument"
    lib.mq_free(None)  # NULL-safe


def test_residual_nnz(mq):
    assert mq.residual_nnz(4096, 4096, 0.005) == 4096 * 20
    assert mq.residual_nnz(10, 11008, 0.04) == 10 * 440
    assert mq.residual_nnz(3, 128, 0.0) == 0


@pytest.mark.parametrize("N,K,rho,group,status", [
    (4, 100, 0.01, 128, 1),        # K % 128
    (4, 65536 + 128, 0.01, 128, 1),  # K > 65536
    (0, 128, 0.01, 128, 1),        # N = 0
    (4, 128, -0.1, 128, 1),        # rho < 0
    (4, 128, 1.5, 128, 1),         # rho > 1
    (4, 128, 0.01, 64, 2),         # group size
])
def test_shape_errors(mq, N, K, rho, group, status):
    with pytest.raises(mq.MQError) as e:
        mq.residual_nnz(N, K, rho, group)
    assert e.value.status == status


def test_nonfinite_and_overflow_rejected(mq):
    W = np.zeros((2, 128), np.float32)
    W[1, 3] = np.nan
    with pytest.raises(mq.MQError) as e:
        mq.pack_host(W, 0.01)
    assert e.value.status == 1 and "NaN" in str(e.value)
    W[1, 3] = 1e6
    with pytest.raises(mq.MQError) as e:
        mq.pack_host(W, 0.01)
    assert "overflow" in str(e.value)


def test_injected_allocation_failure(mq, monkeypatch):
    # MQ_FAULT_ALLOC=1: packing fails with OUT_OF_MEMORY at its first device
    # allocation, before any CUDA call (so this holds without a GPU too)
    W = np.random.default_rng(0).standard_normal((32, 256)).astype(np.float32) * 0.02
    monkeypatch.setenv("MQ_FAULT_ALLOC", "1")
    with pytest.raises(mq.MQError) as e:
        mq.Weight.pack(W, 0.02, stream=0)      # the default stream: no torch CUDA call
    assert e.value.status == mq.OUT_OF_MEMORY
    assert b"MQ_FAULT_ALLOC" in mq.lib().mq_last_error()


def test_noalloc_capacity_constant_matches_header():
    import re
    from bit_gemm_w4_b200 import mosaicq as mq
    hdr = open(os.path.join(ROOT, "include", "mosaicq.h")).read()
    m = re.search(r"#define MQ_UNFUSED_NOALLOC_MAX_OUTPUTS \(([^)]*)\)", hdr)
    assert m and eval(m.group(1), {}) == mq.UNFUSED_NOALLOC_MAX_OUTPUTS
