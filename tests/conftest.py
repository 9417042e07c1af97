import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(ROOT, "tests", "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA GPU (B200, sm_100a)")
    config.addinivalue_line("markers", "slow: long-running CPU test")


def read_golden(name):
    """Parse a 'key: values' text fixture under tests/golden/."""
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            k, v = line.split(":", 1)
            out[k.strip()] = v.split()
    return out


@pytest.fixture
def golden():
    return read_golden


@pytest.fixture(scope="session")
def mq():
    """The ctypes binding, building libmosaicq.so first if it is stale."""
    from bit_gemm_w4_b200 import build
    build.build()
    from bit_gemm_w4_b200 import mosaicq
    return mosaicq


@pytest.fixture(scope="session")
def cuda(mq):
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")
