"""The multi-GPU path is replicas only: each rank runs the whole step, the
ranks meet at barriers and the reported time is the maximum over ranks. This
runs that plumbing with world size 2 on the gloo backend (CPU)."""

import json
import os
import re
import socket
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_take_the_max_time():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "tests", "dist_worker.py")]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=180, cwd=ROOT,
                         env={**os.environ, "OMP_NUM_THREADS": "1"})
    assert out.returncode == 0, out.stderr[-2000:]
    # the two ranks write to one pipe: take every complete JSON object
    lines = [json.loads(m) for m in re.findall(r"\{[^{}]*\}", out.stdout)]
    assert sorted(l["rank"] for l in lines) == [0, 1]
    for l in lines:
        assert l["world"] == 2 and l["max_ms"] == 15.0
        # 2 replicas x 100 steps x 1 MB in 15 ms
        assert abs(l["value"] - 2 * 100 * 1e6 / 15e-3 / 1e12) < 1e-12
