"""Worker for tests/test_dist_replicas.py: the bench's replica plumbing on
gloo (CPU). Each rank reports a rank-dependent time; every rank must see the
same maximum and the whole-job throughput computed from it."""

import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import bench  # noqa: E402


def main():
    ctx = bench.DistCtx(torch, backend="gloo", timeout_s=60)
    ctx.barrier()
    ms = 10.0 + 5.0 * ctx.rank          # the slower rank decides
    worst = ctx.max(ms)
    value = bench.job_throughput(1_000_000, 100, ctx.world, worst)
    ctx.barrier()
    print(json.dumps({"rank": ctx.rank, "world": ctx.world, "max_ms": worst, "value": value}),
          flush=True)
    ctx.close()


if __name__ == "__main__":
    main()
