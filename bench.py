"""Benchmark of the fused W4 + sparse-residual linear on B200.

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over one batch: the 7B-shaped decode
workload (one token through q/k/v/o 4096x4096, gate/up 11008x4096 and down
4096x11008 linears, rho = 0.5 %), i.e. three fused launches. The metric is
the decode HBM throughput in TB/s of algorithmic bytes (each packed array, X
and Y once). Weights rotate through enough independent packed copies that
every step reads them from HBM, not L2.

Every rank (one per GPU under torchrun) runs the same workload on its own GPU
(independent replicas, weak scaling): the layer has no exchange step, so there
is no data-path collective. Rank 0 prints one JSON line.

Also reported (secondary): the 70B-MLP batched decode (M = 16) in TB/s and
the prefill (M = 2048) in TFLOP/s, each with its roofline fraction.

python bench.py --overhead [--reps R] measures the residual's cost, fused and
unfused, against density 0.

python bench.py --profile-case NAME [--reps R] runs one small case of the hot
path a few times and prints its launch time (the command ncu captures use).

--impl reference times the fp64 CPU oracle on a bounded row sample of the
same workload (rank 0 only) and prints the same JSON line with
"impl": "reference".
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused W4+residual linear: decode HBM TB/s, prefill TFLOP/s, % of roofline"
WORKLOAD = ("7B-shaped decode, M=1: q/k/v/o 4096x4096, gate/up 11008x4096, down 4096x11008; "
            "int4 g128 base + 0.5% int4 CSR residual; bf16 X with 4 channels x20")
SPEC_HBM_GBS = 8000.0  # B200 HBM3e specification figure (context denominator)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def alg_bytes(M: int, N: int, K: int, nnz: int) -> int:
    """Algorithmic bytes of one product: packed base, scale/zero words, CSR
    (row_ptr, col, val, rscale), X and Y, each once."""
    return (N * K // 2 + 4 * N * (K // 128) + 4 * (N + 1) + 2 * nnz + (nnz + 1) // 2 + 2 * N
            + 2 * M * K + 2 * M * N)


# DRAM bytes (read + write) of one launch of the streaming decode kernel per
# 7B shape (M = 1, density 0.5 %), each from one ncu capture of that shape
# (profiles/decode_stream_kernel_7b_m1.txt gives the commands). Set to None
# when the kernel changes until it is captured again.
DECODE_TRAFFIC = {(4096, 4096): 9.193728e6, (11008, 4096): 24.641024e6,
                  (4096, 11008): 24.639488e6}

# DRAM bytes (read + write) of one launch of the tall-layer decode kernel on
# the 70B MLP shape (M = 16, density 1 %), from one ncu capture
# (profiles/decode_tall_kernel_70b_m16.txt). None when the kernel changes.
TALL_TRAFFIC = 130.875648e6 + 3.997696e6


def alg_flops(M: int, N: int, K: int, nnz: int) -> int:
    return 2 * M * N * K + 2 * M * nnz


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the GPU is loaded."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ our arm
class DecodeSet:
    """Packed copies of one workload's shapes plus device X / Y buffers."""

    def __init__(self, mq, torch, name: str, copies: int, dev):
        from bit_gemm_w4_b200 import synth
        cfg = synth.WORKLOADS[name]
        self.M = cfg["M"]
        self.shapes = cfg["shapes"]
        self.weights = []     # [copy][shape]
        self.nnz = []
        for c in range(copies):
            row = []
            for i, (N, K) in enumerate(self.shapes):
                W = synth.weight(N, K, std=cfg["w_std"], outlier_frac=cfg["w_outlier_frac"],
                                 outlier_cols=cfg["w_outlier_cols"], seed=1000 * (i + 1) + 17 * c)
                w = mq.Weight.pack(W, cfg["rho"])
                row.append(w)
                if c == 0:
                    self.nnz.append(w.info()["nnz"])
                del W
            self.weights.append(row)
        self.X = []
        self.Y = []
        for i, (N, K) in enumerate(self.shapes):
            X = synth.activations(self.M, K, seed=7 + i, channels=cfg["x_channels"],
                                  mult=cfg["x_mult"])
            self.X.append(X.to(dev))
            self.Y.append(torch.empty((self.M, N), dtype=torch.bfloat16, device=dev))
        self.bytes_per_launch = [alg_bytes(self.M, N, K, nz)
                                 for (N, K), nz in zip(self.shapes, self.nnz)]
        self.flops_per_launch = [alg_flops(self.M, N, K, nz)
                                 for (N, K), nz in zip(self.shapes, self.nnz)]

    def launch(self, copy: int, i: int, stream, prefetch: bool = False):
        """One layer of the step. With prefetch, mq_linear_prefetch brings the
        next layer's packed weight (the next shape, or the first shape of the
        next step's copy) into L2 while this one runs."""
        w = self.weights[copy][i]
        nxt = None
        if prefetch:
            nsh = len(self.shapes)
            nxt = (self.weights[copy][i + 1] if i + 1 < nsh
                   else self.weights[(copy + 1) % len(self.weights)][0])
        w.linear_raw(self.X[i].data_ptr(), self.M, self.Y[i].data_ptr(), stream=stream,
                     next_weight=nxt)


def time_graph_steps(torch, ds: DecodeSet, steps: int, warmup: int, stream, chunk: int,
                     dist_ctx, sampler_gpu: int):
    """Capture `chunk` steps (rotating weight copies) in a CUDA graph and
    replay it to cover exactly `steps` steps between two events. Nothing but
    the fused launches sits inside the graph, so programmatic dependent
    launch overlaps each launch's weight stream with the previous one's
    tail. Returns total ms (max over ranks) and the clock summary."""
    copies = len(ds.weights)
    nsh = len(ds.shapes)
    for s in range(warmup):
        for i in range(nsh):
            ds.launch(s % copies, i, stream)
    torch.cuda.synchronize()

    def capture(nsteps):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for s in range(nsteps):
                for i in range(nsh):
                    ds.launch(s % copies, i, stream)
        return g

    full, rem = divmod(steps, chunk)
    g = capture(chunk) if full else None
    g_rem = capture(rem) if rem else None
    # settle clocks under the same load before the timed region
    t_end = time.time() + 0.5
    # CUDAGraph.replay() launches on the current stream: make it `stream`
    with ClockSampler(sampler_gpu) as clk, torch.cuda.stream(stream):
        while time.time() < t_end:
            (g or g_rem).replay()
        torch.cuda.synchronize()
        dist_ctx.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(full):
            g.replay()
        if rem:
            g_rem.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dist_ctx.barrier()
    return dist_ctx.max(e0.elapsed_time(e1)), clk.summary()


def time_per_shape(torch, ds: DecodeSet, stream, n: int = 48):
    """Average device time of one launch of each shape: a graph of n
    back-to-back launches (rotating copies, so weights come from HBM)."""
    copies = len(ds.weights)
    out = []
    for i in range(len(ds.shapes)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(n):
                ds.launch(k % copies, i, stream)
        with torch.cuda.stream(stream):
            g.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(5):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        out.append(e0.elapsed_time(e1) / (5 * n))
    return out


def time_e2e(torch, ds: DecodeSet, steps: int, stream, dist_ctx):
    """The public API with host buffers, as a serving loop runs it: every
    step copies its inputs (the three layers' X, packed in one pinned
    buffer) host to device, makes the fused calls, and copies the three
    outputs device to host into pinned memory. Inputs and outputs are
    double-buffered and the copies run on their own streams, ordered by
    events: step s+1's upload and step s-1's download run while step s
    computes, and no buffer is overwritten before its last reader is done.
    The steps are captured once in a CUDA graph and replayed."""
    copies = len(ds.weights)
    dev = ds.X[0].device
    # each layer's slice starts 16-byte aligned (8 bf16 elements)
    xs = [(x.numel() + 7) // 8 * 8 for x in ds.X]
    ys = [(y.numel() + 7) // 8 * 8 for y in ds.Y]
    xo = np.concatenate([[0], np.cumsum(xs)]).astype(int)
    yo = np.concatenate([[0], np.cumsum(ys)]).astype(int)
    hx = [torch.zeros(int(xo[-1]), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for b in range(2):
        for i, x in enumerate(ds.X):
            hx[b][xo[i]:xo[i] + x.numel()] = x.reshape(-1).cpu()
    hy = [torch.empty(int(yo[-1]), dtype=torch.bfloat16, pin_memory=True) for _ in range(2)]
    dx = [torch.empty(int(xo[-1]), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    dy = [torch.empty(int(yo[-1]), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    h2d, d2h = hx[0].numel() * 2, hy[0].numel() * 2
    nsh = len(ds.shapes)
    up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)

    def run(n):
        """Enqueue n steps: upload(s + 1) and download(s - 1) beside compute(s)."""
        ev_up = [torch.cuda.Event() for _ in range(n)]
        ev_cp = [torch.cuda.Event() for _ in range(n)]
        ev_dn = [torch.cuda.Event() for _ in range(n)]
        start = torch.cuda.Event()
        start.record(stream)
        up.wait_event(start)
        down.wait_event(start)

        def upload(s):
            with torch.cuda.stream(up):
                if s >= 2:
                    up.wait_event(ev_cp[s - 2])      # dx[s % 2] last read by compute(s - 2)
                dx[s % 2].copy_(hx[s % 2], non_blocking=True)
                ev_up[s].record(up)

        upload(0)
        for s in range(n):
            stream.wait_event(ev_up[s])
            if s >= 2:
                stream.wait_event(ev_dn[s - 2])      # dy[s % 2] last read by download(s - 2)
            for i in range(nsh):
                ds.weights[s % copies][i].linear_raw(dx[s % 2][xo[i]:].data_ptr(), ds.M,
                                                     dy[s % 2][yo[i]:].data_ptr(), stream=stream)
            ev_cp[s].record(stream)
            if s + 1 < n:
                upload(s + 1)
            with torch.cuda.stream(down):
                down.wait_event(ev_cp[s])
                hy[s % 2].copy_(dy[s % 2], non_blocking=True)
                ev_dn[s].record(down)
        stream.wait_stream(up)
        stream.wait_stream(down)

    with torch.cuda.stream(stream):
        run(3)
        torch.cuda.synchronize()
    chunk = min(steps, copies * 4)
    full, rem = divmod(steps, chunk)

    def capture(n):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            run(n)
        return g

    g = capture(chunk) if full else None
    g_rem = capture(rem) if rem else None
    with torch.cuda.stream(stream):
        (g or g_rem).replay()
        torch.cuda.synchronize()
        dist_ctx.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(full):
            g.replay()
        if rem:
            g_rem.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        dist_ctx.barrier()
    return dist_ctx.max(e0.elapsed_time(e1)), h2d, d2h


def time_read_ceiling(torch, mq, ds: DecodeSet, steps: int, stream, chunk: int) -> float:
    """The attainable read ceiling for the step's chain of launches: the
    library's streaming-read probe (mq_read_probe) over buffers of exactly
    the step's per-launch algorithmic bytes, rotated like the weights,
    captured in a CUDA graph and replayed like the step. Returns GB/s of the
    step's bytes."""
    dev = ds.X[0].device
    copies = len(ds.weights)
    sizes = [(b + 15) // 16 * 16 for b in ds.bytes_per_launch]
    bufs = [[torch.ones(sz, dtype=torch.uint8, device=dev) for sz in sizes] for _ in range(copies)]
    sink = torch.zeros(1, dtype=torch.int32, device=dev)

    def step(c):
        for i, sz in enumerate(sizes):
            mq.read_probe(bufs[c % copies][i].data_ptr(), sz, sink.data_ptr(), stream=stream)

    with torch.cuda.stream(stream):
        for c in range(3):
            step(c)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in range(chunk):
            step(c)
    reps = max(1, steps // chunk)
    with torch.cuda.stream(stream):
        g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    del g, bufs
    return sum(sizes) * reps * chunk / (ms * 1e-3) / 1e9


def time_w16a16(torch, shapes, M: int, steps: int, stream, l2_bytes: int) -> float:
    """The W16A16 analog: torch.matmul in bf16 (cuBLAS) on dense weights of
    the same shapes, the step's products captured in a CUDA graph over
    enough rotating weight copies that each is read from HBM. Returns ms per
    step."""
    dev = torch.device("cuda", torch.cuda.current_device())
    per_copy = sum(2 * N * K for N, K in shapes)
    copies = max(2, int(np.ceil(2.0 * l2_bytes / per_copy)) + 1)
    gen = torch.Generator(device=dev).manual_seed(5)
    Ws = [[torch.randn(N, K, generator=gen, device=dev).to(torch.bfloat16) for N, K in shapes]
          for _ in range(copies)]
    Xs = [torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16) for _, K in shapes]
    Ys = [torch.empty(M, N, dtype=torch.bfloat16, device=dev) for N, _ in shapes]

    def step(c):
        for i in range(len(shapes)):
            torch.matmul(Xs[i], Ws[c % copies][i].t(), out=Ys[i])

    chunk = min(steps, 50)
    with torch.cuda.stream(stream):
        for c in range(3):
            step(c)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for c in range(chunk):
                step(c)
        g.replay()
        torch.cuda.synchronize()
        reps = max(1, steps // chunk)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / (reps * chunk)
    del g, Ws
    return ms


class DistCtx:
    """The replicas' plumbing: one process per GPU (RANK / LOCAL_RANK /
    WORLD_SIZE from the launcher), a barrier around the timed region and the
    maximum of the ranks' times. No data-path collective exists: the ranks
    run independent replicas. backend "gloo" runs the same plumbing on CPU."""

    def __init__(self, torch, backend: str = "nccl", timeout_s: int = 120):
        self.torch = torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.device = "cuda" if backend == "nccl" else "cpu"
        self.pg = None
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                torch.cuda.set_device(self.local)
                kw["device_id"] = torch.device("cuda", self.local)
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = dist

    def barrier(self):
        if self.pg:
            self.pg.barrier()

    def max(self, v: float) -> float:
        if not self.pg:
            return v
        t = self.torch.tensor([v], dtype=self.torch.float64, device=self.device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg:
            self.pg.destroy_process_group()


def job_throughput(step_bytes: int, steps: int, world: int, ms_max: float) -> float:
    """Whole-job TB/s: the bytes every replica processed over the slowest
    rank's time (weak scaling: each rank runs the full step)."""
    return step_bytes * steps * world / (ms_max * 1e-3) / 1e12


def secondary(torch, mq, dev, stream, pk, which: str, reps: int):
    """One secondary workload, device time per launch.

    Decode (the 70B MLP at M = 16): back-to-back launches replayed from a
    CUDA graph, rotating over three packed copies of the weight (396 MB, a
    copy's reuse distance twice the L2), as the primary line times its step. Prefill: single
    launches after an L2 flush (median of `reps`); each launch re-reads its
    weight per token tile, so L2 matters little there."""
    from bit_gemm_w4_b200 import synth
    decode = which != "prefill"
    copies = 3 if decode else 1
    ds = DecodeSet(mq, torch, which, copies, dev)
    N, K = ds.shapes[0]
    for c in range(copies):
        ds.launch(c, 0, stream)
    torch.cuda.synchronize()
    if decode:
        n = 24
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for k in range(n):
                ds.launch(k % copies, 0, stream)
        with torch.cuda.stream(stream):
            g.replay()
            torch.cuda.synchronize()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(reps):
                g.replay()
            e1.record(stream)
            torch.cuda.synchronize()
        ms = e0.elapsed_time(e1) / (reps * n)
        timing = f"CUDA graph of {n} launches over {copies} weight copies, {reps} replays"
        del g
    else:
        flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
        times = []
        for _ in range(reps):
            flush.zero_()                      # evict L2 between launches
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            ds.launch(0, 0, stream)
            b.record(stream)
            torch.cuda.synchronize()
            times.append(a.elapsed_time(b))
        ms = statistics.median(times)
        timing = f"single launches after a 256 MiB L2 flush, median of {reps}"
        del flush
    by, fl = ds.bytes_per_launch[0], ds.flops_per_launch[0]
    out = {"workload": which, "M": ds.M, "N": N, "K": K, "nnz": ds.nnz[0], "ms": ms,
           "kernel": "decode_tall_kernel" if decode else "prefill_kernel",
           "TB_s": by / ms / 1e9, "TFLOP_s": fl / ms / 1e9, "timing": timing}
    if which == "prefill":
        peak = pk["bf16_tflops"]
        out["roofline"] = {"bound": "tensor", "achieved": fl / ms / 1e9, "peak": peak,
                           "unit": "TFLOP/s", "frac": fl / ms / 1e9 / peak}
    else:
        peak = pk["hbm_gbs"]
        out["roofline"] = {"bound": "hbm", "achieved": by / ms / 1e6, "peak": peak,
                           "unit": "GB/s", "frac": by / ms / 1e6 / peak,
                           "traffic": TALL_TRAFFIC}
    del ds
    return out


def run_ours(args):
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq
    dist_ctx = DistCtx(torch)
    dev = torch.device("cuda", dist_ctx.local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    pk, pk_src = peaks()
    # enough copies that consecutive reuse of one copy is > 2x L2 apart
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    per_copy = sum(alg_bytes(1, N, K, 0) for N, K in [(4096, 4096), (11008, 4096), (4096, 11008)])
    copies = max(2, int(np.ceil(2.0 * l2 / per_copy)) + 1)
    ds = DecodeSet(mq, torch, "7b_decode", copies, dev)
    chunk = min(args.steps, 100)
    ms, clocks = time_graph_steps(torch, ds, args.steps, args.warmup, stream, chunk,
                                  dist_ctx, dist_ctx.local)
    per_shape = time_per_shape(torch, ds, stream)
    step_bytes = sum(ds.bytes_per_launch)
    value = job_throughput(step_bytes, args.steps, dist_ctx.world, ms)
    e2e_steps = min(args.steps, 500)
    ms_e2e, h2d, d2h = time_e2e(torch, ds, e2e_steps, stream, dist_ctx)
    e2e = job_throughput(step_bytes, e2e_steps, dist_ctx.world, ms_e2e)
    # the fused decode kernel is the only kernel of a step: its achieved
    # bandwidth is the step's algorithmic bytes over the step's device time
    achieved = step_bytes * args.steps / (ms * 1e-3) / 1e9
    read_ceiling = time_read_ceiling(torch, mq, ds, min(args.steps, 500), stream, chunk)
    w16_ms = time_w16a16(torch, ds.shapes, ds.M, min(args.steps, 500), stream, l2)
    result = {
        "metric": METRIC, "value": round(value, 4), "unit": "TB/s", "n_gpus": dist_ctx.world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": WORKLOAD, "M": 1,
                   "shapes_NxK": [list(s) for s in ds.shapes], "rho": 0.005,
                   "alg_bytes_per_step": step_bytes,
                   "l2": f"inputs larger than L2: {copies} rotating weight copies "
                         f"({copies * step_bytes / 1e6:.0f} MB) vs L2 {l2 / 1e6:.0f} MB",
                   "parallelism": f"replicas x{dist_ctx.world}", "timing": "CUDA graph replay"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": round(achieved / pk["hbm_gbs"], 4),
                     "traffic": (None if DECODE_TRAFFIC is None else
                                 round(sum(DECODE_TRAFFIC[(N, K)]
                                           for N, K in ds.shapes))),
                     "traffic_note": "DRAM bytes per step (3 launches): the sum of one ncu "
                                     "capture of each shape's launch",
                     "peak_source": pk_src,
                     "spec_gbs": SPEC_HBM_GBS,
                     "frac_of_spec": round(achieved / SPEC_HBM_GBS, 4),
                     "read_ceiling_gbs": round(read_ceiling, 1),
                     "frac_of_read_ceiling": round(achieved / read_ceiling, 4),
                     "read_ceiling_note": "mq_read_probe over the step's three per-launch byte "
                                          "counts, rotated and replayed like the step",
                     "kernel": "decode_stream_kernel (the step's three launches)",
                     "per_shape_us": {f"{N}x{K}": round(t * 1e3, 3)
                                      for (N, K), t in zip(ds.shapes, per_shape)},
                     "per_shape_frac": {f"{N}x{K}": round(b / (t * 1e-3) / 1e9 / pk["hbm_gbs"], 4)
                                        for (N, K), t, b in zip(ds.shapes, per_shape,
                                                                ds.bytes_per_launch)}},
        "e2e": {"value": round(e2e, 4), "unit": "TB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "how": "mq_linear per layer with host buffers: each step's X uploaded from pinned "
                       "memory and its Y downloaded to pinned memory, double-buffered, the copies "
                       "on their own streams beside the previous/next step's compute; CUDA graph"},
        "gpu_launches": args.steps * len(ds.shapes),
        "w16a16_context": {"ms_per_step": round(w16_ms, 5),
                           "speedup_vs_w16a16": round(w16_ms / (ms / args.steps), 3),
                           "how": "torch.matmul bf16 (cuBLAS) on dense weights of the same three "
                                  "shapes, CUDA graph over rotating copies",
                           "pages": "up to 1.24x over W16A16, W4A4 end to end on an RTX 4090"},
        "clocks": clocks,
    }
    del ds
    torch.cuda.empty_cache()
    if not args.no_secondary:
        sec = []
        for which in ("70b_mlp", "prefill"):
            try:
                sec.append(secondary(torch, mq, dev, stream, pk, which, reps=10))
            except Exception as e:  # report, never hide
                sec.append({"workload": which, "error": str(e)})
            torch.cuda.empty_cache()
        result["secondary"] = sec
    if dist_ctx.rank == 0 and not args.skip_cpu_baseline and dist_ctx.world == 1:
        result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_seconds)
    if dist_ctx.rank == 0:
        print(json.dumps(result), flush=True)
    dist_ctx.close()


# ------------------------------------------------------------------ oracle arm
def _oracle_sample(rows_per_shape: int):
    """Row samples of the 7B decode workload decomposed by the oracle."""
    import oracle
    from bit_gemm_w4_b200 import synth
    cfg = synth.WORKLOADS["7b_decode"]
    parts = []
    for i, (N, K) in enumerate(cfg["shapes"]):
        rows = np.linspace(0, N - 1, rows_per_shape).astype(np.int64)
        W, X, rho = synth.workload_inputs("7b_decode", i, rows=rows)
        d = oracle.decompose(W, rho)
        parts.append((X, d, alg_bytes(1, rows_per_shape, K, d.nnz)))
    return parts


def cpu_baseline(budget_s: float = 10.0, rows_per_shape: int = 512):
    import oracle
    parts = _oracle_sample(rows_per_shape)
    byts = sum(p[2] for p in parts)
    t0 = time.perf_counter()
    n = 0
    while True:
        for X, d, _ in parts:
            oracle.linear(X, d)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": byts * n / dt / 1e12, "unit": "TB/s", "cores": len(os.sched_getaffinity(0)),
            "kind": "oracle",
            "sample": f"{rows_per_shape} rows of each of the 3 shapes (M=1), {n} passes in {dt:.1f} s"}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    rows = 64
    parts = _oracle_sample(rows)
    byts = sum(p[2] for p in parts)
    for _ in range(args.warmup):
        for X, d, _ in parts:
            oracle.linear(X, d)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        for X, d, _ in parts:
            oracle.linear(X, d)
    dt = time.perf_counter() - t0
    value = byts * args.steps / dt / 1e12
    cores = len(os.sched_getaffinity(0))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no model weights)",
        "config": {"workload": WORKLOAD, "M": 1, "sample": f"{rows} rows of each shape"},
        "cpu_baseline": {"value": value, "unit": "TB/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} rows of each of the 3 shapes per step"},
        "e2e": {"value": value, "unit": "TB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ profile cases
PROFILE_CASES = {
    # name: (N, K, M, rho, path)
    "decode-4096x4096-m1": (4096, 4096, 1, 0.005, "auto"),
    "decode-11008x4096-m1": (11008, 4096, 1, 0.005, "auto"),
    "decode-4096x11008-m1": (4096, 11008, 1, 0.005, "auto"),
    "decode-28672x8192-m16": (28672, 8192, 16, 0.01, "auto"),
    "prefill-14336x4096-m256": (14336, 4096, 256, 0.005, "prefill"),
    "prefill-14336x4096-m2048": (14336, 4096, 2048, 0.005, "prefill"),
    "prefill-14336x4096-m2048-dense": (14336, 4096, 2048, 0.0, "prefill"),
    "prefill-w4a4-14336x4096-m2048": (14336, 4096, 2048, 0.005, "w4a4"),
}


def run_profile_case(name: str, reps: int):
    """One small case of the hot path, a few timed launches (CUDA events,
    L2 flushed before each): the command the ncu summaries are taken with.
    Prints one JSON line with the median launch time; not a bench line."""
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq, synth
    N, K, M, rho, path = PROFILE_CASES[name]
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=1)
    w = mq.Weight.pack(W, rho)
    X = synth.activations(M, K, seed=2, channels=8, mult=30.0).to(dev)
    ws = None
    if path == "w4a4":  # activation quantization, then the fused W4A4 pass
        ws = torch.empty(int(mq._lib.mq_w4a4_workspace_bytes(w._h, M)), dtype=torch.uint8, device=dev)
        Y = w.linear_w4a4(X, workspace=ws)
    else:
        Y = w.linear(X, path=path)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    ts = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if ws is not None:
            w.linear_w4a4(X, Y, ws)
        else:
            w.linear(X, Y, path=path)
        b.record()
        torch.cuda.synchronize()
        ts.append(a.elapsed_time(b) * 1e3)
    if w.device_error() != 0:
        raise RuntimeError("device error word set")
    nnz = w.info()["nnz"]
    t = statistics.median(ts)
    print(json.dumps({"profile_case": name, "N": N, "K": K, "M": M, "rho": rho, "path": path,
                      "us": round(t, 2), "TB_s": round(alg_bytes(M, N, K, nnz) / t / 1e6, 3),
                      "TFLOP_s": round(alg_flops(M, N, K, nnz) / t / 1e6, 1)}))


# ------------------------------------------------------------------ residual overhead
def run_overhead(reps: int):
    """The cost of the residual, fused and unfused: each shape packed at
    several densities from the same weight; every launch timed with CUDA
    events after an L2 flush (median of reps). Reports, per shape and density,
    the fused time, the unfused (dense kernel + separate residual kernel) time
    and the fused overhead over density 0 (MosaicQuant, "Experimental Results":
    the fused sparse branches' latency overhead). Prints one JSON line."""
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq, synth
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    flush = torch.empty(256 * 2**20, dtype=torch.uint8, device=dev)
    cases = [("qkvo", 4096, 4096, 1), ("gateup", 11008, 4096, 1), ("down", 4096, 11008, 1),
             ("qkvo", 4096, 4096, 16), ("prefill", 14336, 4096, 2048)]
    rhos = (0.0, 0.0025, 0.005, 0.01, 0.04)

    def timed(fn):
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    rows = []
    # row mode at each density, then block mode ("Methodology" 2) at each
    # fraction of 16 x 64 blocks (weights: the squared calibration activations)
    variants = [("row", r) for r in rhos] + [("block", f) for f in (0.025, 0.05, 0.1)]
    for name, N, K, M in cases:
        W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=1)
        X = synth.activations(M, K, seed=2, channels=8, mult=30.0).to(dev)
        Xc = synth.activations(128, K, seed=3, channels=8, mult=30.0).double()
        h = (Xc * Xc).sum(0).float().numpy()
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.empty((M, N), dtype=torch.float32, device=dev)
        base = None
        for mode, rho in variants:
            w = (mq.Weight.pack(W, rho) if mode == "row"
                 else mq.Weight.pack(W, block_fraction=rho, channel_weight=h))
            w.linear(X, Y)
            w.linear_unfused(X, Y, ws)
            torch.cuda.synchronize()
            fused = timed(lambda: w.linear(X, Y))
            unfused = timed(lambda: w.linear_unfused(X, Y, ws))
            if w.device_error() != 0:
                raise RuntimeError("device error word set")
            base = fused if (mode == "row" and rho == 0.0) else base
            rows.append({"shape": name, "N": N, "K": K, "M": M, "mode": mode,
                         "rho" if mode == "row" else "block_fraction": rho,
                         "nnz": w.info()["nnz"], "fused_us": round(fused, 2),
                         "unfused_us": round(unfused, 2),
                         "fused_overhead_vs_rho0": round(fused / base - 1.0, 4),
                         "unfused_over_fused": round(unfused / fused, 3)})
            w.free()
    print(json.dumps({"overhead": rows, "timing": f"CUDA events, L2 flushed, median of {reps}"}))


# ------------------------------------------------------------------ distortion
def run_distortion():
    """Output distortion left by the decomposition, as a fraction of what the
    plain 4-bit base leaves, against the share of weights given a residual:
    block mode with the delta score weighted by calibration activations
    ("Methodology" 2), block mode unweighted, and row mode with the same
    residual entry count. Y comes from the library (bf16), the reference is
    X W^T in fp64; the bf16 rounding floor is reported beside it. Synthetic
    weights and activations (no model weights exist here)."""
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq, synth
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    N, K = 4096, 4096
    W = synth.weight(N, K, std=0.02, outlier_frac=0.005, seed=51)
    # calibration and evaluation tokens of one layer: separate draws that
    # share the layer's outlier channels
    Xc = synth.activations(256, K, seed=52, channels=8, mult=30.0, channel_seed=50)
    Xe = synth.activations(256, K, seed=53, channels=8, mult=30.0, channel_seed=50)
    h = (Xc.double() ** 2).sum(0).float().numpy()
    Xe_d = Xe.to(dev)
    Yref = Xe_d.double() @ torch.from_numpy(W).to(dev).double().T
    floor = float(((Yref.to(torch.bfloat16).double() - Yref) ** 2).sum())

    def dist(w):
        Y = w.linear(Xe_d)
        torch.cuda.synchronize()
        v = float(((Y.double() - Yref) ** 2).sum())
        w.free()
        return v

    d0 = dist(mq.Weight.pack(W, 0.0))
    out = []
    for f in (0.0, 0.025, 0.05, 0.1, 0.2):
        rec = {"fraction": f}
        rec["block_delta_weighted"] = round(dist(mq.Weight.pack(W, block_fraction=f, channel_weight=h)) / d0, 4)
        rec["block_unweighted"] = round(dist(mq.Weight.pack(W, block_fraction=f)) / d0, 4)
        rec["row_topk_same_count"] = round(dist(mq.Weight.pack(W, f)) / d0, 4)
        out.append(rec)
    print(json.dumps({"distortion_left_vs_base": out, "bf16_floor_vs_base": round(floor / d0, 4),
                      "shape": [N, K], "tokens": 256,
                      "data": "synthetic: W ~ N(0,0.02) + 0.5% 0.2*t3 outliers; X ~ N(0,1) with 8 "
                              "channels x30; separate calibration and evaluation draws sharing "
                              "the outlier channels"}))


# ------------------------------------------------------------------ W4A4
def run_w4a4():
    """The W4A4 variant against W4A16 on the same packed weights: the three
    7B decode shapes at M = 1, the 70B MLP at M = 16 and the prefill
    workload at M = 2048. Each path is timed as a CUDA graph of 48
    back-to-back calls, weights rotated through copies larger than L2 (the
    W4A4 call is two launches: quantization, then the fused product). Bytes
    are the algorithmic bytes of the W4A16 call (packed weight, CSR, bf16 X
    and Y once); at M > 16 the line also gives TFLOP/s against the tensor
    peak of the call's MMA kind (bf16 measured; int8 = 2 x the measured bf16
    figure, the nominal dense ratio). Prints one JSON line."""
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq, synth
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)
    pk, _ = peaks()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    rows = []
    for name in ("7b_decode", "70b_mlp", "prefill"):
        cfg = synth.WORKLOADS[name]
        for i, (N, K) in enumerate(cfg["shapes"]):
            per = alg_bytes(cfg["M"], N, K, 0)
            copies = max(1, int(np.ceil(2.0 * l2 / per)) + 1) if per < 2 * l2 else 1
            ws = []
            for c in range(copies):
                W = synth.weight(N, K, std=cfg["w_std"], outlier_frac=cfg["w_outlier_frac"],
                                 outlier_cols=cfg["w_outlier_cols"], seed=1000 * (i + 1) + 17 * c)
                ws.append(mq.Weight.pack(W, cfg["rho"]))
                del W
            M = cfg["M"]
            X = synth.activations(M, K, seed=7 + i, channels=cfg["x_channels"],
                                  mult=cfg["x_mult"]).to(dev)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
            wsp = torch.empty(int(mq._lib.mq_w4a4_workspace_bytes(ws[0]._h, M)), dtype=torch.uint8,
                              device=dev)
            nnz = ws[0].info()["nnz"]
            out = {"shape": f"{N}x{K}", "M": M, "nnz": nnz}
            for path in ("w4a16", "w4a4"):
                def call(k):
                    w = ws[k % copies]
                    if path == "w4a16":
                        w.linear_raw(X.data_ptr(), M, Y.data_ptr(), stream=stream)
                    else:
                        w.linear_w4a4(X, Y, wsp, stream=stream)
                with torch.cuda.stream(stream):
                    for k in range(copies):
                        call(k)
                torch.cuda.synchronize()
                g = torch.cuda.CUDAGraph()
                n = 48
                with torch.cuda.graph(g, stream=stream):
                    for k in range(n):
                        call(k)
                with torch.cuda.stream(stream):
                    g.replay()
                    torch.cuda.synchronize()
                    e0 = torch.cuda.Event(enable_timing=True)
                    e1 = torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    for _ in range(5):
                        g.replay()
                    e1.record(stream)
                    torch.cuda.synchronize()
                us = e0.elapsed_time(e1) * 1e3 / (5 * n)
                by = alg_bytes(M, N, K, nnz)
                out[path] = {"us": round(us, 3), "TB_s": round(by / us / 1e6, 3),
                             "frac": round(by / us / 1e3 / pk["hbm_gbs"], 4)}
                if M > 16:
                    tf = alg_flops(M, N, K, nnz) / us / 1e6
                    peak = pk["bf16_tflops"] * (2.0 if path == "w4a4" else 1.0)
                    out[path].update({"TFLOP_s": round(tf, 1), "tensor_peak_tflops": round(peak, 1),
                                      "tensor_frac": round(tf / peak, 4)})
                del g
            rows.append(out)
            del ws
            torch.cuda.empty_cache()
    print(json.dumps({"w4a4_vs_w4a16": rows, "timing": "CUDA graph of 48 calls, mean over 5 replays",
                      "peak_hbm_gbs": pk["hbm_gbs"]}))


SWEEP_SHAPES = [(4096, 4096), (11008, 4096), (4096, 11008)]
SWEEP_M = [1, 8, 64, 512, 4096]
SWEEP_RHO = [0.0, 0.0025, 0.01, 0.04]


def run_sweep(reps: int):
    """The density sweep: the Llama-7B block linears at every M and residual
    density of the sweep workload, each on a synthetic decomposition drawn
    directly (70 % of a row's residual entries in the 128-column groups of 8
    seeded channels). Every launch is timed alone with CUDA events after a
    256 MiB L2 flush (median of reps), so weights come from HBM; torch.matmul
    in bf16 on a dense weight of the same shape is timed the same way as the
    W16A16 analog. Prints one JSON line with the 60 points."""
    import torch
    from bit_gemm_w4_b200 import mosaicq as mq, synth
    dev = torch.device("cuda:0")
    torch.cuda.set_device(dev)
    pk, pk_src = peaks()
    flush = torch.empty(256 * 2 ** 20, dtype=torch.uint8, device=dev)
    gen = torch.Generator(device=dev).manual_seed(3)

    def timed(fn):
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    points, dense = [], {}
    for N, K in SWEEP_SHAPES:
        Wd = torch.randn(N, K, generator=gen, device=dev).to(torch.bfloat16)
        for M in SWEEP_M:
            X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
            Yd = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            torch.matmul(X, Wd.t(), out=Yd)
            dense[(N, K, M)] = timed(lambda: torch.matmul(X, Wd.t(), out=Yd))
        del Wd
        for rho in SWEEP_RHO:
            k_n = int(np.floor(rho * K + 0.5))
            w = mq.Weight.pack_decomposed(synth.sweep_decomposition(N, K, k_n, seed=N + K + k_n))
            for M in SWEEP_M:
                X = torch.randn(M, K, generator=gen, device=dev).to(torch.bfloat16)
                Y = w.linear(X)
                us = timed(lambda: w.linear(X, Y))
                nnz = N * k_n
                by, fl = alg_bytes(M, N, K, nnz), alg_flops(M, N, K, nnz)
                points.append({
                    "N": N, "K": K, "M": M, "rho": rho, "k_n": k_n, "us": round(us, 2),
                    "TB_s": round(by / us / 1e6, 3), "TFLOP_s": round(fl / us / 1e6, 1),
                    "frac_hbm": round(by / us / 1e3 / pk["hbm_gbs"], 3),
                    "frac_tensor": round(fl / us / 1e6 / pk["bf16_tflops"], 3),
                    "w16a16_us": round(dense[(N, K, M)], 2),
                    "speedup_vs_w16a16": round(dense[(N, K, M)] / us, 2)})
            if w.device_error() != 0:
                raise RuntimeError("device error word set")
            del w
            torch.cuda.empty_cache()
    print(json.dumps({"sweep": points, "timing": f"single launches after a 256 MiB L2 flush, "
                      f"median of {reps}; W16A16: torch.matmul bf16 on a dense weight, same timing",
                      "peaks": {"hbm_gbs": pk["hbm_gbs"], "bf16_tflops": pk["bf16_tflops"],
                                "source": pk_src}}), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-case", choices=sorted(PROFILE_CASES),
                    help="run one small case a few times (the ncu capture command) and exit")
    ap.add_argument("--reps", type=int, default=5)
    ap.add_argument("--distortion", action="store_true",
                    help="measure the output distortion left at each residual share and exit")
    ap.add_argument("--w4a4", action="store_true",
                    help="time the W4A4 variant against W4A16 on the same weights and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="time the 60-point density sweep (and the W16A16 analog) and exit")
    ap.add_argument("--overhead", action="store_true",
                    help="measure the residual's fused and unfused overhead over density 0 and exit")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    args = ap.parse_args(argv)
    if args.profile_case:
        run_profile_case(args.profile_case, args.reps)
        return
    if args.overhead:
        run_overhead(max(args.reps, 5))
        return
    if args.sweep:
        run_sweep(max(args.reps, 5))
        return
    if args.distortion:
        run_distortion()
        return
    if args.w4a4:
        run_w4a4()
        return
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
