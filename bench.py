#!/usr/bin/env python
"""Benchmark of the Parallax hot path on B200 (one JSON line on rank 0).

Headline workload: single-token decode over a bf16 KV cache, B=32, H_q=16,
H_kv=8, d=128, context 4096 (``decode_b32_ctx4096``).  One step is one
``plx_decode`` call (score, probe score, online softmax, both accumulators,
split merge).  The causal prefill rows of the hot path are measured in the same
run on ``prefill_b8_l4096`` (B=8, L=4096, H_q=16, H_kv=8, d=128) and reported
under ``"prefill"``, the long-context prefill ``prefill_b1_l32768`` (B=1,
L=32768, H_q=32, H_kv=8) under ``"prefill_long"``, the gradients of the prefill
(``plx_prefill_bwd`` on ``prefill_b8_l4096``, 16d flops per visible pair) under
``"prefill_bwd"``, the probe projection rho = x W_R^T at the prefill and the
decode sizes under ``"probe_projection"``, and the decode grid (batch
1-2048 x context 128-32768, ragged lengths) under ``"sweep"``: per cell the
device time per call with L2 flushed before every call, HBM GB/s from the
actual lengths and the fraction of the measured copy bandwidth.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and
a device synchronisation, timed with CUDA events on the launching stream; the
elapsed time is the maximum over ranks.  The KV cache rotates over three
independent copies of 537 MB each (inputs larger than the 126 MB L2), so every
step reads its cache from HBM.

Multi-GPU (torchrun, one process per GPU): the decode batches are independent
problems, so every rank runs its own batch with no data-path collective
("scaling": "weak"); value = all ranks' tokens / max-over-ranks time.

``--impl reference`` times the fp64 CPU oracle instead (on rank 0 only), on the
same workload and metric, one bounded sample of decode rows per step.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s & HBM GB/s (% of roofline); prefill TFLOP/s (% bf16 peak)"
HEADLINE = "decode_b32_ctx4096"
PREFILL = "prefill_b8_l4096"
PREFILL_LONG = "prefill_b1_l32768"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
DECODE_SOURCES = ["plx_decode.cu", "plx_decode.cuh", "plx_device.cuh"]
PREFILL_SOURCES = ["plx_prefill_tc.cu", "plx_device.cuh"]


# --------------------------------------------------------------------------- util
def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def source_digest(names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "covariance_corrected_softmax_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def recorded_traffic(kernel, workload, names):
    """DRAM bytes per launch from profiles/dram_traffic.txt, if taken on the
    current kernel source (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    digest = source_digest(names)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and \
                    parts[1] == workload and parts[3] == digest:
                return float(parts[2])
    return None


def max_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device=device if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def gpu_index() -> int:
    """nvidia-smi index of the current device."""
    import torch
    idx = torch.cuda.current_device()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        try:
            idx = int(vis.split(",")[idx])
        except (ValueError, IndexError):
            pass
    return idx


def aggregate_rate(world: int, units_per_rank: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput: every rank processes units_per_rank units per step,
    the job takes the slowest rank's time (max_ms for all steps)."""
    return world * units_per_rank * steps / (max_ms / 1e3)


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 20 ms around the
    timed region; the summary keeps the samples taken inside it (host clock
    between entering and leaving the `with` block, 0.3 s pre-roll excluded)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 20):
        self.idx = gpu_index
        self.period = period_ms
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period)],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        self.t0 = time.time()
        return self

    def __exit__(self, *exc):
        self.t1 = time.time()
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    @staticmethod
    def _epoch(stamp):
        for fmt in ("%Y/%m/%d %H:%M:%S.%f", "%Y/%m/%d %H:%M:%S"):
            try:
                return datetime.datetime.strptime(stamp, fmt).timestamp()
            except ValueError:
                continue
        return None

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) < 10:
                        continue
                    try:
                        rows.append((self._epoch(p[0]), float(p[2]), float(p[3]), float(p[4]),
                                     p[6:10]))
                    except ValueError:
                        continue
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        window = [r for r in rows if r[0] is not None and self.t0 is not None and
                  self.t0 <= r[0] <= self.t1 + self.period / 1000.0]
        if not window:
            # a region shorter than the sampling period: the first sample after it began
            after = [r for r in rows if r[0] is not None and self.t0 is not None and r[0] >= self.t0]
            window = after[:1] or rows[-1:]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in window for i, v in enumerate(r[4]) if v == "Active"})
        return {"sm_mhz": statistics.median(r[1] for r in window),
                "sm_max_mhz": max(r[2] for r in rows),
                "power_w_max": max(r[3] for r in window), "reasons": reasons,
                "samples": len(window),
                "window_ms": round(1000.0 * (self.t1 - self.t0), 1) if self.t1 else None}


# ------------------------------------------------------------------------ decode
def decode_alg_bytes(shape, seqlens) -> float:
    esz = 2
    kv = float(seqlens.sum().item()) * shape.Hkv * shape.d * esz * 2
    return kv + shape.B * shape.Hq * shape.d * esz * 3


def bench_decode(plx, W, shape, steps, warmup, world, device, rank):
    import torch
    inp = W.make_decode(shape, seed=rank, device=device, copies=3)
    ws = plx.decode_workspace(shape.B, shape.Hq, shape.Hkv, shape.d, shape.S_max, device=device)
    out = torch.empty_like(inp["q"])
    stream = torch.cuda.current_stream()

    def step(i):
        plx.decode(inp["q"], inp["rho"], inp["k_caches"][i % 3], inp["v_caches"][i % 3],
                   inp["seqlens"], softmax_scale=1.0, out=out, workspace=ws, stream=stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index()) as clk:
        s.record(stream)
        for i in range(steps):
            step(warmup + i)
        e.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    local_ms = s.elapsed_time(e)
    total_ms = max_over_ranks(local_ms, world, device)
    assert plx.device_error() == 0, "decode kernels reported a device error"
    return {"ms": total_ms, "alg_bytes": decode_alg_bytes(shape, inp["seqlens"]),
            "clocks": clk.summary(), "inp": inp}


def bench_decode_e2e(plx, W, shape, steps, warmup, world, device, rank):
    """Same metric through the public serving call with host I/O every step: the
    new token's q, rho, k, v and the lengths (which count the new token) are
    packed in one pinned host buffer and copied host -> device; plx_decode_append
    writes k, v into the cache and decodes; out comes back to pinned host
    memory.  As a serving loop would run it, one step is one replay of a CUDA
    graph captured from those calls, with the copies on side branches of the
    graph: step i's graph decodes step i while it uploads step i+1's inputs and
    downloads step i-1's output (double-buffered; every step still moves its own
    inputs and output).  The time runs from the first upload to the last output
    landing in host memory."""
    import torch
    inp = W.make_decode(shape, seed=100 + rank, device=device, copies=3)
    B, Hq, Hkv, d = shape.B, shape.Hq, shape.Hkv, shape.d
    pos = shape.ctx - 1
    parts = [("q", inp["q"]), ("rho", inp["rho"]),
             ("k", inp["k_cache"][:, pos].contiguous()), ("v", inp["v_cache"][:, pos].contiguous()),
             ("sl", inp["seqlens"])]
    offs, off = {}, 0
    for name, t in parts:
        nbytes = t.numel() * t.element_size()
        offs[name] = (off, nbytes, t.dtype, tuple(t.shape))
        off += (nbytes + 255) // 256 * 256
    hbufs, dbufs, outs_h, outs_d, views = [], [], [], [], []
    for _ in range(2):
        hbuf = torch.empty(off, dtype=torch.uint8).pin_memory()
        for name, t in parts:
            o, n, _, _ = offs[name]
            hbuf[o:o + n].copy_(t.contiguous().view(torch.uint8).reshape(-1).cpu())
        dbuf = torch.empty(off, dtype=torch.uint8, device=device)
        hbufs.append(hbuf)
        dbufs.append(dbuf)
        views.append({n_: dbuf[o:o + n].view(dt).view(shp)
                      for n_, (o, n, dt, shp) in offs.items()})
        outs_h.append(torch.empty((B, Hq, d), dtype=inp["q"].dtype).pin_memory())
        outs_d.append(torch.empty_like(inp["q"]))
    ws = plx.decode_workspace(B, Hq, Hkv, d, shape.S_max, device=device)
    cap = torch.cuda.Stream(device=device)
    s_in = torch.cuda.Stream(device=device)
    s_out = torch.cuda.Stream(device=device)

    def serve(pb, c, stream):
        v = views[pb]
        plx.decode_append(v["q"], v["rho"], v["k"], v["v"], inp["k_caches"][c],
                          inp["v_caches"][c], v["sl"], softmax_scale=1.0, out=outs_d[pb],
                          workspace=ws, stream=stream)

    # warm up outside capture (first-call set-up of the library, the allocator)
    cap.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(cap):
        for pb in range(2):
            dbufs[pb].copy_(hbufs[pb], non_blocking=True)
            serve(pb, 0, cap)
            outs_h[pb].copy_(outs_d[pb], non_blocking=True)
    torch.cuda.synchronize()

    graphs = {}
    for pb in range(2):          # parity of the step (which I/O buffers)
        for c in range(3):       # which of the three rotating caches
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cap):
                fork = torch.cuda.Event()
                fork.record(cap)
                s_in.wait_event(fork)
                s_out.wait_event(fork)
                with torch.cuda.stream(s_in):    # the next step's inputs
                    dbufs[1 - pb].copy_(hbufs[1 - pb], non_blocking=True)
                with torch.cuda.stream(s_out):   # the previous step's output
                    outs_h[1 - pb].copy_(outs_d[1 - pb], non_blocking=True)
                serve(pb, c, cap)                # this step
                cap.wait_stream(s_in)
                cap.wait_stream(s_out)
            graphs[(pb, c)] = g
    main = torch.cuda.current_stream()

    def run(n, first):
        dbufs[first % 2].copy_(hbufs[first % 2], non_blocking=True)  # the first step's inputs
        for i in range(first, first + n):
            graphs[(i % 2, i % 3)].replay()
        last = (first + n - 1) % 2
        outs_h[last].copy_(outs_d[last], non_blocking=True)          # the last step's output

    run(warmup, 0)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(main)
    run(steps, warmup)
    e.record(main)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world, device)
    del graphs
    h2d = hbufs[0].numel()
    d2h = outs_h[0].numel() * outs_h[0].element_size()
    return {"ms": ms, "h2d": h2d, "d2h": d2h}


def cpu_baseline_decode(inp, shape, seconds: float = 12.0):
    """The oracle (explicit covariance form) on sampled rows of the same decode
    batch, on all host cores; tokens/s = rows/s / H_q."""
    import numpy as np
    import oracle
    from covariance_corrected_softmax_b200 import workloads as W
    threads = oracle.default_threads()
    q, rho = inp["q"].float().cpu(), inp["rho"].float().cpu()
    kc, vc = inp["k_cache"], inp["v_cache"]
    sl = inp["seqlens"].cpu()
    rows = W.sample_rows_decode(shape.B, shape.Hq, shape.B * shape.Hq, seed=2)
    done, t_used, n = 0, 0.0, max(1, threads)
    while t_used < seconds:
        idx = [(done + j) % len(rows) for j in range(n)]
        t0 = time.perf_counter()
        oracle.decode(q, rho, kc, vc, sl, 1.0, rows=rows[idx], threads=threads)
        t_used += time.perf_counter() - t0
        done += n
        if t_used < seconds / 4:
            n = min(4 * n, len(rows))
    rows_per_s = done / t_used
    return {"value": rows_per_s / shape.Hq, "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{done} (b, h) rows (cycling over all {shape.B * shape.Hq}) of "
                      f"{HEADLINE} (explicit fp64 covariance form), {t_used:.1f} s"}


# ----------------------------------------------------------------------- prefill
def bench_prefill(plx, W, shape, steps, warmup, world, device, rank):
    import torch
    inp = [W.make_prefill(shape, seed=10 + rank + 7 * c, device=device) for c in range(2)]
    out = torch.empty_like(inp[0]["q"])
    lse = torch.empty((shape.B, shape.Hq, shape.L), dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream()

    def step(i):
        x = inp[i % 2]
        plx.prefill(x["q"], x["rho"], x["k"], x["v"], causal=shape.causal, softmax_scale=1.0,
                    out=out, lse=lse, stream=stream)

    try:
        step(0)
    except plx.PlxError as e:
        return {"status": str(e)}
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index()) as clk:
        s.record(stream)
        for i in range(steps):
            step(i)
        e.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world, device)
    assert plx.device_error() == 0, "prefill kernel reported a device error"
    return {"ms": ms, "clocks": clk.summary()}


def bench_prefill_bwd(plx, W, shape, steps, warmup, world, device, rank):
    """plx_prefill_bwd (bf16: the two tensor-core kernels) on the prefill
    workload with a seeded dout; the gradients and the statistics workspace are
    allocated once, outside the timed region."""
    import torch
    x = W.make_prefill(shape, seed=40 + rank, device=device)
    g = torch.Generator(device=device).manual_seed(41 + rank)
    dout = torch.randn(x["q"].shape, generator=g, device=device).to(x["q"].dtype)
    grads = [torch.empty(x[n].shape, dtype=torch.float32, device=device)
             for n in ("q", "rho", "k", "v")]
    ws = torch.empty(plx.prefill_bwd_workspace_bytes(shape.B, shape.L, shape.Hq),
                     dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()

    def step():
        plx.prefill_bwd(x["q"], x["rho"], x["k"], x["v"], dout, causal=shape.causal,
                        softmax_scale=1.0, grads=grads, workspace=ws, stream=stream)

    try:
        step()
    except plx.PlxError as e:
        return {"status": str(e)}
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index()) as clk:
        s.record(stream)
        for _ in range(steps):
            step()
        e.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(s.elapsed_time(e), world, device)
    assert plx.device_error() == 0, "backward kernels reported a device error"
    return {"ms": ms, "clocks": clk.summary()}


def bench_projection(plx, W, peaks, peak_src, device):
    """The probe projection rho = x W_R^T (plx_probe_projection) at the prefill
    workload's size (x [8 * 4096, 2048], W_R [16 * 128, 2048]; tensor-bound:
    2 M N K flops, 20 calls alternating two inputs larger than L2) and at the
    decode workload's (x [32, 2048]: bound by reading W_R, 8.4 MB; each call
    timed alone after the L2 flush and clean-up read, median of 30)."""
    import torch
    res = {}
    M, N, K = 8 * 4096, 16 * 128, 2048
    xs = [W.make_probe_inputs((M,), K, N, seed=50 + c, device=device) for c in range(2)]
    out = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    for i in range(3):
        plx.probe_projection(xs[i % 2][0], xs[i % 2][1], out=out)
    torch.cuda.synchronize()
    steps = 20
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_index()) as clk:
        s.record()
        for i in range(steps):
            plx.probe_projection(xs[i % 2][0], xs[i % 2][1], out=out)
        e.record()
        torch.cuda.synchronize()
    ms = s.elapsed_time(e) / steps
    tflops = 2.0 * M * N * K / (ms / 1e3) / 1e12
    res["prefill"] = {"M": M, "N": N, "K": K, "ms_per_call": ms, "tflops": tflops,
                      "roofline": {"bound": "tensor", "achieved": tflops,
                                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                   "frac": tflops / peaks["bf16_tflops"],
                                   "peak_source": f"{peak_src} bf16 dense (burst)"},
                      "clocks": clk.summary()}
    del xs, out
    M = 32
    x, w = W.make_probe_inputs((M,), K, N, seed=60, device=device)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.zeros(32 << 20, dtype=torch.int64, device=device)
    for _ in range(3):
        plx.probe_projection(x, w, out=out)
    times = []
    for _ in range(30):
        flush.fill_(1)
        clean.sum()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        plx.probe_projection(x, w, out=out)
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    ms = statistics.median(times)
    nbytes = 2.0 * (N * K + M * K + M * N)
    gbs = nbytes / (ms / 1e3) / 1e9
    res["decode"] = {"M": M, "N": N, "K": K, "us_per_call": ms * 1e3, "gbs": gbs,
                     "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": gbs / peaks["hbm_gbs"],
                                  "peak_source": f"{peak_src} HBM copy bandwidth",
                                  "bytes_per_call": nbytes},
                     "launch_bound": nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6 < 20.0}
    assert plx.device_error() == 0, "projection kernels reported a device error"
    del x, w, out, flush, clean
    torch.cuda.empty_cache()
    return res


def prefill_bwd_record(name, pshape, pr, psteps, peaks, peak_src):
    pms = pr["ms"] / psteps
    # 16d flops per visible (query, key) pair: the eight products S, T, GV,
    # dV, dQ, dR and the two of dK, each 2d per pair (recomputation of the row
    # statistics not counted)
    flops = 2.0 * pshape.flops()
    tflops = flops / (pms / 1e3) / 1e12
    return {
        "workload": name, "B": pshape.B, "L": pshape.L, "H_q": pshape.Hq, "H_kv": pshape.Hkv,
        "d": pshape.d, "causal": pshape.causal, "steps": psteps, "ms_per_call": pms,
        "tflops": tflops,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     "peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": tflops / peaks["bf16_tflops_sustained"],
                     "flops_per_call": flops, "traffic": None},
        # the rows kernel (dq, drho, row statistics) and the keys kernel (dk, dv)
        "gpu_launches_per_call": 2,
        "clocks": pr["clocks"],
    }


# ------------------------------------------------------------------ decode grid
def bench_decode_sweep(plx, W, peaks, device, only=None):
    """Every cell of the decode grid (batch x context, ragged lengths U[ctx/2,
    ctx], caches capped under 120e9 bytes).  Each call is timed alone with CUDA
    events, after a 256 MiB buffer (twice the L2) has been written, so every
    call reads its cache from HBM, and a second 256 MiB buffer has been read, so
    that the lines the write left dirty are written back before the timed call
    rather than during it; the median over the calls is reported."""
    import torch
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    clean = torch.zeros(32 << 20, dtype=torch.int64, device=device)  # 256 MiB
    stream = torch.cuda.current_stream()
    cells = []
    for cell in W.sweep_cells():
        if only and f"{cell.B}x{cell.ctx}" not in only:
            continue
        inp = W.make_decode(cell, seed=0, device=device)
        ws = plx.decode_workspace(cell.B, cell.Hq, cell.Hkv, cell.d, cell.S_max, device=device)
        out = torch.empty_like(inp["q"])
        alg = decode_alg_bytes(cell, inp["seqlens"])
        n = 10 if alg > 4e9 else 30

        def call():
            plx.decode(inp["q"], inp["rho"], inp["k_cache"], inp["v_cache"], inp["seqlens"],
                       softmax_scale=1.0, out=out, workspace=ws, stream=stream)

        for _ in range(3):
            call()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n)]
        for s_, e_ in ev:
            flush.fill_(1)
            clean.sum()
            s_.record(stream)
            call()
            e_.record(stream)
        torch.cuda.synchronize()
        ms = statistics.median(s_.elapsed_time(e_) for s_, e_ in ev)
        gbs = alg / (ms / 1e3) / 1e9
        roof_us = alg / (peaks["hbm_gbs"] * 1e9) * 1e6
        cells.append({"B": cell.B, "context": cell.ctx, "mean_len": float(inp["seqlens"].float().mean()),
                      "us_per_call": ms * 1e3, "tokens_per_s": cell.B / (ms / 1e3),
                      "hbm_gbs": gbs, "frac": gbs / peaks["hbm_gbs"], "bytes_per_call": alg,
                      "calls": n, "launch_bound": roof_us < 20.0})
        del inp, ws, out
        torch.cuda.empty_cache()
    assert plx.device_error() == 0, "decode kernels reported a device error in the sweep"
    del flush, clean
    torch.cuda.empty_cache()
    return cells


def prefill_record(name, pshape, pr, psteps, world, peaks, peak_src, traffic):
    pms = pr["ms"] / psteps
    tflops = pshape.flops() / (pms / 1e3) / 1e12
    return {
        "workload": name, "B": pshape.B, "L": pshape.L, "H_q": pshape.Hq,
        "H_kv": pshape.Hkv, "d": pshape.d, "causal": pshape.causal, "steps": psteps,
        "ms_per_call": pms, "tflops": tflops,
        "tokens_per_s": aggregate_rate(world, pshape.B * pshape.L, psteps, pr["ms"]),
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": tflops / peaks["bf16_tflops"],
                     "peak_source": f"{peak_src} bf16 dense (burst)",
                     # the leg runs `psteps` calls back to back (a long loop under
                     # the power cap): the sustained GEMM figure, for comparison
                     "peak_sustained": peaks["bf16_tflops_sustained"],
                     "frac_sustained": tflops / peaks["bf16_tflops_sustained"],
                     "flops_per_call": pshape.flops(), "traffic": traffic},
        # the fast instance and the recomputing one (which returns at once
        # when no unit's V is out of fp16's range)
        "gpu_launches_per_call": 2,
        "clocks": pr["clocks"],
    }


# -------------------------------------------------------------------- reference
def reference_arm(args):
    """The oracle as it stands on the host cores, same workload and metric."""
    rank, _, world = env_rank()
    if rank != 0:
        return 0
    import torch
    import oracle
    from covariance_corrected_softmax_b200 import workloads as W
    shape = W.WORKLOADS[HEADLINE]
    inp = W.make_decode(shape, seed=0, device="cpu")
    threads = oracle.default_threads()
    rows = W.sample_rows_decode(shape.B, shape.Hq, shape.B * shape.Hq, seed=3)
    q, rho = inp["q"].float(), inp["rho"].float()
    # A step is one row per host thread, evaluated in parallel; if K + W such
    # steps would run past ~2.5 minutes, a step is a single row on one thread.
    per_step = threads
    t0 = time.perf_counter()
    oracle.decode(q, rho, inp["k_cache"], inp["v_cache"], inp["seqlens"], 1.0,
                  rows=rows[:per_step], threads=threads)
    step_s = time.perf_counter() - t0
    if (args.steps + args.warmup) * step_s > 150:
        per_step = 1
    used = min(threads, per_step)
    k = 0

    def run_step():
        nonlocal k
        idx = [(k + j) % len(rows) for j in range(per_step)]
        k += per_step
        oracle.decode(q, rho, inp["k_cache"], inp["v_cache"], inp["seqlens"], 1.0,
                      rows=rows[idx], threads=used)

    for _ in range(args.warmup):
        run_step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run_step()
    secs = time.perf_counter() - t0
    tok_s = args.steps * per_step / shape.Hq / secs
    rec = {
        "impl": "reference", "metric": METRIC, "value": tok_s, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": secs * 1e3 / max(1, args.steps), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": headline_config(shape, world),
        "cpu_baseline": {"value": tok_s, "unit": "tokens/s", "cores": used, "kind": "oracle",
                         "sample": f"{per_step} (b, h) rows of {HEADLINE} per step "
                                   "(explicit fp64 covariance form)"},
        "e2e": {"value": tok_s, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(rec), flush=True)
    return 0


def headline_config(shape, world):
    return {"workload": HEADLINE, "B": shape.B, "H_q": shape.Hq, "H_kv": shape.Hkv,
            "d": shape.d, "context": shape.ctx, "softmax_scale": 1.0,
            "kv_cache_bytes": shape.B * shape.S_max * shape.Hkv * shape.d * 2 * 2,
            "l2": "inputs larger than L2: 3 rotating KV cache copies of 537 MB",
            "parallelism": f"replicas x{world} (independent decode batches per GPU)"}


# ------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["plx", "reference"], default="plx")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-prefill-long", action="store_true",
                    help="skip the long-context prefill leg (profiling)")
    ap.add_argument("--no-prefill-bwd", action="store_true", help="skip the backward leg")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-I/O leg (profiling)")
    ap.add_argument("--no-sweep", action="store_true", help="skip the decode grid")
    ap.add_argument("--sweep-cells", nargs="*", default=None,
                    help="run only these grid cells, as BATCHxCONTEXT (e.g. 64x32768)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.impl == "reference":
        return reference_arm(args)

    import torch
    from covariance_corrected_softmax_b200 import plx, workloads as W

    rank, local_rank, world = env_rank()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    peaks, peak_src = load_peaks()

    shape = W.WORKLOADS[HEADLINE]
    dec = bench_decode(plx, W, shape, args.steps, args.warmup, world, device, rank)
    ms_step = dec["ms"] / args.steps
    tok_s = aggregate_rate(world, shape.B, args.steps, dec["ms"])
    gbs = dec["alg_bytes"] / (ms_step / 1e3) / 1e9
    e2e_rec = None  # serving step: append the new token + decode, host I/O included
    if not args.no_e2e:
        e2e = bench_decode_e2e(plx, W, shape, args.steps, args.warmup, world, device, rank)
        e2e_rec = {"value": aggregate_rate(world, shape.B, args.steps, e2e["ms"]),
                   "unit": "tokens/s",
                   "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                   "ms_per_step": e2e["ms"] / args.steps,
                   "call": "plx_decode_append (KV append + decode), one CUDA-graph replay per "
                           "step with the copies of the neighbouring steps on side branches",
                   "gpu_launches": 2 * args.steps}

    prefill = prefill_long = None
    if not args.no_prefill:
        legs = ((PREFILL, 40),) if args.no_prefill_long else ((PREFILL, 40), (PREFILL_LONG, 8))
        for name, psteps in legs:
            pshape = W.WORKLOADS[name]
            pr = bench_prefill(plx, W, pshape, psteps, 3, world, device, rank)
            if "ms" in pr:
                rec_p = prefill_record(name, pshape, pr, psteps, world, peaks, peak_src,
                                       recorded_traffic("plx_prefill_tc", name, PREFILL_SOURCES))
            else:
                rec_p = {"workload": name, **pr}
            if name == PREFILL:
                prefill = rec_p
            else:
                prefill_long = rec_p

    prefill_bwd = None
    if not args.no_prefill and not args.no_prefill_bwd:
        pshape = W.WORKLOADS[PREFILL]
        pr = bench_prefill_bwd(plx, W, pshape, 10, 3, world, device, rank)
        prefill_bwd = (prefill_bwd_record(PREFILL, pshape, pr, 10, peaks, peak_src)
                       if "ms" in pr else {"workload": PREFILL, **pr})

    projection = None
    if not args.no_prefill and world == 1:
        projection = bench_projection(plx, W, peaks, peak_src, device)

    sweep = None
    if not args.no_sweep:
        with ClockSampler(gpu_index()) as clk:
            cells = bench_decode_sweep(plx, W, peaks, device, args.sweep_cells)
        long_ctx = [c for c in cells if c["context"] >= 8192 and not c["launch_bound"]]
        sweep = {"grid": "H_q=16, H_kv=8, d=128, bf16; batch x context, lengths U[ctx/2, ctx]",
                 "timing": "median of per-call CUDA-event times; before each call a 256 MiB "
                           "buffer is written (L2 flush) and another 256 MiB read (dirty "
                           "lines written back before the call)",
                 "peak": peaks["hbm_gbs"], "peak_source": f"{peak_src} HBM copy bandwidth",
                 "cells": cells,
                 "min_frac_ctx_ge_8192": min((c["frac"] for c in long_ctx), default=None),
                 "clocks": clk.summary()}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_decode(dec["inp"], shape)

    traffic = recorded_traffic("plx_decode", HEADLINE, DECODE_SOURCES)
    rec = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": headline_config(shape, world),
        "hbm_gbs": gbs,
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": gbs / peaks["hbm_gbs"],
                     "kernel": "plx_decode (one persistent split-K kernel, merge included)",
                     "peak_source": f"{peak_src} HBM copy bandwidth",
                     "bytes_per_call": dec["alg_bytes"], "traffic": traffic},
        "cpu_baseline": cpu,
        "e2e": e2e_rec,
        "gpu_launches": args.steps,
        "clocks": dec["clocks"],
        "prefill": prefill,
        "prefill_long": prefill_long,
        "prefill_bwd": prefill_bwd,
        "probe_projection": projection,
        "sweep": sweep,
    }
    if rank == 0:
        print(json.dumps(rec), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
