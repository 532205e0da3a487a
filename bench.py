#!/usr/bin/env python
"""Benchmark of one adaptive block-sparse attention layer (pool -> route -> attention)
on the Wan2.1-1.3B 480p self-attention shape (12 heads, 21x30x52 latent = 32760 tokens,
d = 128, 3D blocks 1x8x16, p = 0.9, k_floor = 4), seeded synthetic inputs.

One step = fvattn_block_pool + fvattn_route + fvattn_block_sparse_attn over the whole
layer, inputs resident in HBM, replayed from a CUDA graph captured once (LayerGraph;
--no-graph makes the three calls directly).  Each step is timed on the device with CUDA
events on the launching stream; L2 is flushed (256 MiB write) between steps, outside the
events.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--sweep]

With --gpus N > 1 (launched by torchrun) every rank runs an independent replica (the
path has no exchange step); the time is the max over ranks and the value counts the
work of all ranks.  --impl reference times the fp64 CPU oracle on a bounded sample of
the same workload.  Prints one JSON line (rank 0).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from free_adaptive_block_b200 import metrics as MX  # noqa: E402
from free_adaptive_block_b200 import workloads as W  # noqa: E402

METRIC = "sparse-attn ms/layer + effective TFLOPS (Wan2.1-480p shape), % of bf16 peak"

# DRAM bytes (read + write) of one attention-kernel launch on the Wan2.1-480p workload,
# from an ncu capture of dram__bytes_read.sum + dram__bytes_write.sum; valid only for
# that workload and the kernel source it was taken from.
ATTN_NCU_TRAFFIC = {"fv_attn.cu sha256[:16]": "c3520db57f7689b4", "bytes": 389974272,
                    "workload": "wan21_1.3b_480p_h12_21x30x52"}


def attn_traffic(workload: str):
    import hashlib
    if workload != ATTN_NCU_TRAFFIC["workload"]:
        return None
    src = os.path.join(ROOT, "free_adaptive_block_b200", "csrc", "fv_attn.cu")
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except OSError:
        return None
    return ATTN_NCU_TRAFFIC["bytes"] if h == ATTN_NCU_TRAFFIC["fv_attn.cu sha256[:16]"] else None
UNIT = "TFLOP/s"


def e2e_chunks(requested: int, slices: int) -> int:
    """Chunks of the end-to-end leg: the requested count, or by default the largest divisor
    of the slice count up to 6, so that the chunks are equal (on one B200 at 480p, 6 chunks
    of 2 heads gave 6.9 ms per step against 7.0 for 12, 7.5 for 8 and 7.5 for 4)."""
    if requested > 0:
        return min(requested, slices)
    d = max(c for c in range(1, min(6, slices) + 1) if slices % c == 0)
    return d if d > 1 or slices == 1 else min(4, slices)     # a prime count: uneven chunks


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return dict(bf16=float(pk["bf16_tflops"]), bf16_sustained=float(pk["bf16_tflops_sustained"]),
                    hbm=float(pk["hbm_gbs"]), source="measured")
    except Exception:
        return dict(bf16=1590.0, bf16_sustained=1400.0, hbm=6650.0, source="fallback")


def config_of(wl, extra=None):
    c = {"workload": wl.name, "B": wl.B, "H": wl.H, "N": wl.N, "latent": f"{wl.T}x{wl.Hs}x{wl.Ws}",
         "d": wl.d, "block": f"{wl.bt}x{wl.bh}x{wl.bw}", "p": wl.p, "k_floor": wl.k_floor,
         "l2": "flushed between steps (256 MiB write, outside the timed events)"}
    if extra:
        c.update(extra)
    return c


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples nvidia-smi SM clocks and throttle reasons while the timed region runs.

    nvidia-smi takes a while to start, and a timed region can be shorter than its
    sampling interval, so the bench waits for the first sample before it opens the
    timed region, marks the region's ends, and after it closes waits for the next
    sample; the report keeps the samples that arrived inside the region plus that
    one (reasons are sticky per interval, so it still covers the region's tail).
    """
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    INTERVAL_MS = 50

    def __init__(self, local_rank: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "").split(",")
        vis = [v.strip() for v in vis if v.strip()]
        # nvidia-smi numbers GPUs physically; CUDA_VISIBLE_DEVICES maps the rank's
        # device to that numbering when it is set, else the local rank is the index.
        self.ids = [str(local_rank)]
        if local_rank < len(vis) and vis[local_rank] != str(local_rank):
            self.ids.insert(0, vis[local_rank])
        self.index = self.ids[0]
        self.proc = None
        self.lines = []          # (arrival time, csv line)
        self.thread = None
        self.t_begin = self.t_end = None

    def start(self, wait_s: float = 5.0):
        for idx in self.ids:
            self.index = idx
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", f"--id={idx}", f"--query-gpu={self.FIELDS}",
                     "--format=csv,noheader,nounits", "-lms", str(self.INTERVAL_MS)],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                self.proc = None
                return
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.monotonic() + wait_s
            while not self.lines and time.monotonic() < deadline and self.proc.poll() is None:
                time.sleep(0.01)
            if self.lines or self.proc.poll() is None:
                return
            self.thread.join(timeout=2)      # this id was refused: try the next one

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))

    def begin(self):
        self.t_begin = time.monotonic()

    def end(self):
        self.t_end = time.monotonic()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        t_end = self.t_end if self.t_end is not None else time.monotonic()
        deadline = time.monotonic() + 2.0
        while (not any(t > t_end for t, _ in self.lines) and time.monotonic() < deadline
               and self.proc.poll() is None):
            time.sleep(0.01)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        t_begin = self.t_begin if self.t_begin is not None else 0.0
        inside = [ln for t, ln in self.lines if t_begin <= t <= t_end]
        after = [ln for t, ln in self.lines if t > t_end][:1]
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in inside + after:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "samples_inside_timed_region": len(inside),
                "interval_ms": self.INTERVAL_MS}


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, world: int, device=None) -> float:
    """The largest x over all ranks (x itself at world size 1). Every rank must call it
    at the same point: it is one all-reduce. `device` is where the reduced tensor lives:
    the rank's GPU under NCCL, the CPU under gloo."""
    if world <= 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(eff_flop_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes the same workload (replicas), so the
    job's FLOPs per step are world x one rank's, over the slowest rank's step time."""
    return eff_flop_per_rank * world / (ms_per_step * 1e-3) / 1e12


# ----------------------------------------------------------------------------- GPU arm
def run_ours(args, rank, world, local_rank, wl=None):
    import torch
    import free_adaptive_block_b200 as fv

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl = wl or W.WAN21_480P
    g = fv.Geometry(**wl.geom())
    scale = float(np.float32(1.0 / math.sqrt(wl.d)))
    peaks = load_peaks()

    x = W.generate(wl)
    host = {n: torch.from_numpy(W.bf16_bits(x[n])).view(torch.bfloat16) for n in ("q", "k", "v")}
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    buf = fv.LayerBuffers.allocate(g, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    # The layer step: pool -> route -> attention captured once in a CUDA graph (the
    # library's LayerGraph), so a step is five kernel launches with no host work between
    # them; --no-graph times the three direct calls instead.
    lg = fv.LayerGraph(g, q, k, v, wl.p, wl.k_floor, scale, buf) if args.graph else None

    def step():
        if lg is not None:
            lg.replay()
        else:
            fv.attention_layer(g, q, k, v, wl.p, wl.k_floor, scale, buf, stream)

    # warm-up (also the mask used for the FLOP count)
    for _ in range(max(args.warmup, 3)):
        step()
        flush.fill_(1.0)
    torch.cuda.synchronize(dev)
    if fv.fvattn_device_status(buf.workspace, stream) != 0:
        raise RuntimeError("attention kernel reported a timeout")
    keep = MX.unpack_words(buf.mask.cpu().numpy().view(np.uint32), g.nB)
    real = MX.real_counts(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    eff = MX.effective_flops(keep, real, wl.d)
    kept_frac = float(keep.mean())

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    sampler = ClockSampler(local_rank) if rank == 0 else None
    if sampler:
        sampler.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.begin()
    for i in range(args.steps):
        ev[i][0].record(stream)
        step()
        ev[i][1].record(stream)
        flush.fill_(float(i))
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.end()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    t_layer = [ev[i][0].elapsed_time(ev[i][1]) for i in range(args.steps)]
    total_ms = max_over_ranks(sum(t_layer), world, dev)
    busy = buf.sm_busy_ns.cpu().numpy()
    busy = busy[busy > 0]
    if fv.fvattn_device_status(buf.workspace, stream) != 0:
        raise RuntimeError("attention kernel reported a timeout")

    def graph_of(fn):
        side = torch.cuda.Stream(dev)
        side.wait_stream(stream)
        with torch.cuda.stream(side):
            fn()
        stream.wait_stream(side)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            fn()
        return gr

    def per_call(gr, reps):
        """Device times of `reps` replays, each in its place in the layer: L2 flushed, then
        pool and route (untimed; they also absorb the write-back of the flush's dirty
        lines), then the timed replay."""
        ts = []
        for i in range(3 + reps):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            flush.fill_(float(i))
            fv.fvattn_block_pool(g, q, k, buf.q_pool, buf.k_pool, stream)
            fv.fvattn_route_ws(g, buf.q_pool, buf.k_pool, wl.p, wl.k_floor, scale, buf.mask, buf.counts,
                               buf.route_ws, stream)
            a.record(stream)
            gr.replay()
            b.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 3:
                ts.append(a.elapsed_time(b))
        return ts

    def back_to_back(fn, reps=20):
        """Device time per call of `reps` calls in a row, captured in one CUDA graph (no host
        work between them; the timing protocol of the layer).  fn(s) issues the call on
        stream s; inside a capture s is None, the capturing stream."""
        gr = graph_of(lambda: [fn(None) for _ in range(reps)])
        for _ in range(2):
            gr.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        flush.fill_(0.5)
        a.record(stream)
        gr.replay()
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps

    # Per-stage device times (not added to the layer time above).  Pool streams 201 MB
    # (more than L2); route reads the pooled rows pool has just written.
    t_pool = back_to_back(lambda s: fv.fvattn_block_pool(g, q, k, buf.q_pool, buf.k_pool, s))
    t_route = back_to_back(lambda s: fv.fvattn_route_ws(g, buf.q_pool, buf.k_pool, wl.p, wl.k_floor, scale,
                                                        buf.mask, buf.counts, buf.route_ws, s))
    t_route1 = back_to_back(lambda s: fv.fvattn_route(g, buf.q_pool, buf.k_pool, wl.p, wl.k_floor, scale,
                                                      buf.mask, buf.counts, s), reps=5)
    # the layer's pool and route (fvattn_pool_route: pool, then the workspace route)
    fused = buf.pool_route_ws is not None
    t_pool_route = back_to_back(lambda s: fv.fvattn_pool_route(g, q, k, wl.p, wl.k_floor, scale, buf.q_pool,
                                                               buf.k_pool, buf.mask, buf.counts,
                                                               buf.pool_route_ws, s))
    # (inside a capture the calls must use the capturing stream: stream=None = current)
    attn_graph = graph_of(lambda: fv.fvattn_block_sparse_attn(g, q, k, v, buf.mask, scale, buf.out, buf.lse,
                                                              buf.workspace, buf.sm_busy_ns))
    attn_ts = per_call(attn_graph, min(max(args.steps, 5), 20))
    attn_ms = statistics.median(attn_ts)
    attn_ms_mean = statistics.mean(attn_ts)

    if args.layer_only:
        ms_step = total_ms / args.steps
        return {"metric": METRIC, "value": round(whole_job_tflops(eff, world, ms_step), 3), "unit": UNIT,
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms_step, 4), "attn_ms": round(attn_ms, 4),
                "layer_only": True}

    # Host time of one direct call (Python binding, C entry point, three launches), with
    # the GPU kept busy by the calls queued before it; outside every timed region.
    torch.cuda.synchronize(dev)
    h0 = time.perf_counter()
    for _ in range(20):
        fv.fvattn_block_sparse_attn(g, q, k, v, buf.mask, scale, buf.out, buf.lse, buf.workspace,
                                    buf.sm_busy_ns, stream)
    attn_host_us = (time.perf_counter() - h0) / 20 * 1e6
    torch.cuda.synchronize(dev)

    # dense baseline (p = 1 through the same kernel), same protocol
    dense_graph = graph_of(lambda: fv.fvattn_dense_attn(g, q, k, v, scale, buf.out, buf.lse, buf.workspace,
                                                        None))
    dense_ms = statistics.median(per_call(dense_graph, min(args.steps, 10)))

    # end to end through the public API with host buffers (pinned), copies timed.
    # HostPipeline (the e2e figure): the slices in chunks, each chunk's copies in and out
    # overlapped with the neighbouring chunks' kernels.  For comparison, the serial form:
    # copy Q/K/V into the captured buffers, replay the layer, read out and lse back.
    pinned = {n: host[n].pin_memory() for n in ("q", "k", "v")}
    out_h = torch.empty(buf.out.shape, dtype=torch.bfloat16).pin_memory()
    lse_h = torch.empty(buf.lse.shape, dtype=torch.float32).pin_memory()
    n_e2e = min(args.steps, 5)
    pipe = fv.HostPipeline(g, wl.p, wl.k_floor, scale, chunks=e2e_chunks(args.e2e_chunks, g.B * g.H), device=dev)

    def e2e_time(fn):
        ts = []
        for i in range(2 + n_e2e):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fn()
            b.record(stream)
            torch.cuda.synchronize(dev)
            if i >= 2:
                ts.append(a.elapsed_time(b))
        return max_over_ranks(statistics.mean(ts), world, dev)

    def serial():
        q.copy_(pinned["q"], non_blocking=True)
        k.copy_(pinned["k"], non_blocking=True)
        v.copy_(pinned["v"], non_blocking=True)
        step()
        out_h.copy_(buf.out, non_blocking=True)
        lse_h.copy_(buf.lse, non_blocking=True)

    e2e_ms = e2e_time(lambda: pipe.run(pinned["q"], pinned["k"], pinned["v"], out_h, lse_h))
    e2e_serial_ms = e2e_time(serial)
    h2d = sum(pinned[n].numel() * 2 for n in ("q", "k", "v"))
    d2h = out_h.numel() * 2 + lse_h.numel() * 4

    # the library's kernels one layer step launches: pool; route (logits + select through
    # the route workspace, else the one-kernel route); prep_cost, prep_order, attention
    launches_per_step = 1 + (2 if (fused or buf.route_ws is not None) else 1) + 3
    ms_step = total_ms / args.steps
    value = whole_job_tflops(eff, world, ms_step)
    attn_tflops = eff / (attn_ms * 1e-3) / 1e12
    # the roofline divides by the average duration of the same timed calls
    attn_tflops_avg = eff / (attn_ms_mean * 1e-3) / 1e12
    pr_bytes = MX.pool_route_bytes(wl.B, wl.H, wl.N, g.nB, wl.d, g.words)
    pr_ms = t_pool_route if buf.pool_route_ws is not None else t_pool + t_route
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic", "config": config_of(wl),
        "ms_per_layer": round(ms_step, 4),
        # this rank's per-step spread (the headline above is the mean, max over ranks)
        "ms_per_layer_median": round(statistics.median(t_layer), 4),
        "ms_per_layer_min": round(min(t_layer), 4), "ms_per_layer_max": round(max(t_layer), 4),
        "attn_ms": round(attn_ms, 4),
        "attn_ms_mean": round(attn_ms_mean, 4),
        "attn_call_host_us": round(attn_host_us, 1),
        "attn_effective_tflops": round(attn_tflops, 2),
        "attn_frac_of_bf16_peak": round(attn_tflops / peaks["bf16"], 4),
        "pool_ms": round(t_pool, 4), "route_ms": round(t_route, 4),
        "pool_route_ms": round(t_pool_route, 4),
        "pool_route_kernel": ("fvattn_pool_route: pool, then the workspace route (logits, selection)" if fused
                              else "pool + two-kernel route"),
        "route_one_kernel_ms": round(t_route1, 4),
        "stage_timing": "pool, route (fvattn_route_ws), pool_route (fvattn_pool_route, the layer's): device "
                        "time per call of 20 back-to-back calls replayed from one CUDA graph (route_one_kernel: "
                        "5); attention: one captured call after L2 flush + pool + route "
                        "(attn_ms median, attn_ms_mean and roofline mean)",
        "layer_step": "CUDA graph of pool -> route -> attention (LayerGraph)" if args.graph else "direct calls",
        "pool_route_gbs": round(pr_bytes / (pr_ms * 1e-3) / 1e9, 1),
        "pool_route_frac_of_hbm": round(pr_bytes / (pr_ms * 1e-3) / 1e9 / peaks["hbm"], 4),
        "dense_attn_ms": round(dense_ms, 4),
        "dense_attn_tflops": round(MX.dense_flops(wl.B, wl.H, wl.N, wl.d) / (dense_ms * 1e-3) / 1e12, 2),
        "speedup_vs_dense_attn": round(dense_ms / attn_ms, 3),
        "kept_block_frac": round(kept_frac, 4),
        "effective_flop_per_layer": eff,
        "sm_busy_max_over_mean": round(float(busy.max() / busy.mean()), 4) if busy.size else None,
        "roofline": {"bound": "tensor", "kernel": "fvattn_block_sparse_attn (prep + attn_kernel)",
                     "achieved": round(attn_tflops_avg, 2), "peak": peaks["bf16"], "unit": "TFLOP/s",
                     "frac": round(attn_tflops_avg / peaks["bf16"], 4), "traffic": attn_traffic(wl.name),
                     "duration": f"mean of {len(attn_ts)} event-timed calls, {attn_ms_mean:.4f} ms",
                     "peak_source": f"{peaks['source']} bf16 (burst, cuBLAS)"},
        "e2e": {"value": round(whole_job_tflops(eff, world, e2e_ms), 3), "unit": UNIT,
                "how": f"HostPipeline: pinned host Q/K/V -> device -> out/lse -> pinned host in "
                       f"{len(pipe.ranges)} chunks of slices, copies overlapped with the kernels",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "serial_ms_per_step": round(e2e_serial_ms, 3)},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    return line


# ----------------------------------------------------------------------------- CPU oracle
def oracle_sample(wl, x, n_qblocks: int, seed: int = 5):
    """The oracle on a bounded sample: pool and route of the whole layer, masked
    attention of n_qblocks query blocks per head.  Returns (seconds, effective flops)."""
    sys.path.insert(0, ROOT)
    import oracle as O
    og = O.block_geometry(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
    scale = 1.0 / math.sqrt(wl.d)
    qbs = W.sample_qblocks(wl, n_qblocks, seed=seed)
    t0 = time.perf_counter()
    Qp, Kp = O.pool(x["q"], og), O.pool(x["k"], og)
    r = O.route(Qp, Kp, wl.p, wl.k_floor, scale)
    O.masked_attn(x["q"], x["k"], x["v"], r.keep, og, scale, qbs)
    dt = time.perf_counter() - t0
    real = og.real_count
    sub = r.keep[:, :, qbs, :]
    eff = float(4.0 * wl.d * ((sub.astype(np.int64) @ real) * real[qbs][None, None, :]).sum())
    return dt, eff


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads") for i in threadpool_info() if i.get("num_threads")]
        return int(max(n)) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(wl, x, budget_s: float = 15.0):
    dt, eff = oracle_sample(wl, x, 2)
    n = max(2, min(wl.nB, int(2 * budget_s / max(dt, 1e-3))))
    dt, eff = oracle_sample(wl, x, n)
    return {"value": round(eff / dt / 1e12, 6), "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
            "seconds": round(dt, 2),
            "sample": f"fp64 NumPy oracle: pool + route of the whole layer, masked attention of {n} "
                      f"query blocks per head ({wl.H} heads); TFLOP/s = effective FLOPs of the sample / time"}


def run_reference(args):
    wl = W.WAN21_480P
    x = W.generate(wl)
    # size one step to ~2-4 s of CPU work
    dt, _ = oracle_sample(wl, x, 1)
    n = max(1, min(wl.nB, int(3.0 / max(dt, 1e-3))))
    for _ in range(args.warmup):
        oracle_sample(wl, x, n)
    secs, flops = [], []
    for i in range(args.steps):
        dt, eff = oracle_sample(wl, x, n, seed=100 + i)
        secs.append(dt)
        flops.append(eff)
    total = sum(secs)
    value = sum(flops) / total / 1e12
    sample = (f"fp64 NumPy oracle per step: pool + route of the whole layer and masked attention of "
              f"{n} sampled query blocks per head ({wl.H} heads)")
    return {"metric": METRIC, "value": round(value, 6), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * total / args.steps, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl), "impl": "reference",
            "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def _graph_of(fn, stream):
    """Captures fn() once in a CUDA graph (after one uncaptured run on a side stream)."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        fn()
    stream.wait_stream(side)
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        fn()
    return gr


def _timed_replays(gr, prepare, flush, reps, direct=None):
    """Device times of `reps` replays of gr, each in its place in a layer: L2 flushed, then
    prepare() (pool and route for the point, untimed; it also absorbs the write-back of the
    flush's dirty lines), then the timed replay.  With `direct`, the same for a direct call
    of the function the graph holds.  Returns (replay times, direct times)."""
    import torch
    ts, td = [], []
    for i in range(3 + reps):
        for fn, out in ((lambda: gr.replay(), ts),) + (((direct, td),) if direct else ()):
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            flush.fill_(float(i))
            prepare()
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if i >= 3:
                out.append(a.elapsed_time(b))
    return ts, td


def run_sweep(args, local_rank):
    """Config-5 sweep: p x k_floor at the 480p shape; one JSON line per point (stdout).  Each
    point times the attention call as the headline does: a graph replay after an L2 flush,
    pool and route; the direct (uncaptured) call is timed the same way beside it."""
    import torch
    import free_adaptive_block_b200 as fv
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    wl0 = W.WAN21_480P
    g = fv.Geometry(**wl0.geom())
    scale = float(np.float32(1.0 / math.sqrt(wl0.d)))
    x = W.generate(wl0)
    q, k, v = (torch.from_numpy(W.bf16_bits(x[n])).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
    buf = fv.LayerBuffers.allocate(g, dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    real = MX.real_counts(wl0.T, wl0.Hs, wl0.Ws, wl0.bt, wl0.bh, wl0.bw)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    attn = lambda: fv.fvattn_block_sparse_attn(g, q, k, v, buf.mask, scale, buf.out, buf.lse,  # noqa: E731
                                               buf.workspace, buf.sm_busy_ns)
    dense = lambda: fv.fvattn_dense_attn(g, q, k, v, scale, buf.out, buf.lse, buf.workspace)  # noqa: E731
    route = lambda p, kf: fv.fvattn_pool_route(g, q, k, p, kf, scale, buf.q_pool, buf.k_pool,  # noqa: E731
                                               buf.mask, buf.counts, buf.pool_route_ws)
    route(wl0.p, wl0.k_floor)
    dense_ts, _ = _timed_replays(_graph_of(dense, stream), lambda: route(wl0.p, wl0.k_floor), flush, args.steps)
    dense_ms = statistics.median(dense_ts)
    attn_graph = None
    for wl in W.sweep():
        route(wl.p, wl.k_floor)
        torch.cuda.synchronize()
        keep = MX.unpack_words(buf.mask.cpu().numpy().view(np.uint32), g.nB)
        eff = MX.effective_flops(keep, real, wl.d)
        if attn_graph is None:
            attn_graph = _graph_of(attn, stream)   # the mask buffer is an input: one graph serves
        ts, td = _timed_replays(attn_graph, lambda: route(wl.p, wl.k_floor), flush, args.steps, direct=attn)
        ms, ms_direct = statistics.median(ts), statistics.median(td)
        busy = buf.sm_busy_ns.cpu().numpy()
        busy = busy[busy > 0]
        print(json.dumps({"sweep_point": wl.name, "p": wl.p, "k_floor": wl.k_floor,
                          "kept_block_frac": round(float(keep.mean()), 4), "attn_ms": round(ms, 4),
                          "attn_ms_direct_call": round(ms_direct, 4),
                          "effective_tflops": round(eff / (ms * 1e-3) / 1e12, 2),
                          "frac_of_bf16_peak": round(eff / (ms * 1e-3) / 1e12 / peaks["bf16"], 4),
                          "dense_attn_ms": round(dense_ms, 4), "speedup_vs_dense": round(dense_ms / ms, 3),
                          "timing": "graph replay after L2 flush + pool + route (median); direct call beside it",
                          "sm_busy_max_over_mean": (round(float(busy.max() / busy.mean()), 4)
                                                    if busy.size else None)}), flush=True)


def run_next(args, local_rank):
    """The rows beyond Top-p / Top-k routing, one JSON line each: keyframe blocks at the 6x
    horizon, Top-p over tokens, runtime mask repair and slack-aware augmentation at 480p.
    Each line reports the kept fraction, the attention time (graph replay after L2 flush
    and the row's routing), and its speedup over the dense path on the same inputs."""
    import torch
    import free_adaptive_block_b200 as fv
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    peaks = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for wl, modes in ((W.WAN21_6X, ("plain", "keyframes")),
                      (W.WAN21_480P, ("plain", "token_mass", "repair", "slack_augment"))):
        g = fv.Geometry(**wl.geom())
        scale = float(np.float32(1.0 / math.sqrt(wl.d)))
        x = W.generate(wl)
        q, k, v = (torch.from_numpy(W.bf16_bits(x[n])).view(torch.bfloat16).to(dev) for n in ("q", "k", "v"))
        del x
        buf = fv.LayerBuffers.allocate(g, dev)
        real = MX.real_counts(wl.T, wl.Hs, wl.Ws, wl.bt, wl.bh, wl.bw)
        attn = lambda: fv.fvattn_block_sparse_attn(g, q, k, v, buf.mask, scale, buf.out, buf.lse,  # noqa: E731
                                                   buf.workspace, buf.sm_busy_ns)
        dense = lambda: fv.fvattn_dense_attn(g, q, k, v, scale, buf.out, buf.lse, buf.workspace)  # noqa: E731
        base_opts = dict(p=wl.p, k_floor=wl.k_floor, scale=scale)
        tau = 1.0 / g.nB                        # a block above the uniform score

        def prepare(mode):
            fv.fvattn_block_pool(g, q, k, buf.q_pool, buf.k_pool)
            o = dict(base_opts)
            if mode == "keyframes":
                o.update(kf_stride=20, kf_phase=0)
            elif mode == "token_mass":
                o.update(token_mass=1)
            elif mode == "repair":
                o.update(repair=1)
            fv.fvattn_route_ex(g, buf.q_pool, buf.k_pool, fv.RouteOpts(**o), buf.mask, buf.counts, buf.route_ws)
            if mode == "slack_augment":
                fv.fvattn_slack_augment(g, buf.route_ws, tau, buf.mask, buf.counts, buf.workspace)

        prepare("plain")
        dense_reps = 2 if wl.N > 100000 else 6
        dense_ms = statistics.median(_timed_replays(_graph_of(dense, stream), lambda: prepare("plain"), flush,
                                                    dense_reps)[0])
        gr = _graph_of(attn, stream)
        for mode in modes:
            prepare(mode)
            torch.cuda.synchronize()
            keep = MX.unpack_words(buf.mask.cpu().numpy().view(np.uint32), g.nB)
            eff = MX.effective_flops(keep, real, wl.d)
            reps = min(args.steps, 5 if wl.N > 100000 else 10)
            ts, _ = _timed_replays(gr, lambda: prepare(mode), flush, reps)
            ms = statistics.median(ts)
            busy = buf.sm_busy_ns.cpu().numpy()
            busy = busy[busy > 0]
            line = {"next_row": mode, "workload": wl.name, "p": wl.p, "k_floor": wl.k_floor,
                    "kept_block_frac": round(float(keep.mean()), 4), "attn_ms": round(ms, 4),
                    "effective_tflops": round(eff / (ms * 1e-3) / 1e12, 2),
                    "frac_of_bf16_peak": round(eff / (ms * 1e-3) / 1e12 / peaks["bf16"], 4),
                    "dense_attn_ms": round(dense_ms, 4), "speedup_vs_dense": round(dense_ms / ms, 3),
                    "sm_busy_max_over_mean": round(float(busy.max() / busy.mean()), 4) if busy.size else None}
            if mode == "keyframes":
                line["keyframes"] = "stride 20, phase 0 (latent frames 0, 20, ..., 120)"
            if mode == "slack_augment":
                line["tau"] = tau
            print(json.dumps(line), flush=True)
        del buf, q, k, v
        torch.cuda.empty_cache()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sweep", action="store_true", help="also time the 15 p/k points (config 5)")
    ap.add_argument("--next", dest="next_rows", action="store_true",
                    help="also time keyframes (6x), Top-p over tokens, mask repair, slack augmentation (480p)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--all-configs", action="store_true",
                    help="after the 480p line, one line per other workload (tiny, 720p, 6x horizon)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="time the layer as three direct calls instead of a captured CUDA graph")
    ap.add_argument("--e2e-chunks", type=int, default=0,
                    help="chunks of (b, h) slices in the end-to-end leg (HostPipeline); 0: the largest "
                         "divisor of the slice count up to 6")
    ap.add_argument("--layer-only", action="store_true",
                    help="time the layer steps only (no dense, e2e or CPU legs); for profilers")
    ap.add_argument("--workload", default=None, choices=sorted(W.ALL),
                    help="one line for this workload only, on one GPU (for profilers; the "
                         "headline is the default, Wan2.1-480p)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if args.workload is not None and args.workload != W.WAN21_480P.name:
        if world > 1:
            raise SystemExit("--workload runs on one GPU")
        wl = W.ALL[args.workload]
        line = run_ours(args, 0, 1, local_rank, wl)
        line["metric"] = f"same measurements on the {wl.name} workload (not the headline)"
        print(json.dumps(line), flush=True)
        return
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            if world == 1 and not (args.no_cpu_baseline or args.layer_only):
                line["cpu_baseline"] = cpu_baseline(W.WAN21_480P, W.generate(W.WAN21_480P))
            print(json.dumps(line), flush=True)
        if args.all_configs and rank == 0:
            for wl in (W.TINY, W.WAN22_720P, W.WAN21_6X):
                extra = run_ours(args, 0, 1, local_rank, wl)
                extra["metric"] = f"same measurements on the {wl.name} workload (not the headline)"
                print(json.dumps(extra), flush=True)
        if args.sweep and rank == 0:
            run_sweep(args, local_rank)
        if args.next_rows and rank == 0:
            run_next(args, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
