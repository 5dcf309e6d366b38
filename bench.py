#!/usr/bin/env python
"""Throughput of the chunked SSD forward pass on one or more B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one ssd_forward call (every kernel of the path) over one batch of the
Mamba-2-2.7B-like layer workload: batch 8 x 2048 tokens, 80 heads of dim 64,
state 128, one B/C group, chunk 256, bf16 x/B/C with fp32 dt/A/D, synthetic
seeded inputs resident in HBM.  With N > 1 (torchrun, one rank per GPU) every
rank runs its own batch (weak scaling, no data-path collective); the time is
the max over ranks.  Rank 0 prints one JSON line.

``--impl reference`` times the fp64 CPU oracle instead (rank 0 only) on bounded
samples of the same workload.

On one GPU the line also carries ``workloads``: every workload of the table
(the layer, the state-size sweep, the length sweep and the packed batch), each
with tokens/s, the dominant kernel's time, its roofline fraction and the path it
took (``--no-workloads`` skips them); and ``next``: the decode step, the causal
conv1d + SiLU and the gated RMSNorm timed at the same layer's shapes
(``--no-decode`` skips them).
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "SSD fwd tokens/s at Mamba-2-2.7B layer shape (1 B200); % of roofline"
WORKLOAD = workloads.MAMBA2_2P7B
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ----------------------------------------------------------------- accounting
def algorithmic_bytes(wl, init_present: bool, nseq: int) -> int:
    """Compulsory I/O: read x, dt, B, C (and init when nonzero); write y and the fp32 final state."""
    es = 2 if wl.dtype == "bf16" else 4
    T, H, P, N, G = wl.tokens, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    rd = T * H * P * es + T * H * 4 + 2 * T * G * N * es + 2 * H * 4
    if init_present:
        rd += nseq * H * P * N * 4
    wr = T * H * P * es + nseq * H * P * N * 4
    return rd + wr


def algorithmic_flops(wl, seq_lengths) -> float:
    """Causal block FLOPs of the chunked algorithm: per chunk of length q, q(q+1)N per group
    for C B^T, q(q+1)P per head for the masked product, 4qNP per head for the chunk state
    and the carried-state output."""
    H, P, N, G, Q = wl.nheads, wl.headdim, wl.dstate, wl.ngroups, wl.chunk
    tot = 0.0
    for L in seq_lengths:
        for t0 in range(0, L, Q):
            q = min(Q, L - t0)
            tot += G * q * (q + 1) * N + H * (q * (q + 1) * P + 4 * q * N * P)
    return tot


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel)
    except Exception:
        return None
    if not rec:
        return None
    import hashlib

    src = os.path.join(ROOT, rec["source"])
    try:
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except Exception:
        return None
    if sha != rec.get("source_sha"):
        return None  # the kernel changed since the counters were taken
    return rec.get("dram_bytes_per_launch")


# ----------------------------------------------------------- multi-rank timing
def aggregate_max(seconds: float, world: int, device) -> float:
    """Max over ranks of a per-rank device time (every rank must call it)."""
    t = torch.tensor([seconds], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, steps: int, world: int, max_total_s: float) -> float:
    """Whole-job tokens/s: every rank processed its own batch `steps` times."""
    return world * tokens_per_rank * steps / max_total_s


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons around a timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu: str):
        self.gpu = gpu
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t0 = time.time()
        while time.time() - t0 < 5 and os.path.getsize(self.path) == 0:
            time.sleep(0.05)
        self.t_start = time.time()

    def stop(self):
        self.t_stop = time.time()
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[3], parts[4:]))
            except ValueError:
                continue
        os.unlink(self.path)
        inside = [r for r in rows if self.t_start - 0.1 <= r[0] <= self.t_stop + 0.1]
        use = inside or rows
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in use for i, v in enumerate(r[4][1:5]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[1] for r in use), "sm_max_mhz": max(r[2] for r in use),
                "reasons": reasons, "samples": len(use), "samples_in_window": len(inside)}


def gpu_selector(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [v.strip() for v in vis.split(",") if v.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


# ------------------------------------------------------------ CPU oracle timing
def cpu_oracle_sample(prob, rows, heads, nthreads):
    """Time the oracle on sequences ``rows`` x ``heads`` of ``prob``; returns (seconds, token-equivalents)."""
    import oracle

    pairs = [(s, h) for s in rows for h in heads]
    t0 = time.perf_counter()
    oracle.ssd_forward_problem(prob, pairs=pairs, nthreads=nthreads)
    dt = time.perf_counter() - t0
    toks = sum(prob.seq_offsets[s + 1] - prob.seq_offsets[s] for s in rows) * len(heads) / prob.wl.nheads
    return dt, toks


def cpu_baseline(prob, budget_s=10.0):
    cores = len(os.sched_getaffinity(0))
    H = prob.wl.nheads
    spent, toks, rows = 0.0, 0.0, 0
    while spent < budget_s:  # whole sequences (all heads), cycling over the batch until the budget is spent
        dt, tk = cpu_oracle_sample(prob, [rows % prob.nseq], list(range(H)), cores)
        spent += dt
        toks += tk
        rows += 1
    return {"value": toks / spent, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{rows} sequence passes over the {prob.nseq} sequences x all {H} heads ({int(toks)} tokens), "
                      f"fp64 sequential recurrence, OpenMP over (sequence, head), {spent:.1f} s"}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world, local_rank):
    import ssd_sequence_mixing_b200 as ssd

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = WORKLOAD
    prob = workloads.generate(wl, seed=rank)
    d = {k: (None if getattr(prob, k) is None else getattr(prob, k).to(dev))
         for k in ("x", "dt", "A", "B", "C", "D", "init_state", "cu_seqlens")}
    y = torch.empty_like(d["x"])
    fin = torch.empty((prob.nseq, wl.nheads, wl.headdim, wl.dstate), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    shape = ssd.make_shape(d["x"], d["B"], d["cu_seqlens"])
    path = {ssd.PATH_SIMT: "simt", ssd.PATH_TC: "tc"}.get(ssd.select_path(shape, wl.chunk), "?")

    def step():
        ssd.ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], d["cu_seqlens"], wl.chunk,
                        y=y, final_state=fin, stream=stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()

    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    dom = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    for a, b in dom:  # torch creates the CUDA event on first record; the library re-records it
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_selector(local_rank))
    sampler.start()
    launches0 = ssd.kernel_launch_count()
    for k in range(K):
        flush.zero_()  # evict L2 between timed steps (outside the events)
        ssd.profile_dominant(*dom[k])
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    ssd.profile_dominant(None, None)
    launches = ssd.kernel_launch_count() - launches0
    clocks = sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    assert ssd.query_status() == 0

    step_ms = [a.elapsed_time(b) for a, b in ev]
    dom_ms = [a.elapsed_time(b) for a, b in dom]
    max_total = aggregate_max(sum(step_ms) / 1e3, world, dev)
    value = weak_scaling_value(wl.tokens, K, world, max_total)

    # end to end through the host-buffer entry point: H2D inputs, compute, D2H outputs
    pin = lambda v: None if v is None else v.pin_memory()
    h = {k: pin(getattr(prob, k)) for k in ("x", "dt", "A", "B", "C", "D", "init_state", "cu_seqlens")}
    yh = torch.empty(prob.x.shape, dtype=prob.x.dtype).pin_memory()
    fh = torch.empty(fin.shape, dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in h.values() if v is not None)
    d2h = yh.numel() * yh.element_size() + fh.numel() * fh.element_size()

    def host_step():
        ssd.ssd_forward_host(h["x"], h["dt"], h["A"], h["B"], h["C"], h["D"], h["init_state"], h["cu_seqlens"],
                             wl.chunk, y=yh, final_state=fh, stream=stream)

    host_step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e2e_ms = []
    for _ in range(args.e2e_steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        host_step()
        b.record(stream)
        b.synchronize()
        e2e_ms.append(a.elapsed_time(b))
    e2e_value = weak_scaling_value(wl.tokens, args.e2e_steps, world, aggregate_max(sum(e2e_ms) / 1e3, world, dev))
    link = host_link_gbs(dev) if rank == 0 else None

    if rank != 0:
        return None

    peaks, peak_kind = load_peaks()
    nbytes = algorithmic_bytes(wl, prob.init_state is not None, prob.nseq)
    lens = [prob.seq_offsets[i + 1] - prob.seq_offsets[i] for i in range(prob.nseq)]
    flops = algorithmic_flops(wl, lens)
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    bound = "hbm" if t_mem >= t_flop else "tensor"
    dom_s = statistics.mean(dom_ms) / 1e3
    if bound == "hbm":
        achieved, peak, unit = nbytes / dom_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        achieved, peak, unit = flops / dom_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    kernel = "ssd_fused_tc" if path == "tc" else "chunk_output_kernel"
    roof_s = max(t_mem, t_flop)
    step_s = max_total / K
    out = {
        "metric": METRIC,
        "value": value,
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": step_s * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded; Mamba-2 init distributions; inputs resident in HBM)",
        "config": {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seqlen, "nheads": wl.nheads,
                   "headdim": wl.headdim, "dstate": wl.dstate, "ngroups": wl.ngroups, "chunk": wl.chunk,
                   "io_dtype": "bf16 x/B/C/y, fp32 dt/A/D/states", "parallelism": f"dp{world} (independent batches)",
                   "l2": "flushed between timed steps (256 MB write outside the events)", "path": path},
        "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
                     "traffic": load_traffic(kernel), "kernel": kernel, "peak_source": f"{peak_kind} ({unit})",
                     "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                     "dominant_ms": statistics.mean(dom_ms),
                     "step_roofline_us": roof_s * 1e6, "step_frac": roof_s / step_s},
        "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": args.e2e_steps, "ms_per_step": statistics.mean(e2e_ms),
                "api": "ssd_forward_host (pinned host buffers)",
                # the host link measured on this machine, and the copy time it allows per step
                "link": link,
                "link_bound_ms": 1e3 * max(h2d / (link["h2d_gbs"] * 1e9), d2h / (link["d2h_gbs"] * 1e9),
                                           (h2d + d2h) / (link["bidir_gbs"] * 1e9)),
                "link_frac": 1e3 * max(h2d / (link["h2d_gbs"] * 1e9), d2h / (link["d2h_gbs"] * 1e9),
                                       (h2d + d2h) / (link["bidir_gbs"] * 1e9)) / statistics.mean(e2e_ms)},
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    if world == 1 and not args.no_workloads:
        # configs 1-4 of the workload table (the tiny parity case is launch-bound)
        out["workloads"] = [workload_measurement(w, dev, stream, flush) for w in workloads.ALL
                            if w is not workloads.TINY]
    if world == 1 and not args.no_decode:
        out["next"] = {"decode_step": decode_measurement(dev, stream, flush)}
        out["next"].update(block_measurements(dev, stream, flush))
    if world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(prob, budget_s=args.cpu_budget)
    return out


# ------------------------------------------------------------- the host link
def host_link_gbs(dev, nbytes: int = 256 << 20, reps: int = 5):
    """Pinned host <-> device copy bandwidth of this machine (GB/s, best of ``reps``): host to
    device alone, device to host alone, and both directions at once on two streams."""
    h_src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    h_dst = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    d_a = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    d_b = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def once(h2d: bool, d2h: bool) -> float:
        start = torch.cuda.Event(enable_timing=True)
        ends = []
        start.record(s_in)
        s_out.wait_event(start)
        if h2d:
            with torch.cuda.stream(s_in):
                d_a.copy_(h_src, non_blocking=True)
                e = torch.cuda.Event(enable_timing=True)
                e.record(s_in)
                ends.append(e)
        if d2h:
            with torch.cuda.stream(s_out):
                h_dst.copy_(d_b, non_blocking=True)
                e = torch.cuda.Event(enable_timing=True)
                e.record(s_out)
                ends.append(e)
        torch.cuda.synchronize(dev)
        return max(start.elapsed_time(e) for e in ends) / 1e3

    out = {}
    for name, h2d, d2h in (("h2d_gbs", True, False), ("d2h_gbs", False, True), ("bidir_gbs", True, True)):
        t = min(once(h2d, d2h) for _ in range(reps))
        out[name] = (int(h2d) + int(d2h)) * nbytes / t / 1e9
    return out


# ------------------------------------------------- every workload of the table
def roofline_line(wl, prob, dom_s, peaks, peak_kind):
    """Roofline of one ssd_forward workload: max(bytes / HBM peak, FLOPs / bf16 peak)."""
    nbytes = algorithmic_bytes(wl, prob.init_state is not None, prob.nseq)
    lens = [prob.seq_offsets[i + 1] - prob.seq_offsets[i] for i in range(prob.nseq)]
    flops = algorithmic_flops(wl, lens)
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9)
    t_flop = flops / (peaks["bf16_tflops"] * 1e12)
    if t_mem >= t_flop:
        bound, achieved, peak, unit = "hbm", nbytes / dom_s / 1e9, peaks["hbm_gbs"], "GB/s"
    else:
        bound, achieved, peak, unit = "tensor", flops / dom_s / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
            "peak_source": f"{peak_kind} ({unit})", "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
            "roofline_us": max(t_mem, t_flop) * 1e6}


def workload_measurement(wl, dev, stream, flush, steps=10, warmup=3):
    """Time one ssd_forward call on workload ``wl`` (seeded synthetic inputs resident in
    HBM, L2 flushed between steps): step time and the dominant kernel's time from the
    library's events, median over ``steps``."""
    import ssd_sequence_mixing_b200 as ssd

    prob = workloads.generate(wl, seed=0)
    d = {k: (None if getattr(prob, k) is None else getattr(prob, k).to(dev))
         for k in ("x", "dt", "A", "B", "C", "D", "init_state", "cu_seqlens")}
    y = torch.empty_like(d["x"])
    fin = torch.empty((prob.nseq, wl.nheads, wl.headdim, wl.dstate), dtype=torch.float32, device=dev)
    shape = ssd.make_shape(d["x"], d["B"], d["cu_seqlens"])
    path = {ssd.PATH_SIMT: "simt", ssd.PATH_TC: "tc"}.get(ssd.select_path(shape, wl.chunk), "?")

    def step():
        ssd.ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], d["cu_seqlens"], wl.chunk,
                        y=y, final_state=fin, stream=stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    dom = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in dom:
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize()
    for k in range(steps):
        flush.zero_()
        ssd.profile_dominant(*dom[k])
        ev[k][0].record(stream)
        step()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    ssd.profile_dominant(None, None)
    assert ssd.query_status() == 0
    step_s = statistics.median(a.elapsed_time(b) for a, b in ev) / 1e3
    dom_s = statistics.median(a.elapsed_time(b) for a, b in dom) / 1e3
    peaks, kind = load_peaks()
    roof = roofline_line(wl, prob, dom_s, peaks, kind)
    out = {"workload": wl.name, "path": path, "tokens": wl.tokens, "tokens_per_s": wl.tokens / step_s,
           "step_us": step_s * 1e6, "dominant_us": dom_s * 1e6, "roofline": roof,
           "step_frac": roof["roofline_us"] / (step_s * 1e6)}
    del d, y, fin
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------- decode step (next row)
DECODE = workloads.custom(64, 1, H=80, P=64, N=128, G=1, chunk=64, dtype="bf16", init=True,
                          name="decode_step_b64_H80_P64_N128_bf16")


def decode_measurement(dev, stream, flush, reps: int = 20):
    """One recurrent decode step for 64 sequences at the Mamba-2-2.7B layer shape: the fp32
    state (168 MB, larger than L2) is read and written once.  Median of ``reps`` launches,
    CUDA events on the launching stream, L2 flushed between launches."""
    import ssd_sequence_mixing_b200 as ssd

    wl = DECODE
    prob = workloads.generate(wl, seed=0)
    x, dt, B, C = (getattr(prob, k)[:, 0].contiguous().to(dev) for k in ("x", "dt", "B", "C"))
    A, D = prob.A.to(dev), prob.D.to(dev)
    state = prob.init_state.to(dev)
    y = torch.empty_like(x)
    for _ in range(3):
        ssd.ssd_decode_step(x, dt, A, B, C, D, state, y=y, stream=stream)
    ms = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        ssd.ssd_decode_step(x, dt, A, B, C, D, state, y=y, stream=stream)
        b.record(stream)
        ms.append((a, b))
    torch.cuda.synchronize()
    t = statistics.median(a.elapsed_time(b) for a, b in ms) / 1e3
    rows, H, P, N, G = wl.batch, wl.nheads, wl.headdim, wl.dstate, wl.ngroups
    nbytes = rows * H * P * N * 4 * 2 + rows * H * P * 2 * 2 + rows * G * N * 2 * 2 + rows * H * 4
    peaks, kind = load_peaks()
    gbs = nbytes / t / 1e9
    return {"workload": wl.name, "us": t * 1e6, "tokens_per_s": rows / t, "algorithmic_bytes": nbytes,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{kind} (GB/s)"},
            "l2": "flushed between launches; the state alone exceeds L2"}


def _median_us(fn, stream, flush, reps: int = 20) -> float:
    for _ in range(3):
        fn()
    ev = []
    for _ in range(reps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev) * 1e3


def block_measurements(dev, stream, flush):
    """The Mamba-2 block's steps either side of the SSD at the 2.7B layer shape (batch 8 x
    2048 tokens, d_inner 5120, one B/C group of N = 128, bf16): the causal conv1d + SiLU
    over the 5376 x/B/C channels and the gated RMSNorm over 5120 features.  Both read
    each input once and write each output once; seeded synthetic inputs and weights."""
    import ssd_sequence_mixing_b200 as ssd

    peaks, kind = load_peaks()
    g = torch.Generator(device=dev).manual_seed(0)
    tokens, ch, dim = 8 * 2048, 5120 + 2 * 128, 5120
    xbc = torch.randn((8, 2048, ch), generator=g, device=dev).to(torch.bfloat16)
    w = torch.randn((ch, 4), generator=g, device=dev) * 0.5
    b = torch.randn((ch,), generator=g, device=dev) * 0.1
    out = torch.empty_like(xbc)
    t_conv = _median_us(lambda: ssd.causal_conv1d_silu(xbc, w, b, out=out, stream=stream), stream, flush)
    conv_bytes = tokens * ch * 2 * 2 + ch * 5 * 4
    del xbc, out
    y = torch.randn((tokens, dim), generator=g, device=dev).to(torch.bfloat16)
    z = torch.randn((tokens, dim), generator=g, device=dev).to(torch.bfloat16)
    wn = 1.0 + 0.1 * torch.randn((dim,), generator=g, device=dev)
    o = torch.empty_like(y)
    t_norm = _median_us(lambda: ssd.gated_rmsnorm(y, z, wn, out=o, stream=stream), stream, flush)
    norm_bytes = tokens * dim * 2 * 3 + dim * 4

    def line(name, t_us, nbytes, kernel):
        gbs = nbytes / (t_us * 1e-6) / 1e9
        return {"workload": name, "us": t_us, "algorithmic_bytes": nbytes,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "peak_source": f"{kind} (GB/s)",
                             "traffic": load_traffic(kernel), "kernel": kernel},
                "l2": "flushed between launches"}

    return {"causal_conv1d_silu": line("conv1d_k4_silu_b8_L2048_ch5376_bf16", t_conv, conv_bytes, "conv1d_silu"),
            "gated_rmsnorm": line("gated_rmsnorm_tokens16384_dim5120_bf16", t_norm, norm_bytes, "gated_rmsnorm")}


# ------------------------------------------------------ single-kernel targets for ncu
PROFILE_TARGETS = ("fused", "fused_n64", "fused_n256", "segments", "final_state", "simt", "packed", "decode",
                   "conv", "norm", "seqpar")


def profile_target(name: str, launches: int = 3):
    """Launch one entry point ``launches`` times on the bench's shapes (seeded inputs, L2
    flushed between launches) and nothing else, for one-kernel ncu captures:

    fused       ssd_forward, the Mamba-2-2.7B layer (the fused tensor-core kernel)
    fused_n64   ssd_forward, the state-size sweep at N = 64
    fused_n256  ssd_forward, the state-size sweep at N = 256 (two launches on column halves)
    segments    ssd_forward, the (2, 65536) length-sweep point (cut into segments)
    final_state ssd_forward with y = NULL on the layer workload
    simt        ssd_forward on the SIMT path, the layer workload
    packed      ssd_forward, the packed G = 8 workload (chunk-table kernel + fused kernel)
    decode      ssd_decode_step, 64 sequences at the layer shape
    conv        ssd_causal_conv1d_silu, batch 8 x 2048 x 5376 channels
    norm        ssd_gated_rmsnorm, 16384 tokens x 5120 features
    seqpar      ssd_segment_logdecay and ssd_state_prefix at the layer shape
    """
    import ssd_sequence_mixing_b200 as ssd

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    wl = {"fused": WORKLOAD, "fused_n64": workloads.STATE_SWEEP[2], "fused_n256": workloads.STATE_SWEEP[4],
          "segments": workloads.LENGTH_SWEEP[4], "final_state": WORKLOAD, "simt": WORKLOAD,
          "packed": workloads.PACKED}.get(name)
    if wl is not None:
        prob = workloads.generate(wl, seed=0)
        d = {k: (None if getattr(prob, k) is None else getattr(prob, k).to(dev))
             for k in ("x", "dt", "A", "B", "C", "D", "init_state", "cu_seqlens")}
        if name == "simt":
            ssd.set_path(ssd.PATH_SIMT)
        for _ in range(launches):
            flush.zero_()
            if name == "final_state":
                ssd.ssd_final_state(d["x"], d["dt"], d["A"], d["B"], d["init_state"], d["cu_seqlens"], wl.chunk,
                                    stream=stream)
            else:
                ssd.ssd_forward(d["x"], d["dt"], d["A"], d["B"], d["C"], d["D"], d["init_state"], d["cu_seqlens"],
                                wl.chunk, stream=stream)
    elif name == "decode":
        prob = workloads.generate(DECODE, seed=0)
        x, dt, B, C = (getattr(prob, k)[:, 0].contiguous().to(dev) for k in ("x", "dt", "B", "C"))
        A, D, state = prob.A.to(dev), prob.D.to(dev), prob.init_state.to(dev)
        for _ in range(launches):
            flush.zero_()
            ssd.ssd_decode_step(x, dt, A, B, C, D, state, stream=stream)
    elif name in ("conv", "norm"):
        g = torch.Generator(device=dev).manual_seed(0)
        if name == "conv":
            ch = 5120 + 2 * 128
            xbc = torch.randn((8, 2048, ch), generator=g, device=dev).to(torch.bfloat16)
            w, b = torch.randn((ch, 4), generator=g, device=dev) * 0.5, torch.randn((ch,), generator=g, device=dev)
            out = torch.empty_like(xbc)
            for _ in range(launches):
                flush.zero_()
                ssd.causal_conv1d_silu(xbc, w, b, out=out, stream=stream)
        else:
            y = torch.randn((16384, 5120), generator=g, device=dev).to(torch.bfloat16)
            z = torch.randn((16384, 5120), generator=g, device=dev).to(torch.bfloat16)
            wn = 1.0 + 0.1 * torch.randn((5120,), generator=g, device=dev)
            o = torch.empty_like(y)
            for _ in range(launches):
                flush.zero_()
                ssd.gated_rmsnorm(y, z, wn, out=o, stream=stream)
    elif name == "seqpar":
        prob = workloads.generate(WORKLOAD, seed=0)
        dt, A = prob.dt[0].contiguous().to(dev), prob.A.to(dev)
        H, P, N = WORKLOAD.nheads, WORKLOAD.headdim, WORKLOAD.dstate
        states = torch.randn((8, H, P, N), device=dev) * 0.1
        lams = -torch.rand((8, H), device=dev)
        for _ in range(launches):
            flush.zero_()
            ssd.segment_logdecay(dt, A)
            ssd.state_prefix(7, states, lams, None)
    else:
        raise SystemExit(f"unknown target {name}; one of {PROFILE_TARGETS}")
    torch.cuda.synchronize()
    assert ssd.query_status() == 0
    print(f"profile target {name}: {launches} launches done", flush=True)


# ------------------------------------------------------------ reference arm
def run_reference(args):
    """The fp64 CPU oracle on this workload: each step is a bounded sample (one sequence x
    ``--ref-heads`` heads), reported in token-equivalents of the full workload per second."""
    wl = WORKLOAD
    prob = workloads.generate(wl, seed=0)
    cores = len(os.sched_getaffinity(0))
    H = wl.nheads
    nh = min(args.ref_heads, H)
    times, toks = [], []
    for k in range(args.warmup + args.steps):
        s = k % prob.nseq
        heads = [(k * nh + i) % H for i in range(nh)]
        dt, tk = cpu_oracle_sample(prob, [s], heads, cores)
        if k >= args.warmup:
            times.append(dt)
            toks.append(tk)
    value = sum(toks) / sum(times)
    sample = f"per step 1 sequence x {nh} of {H} heads ({int(toks[0])} token-equivalents), fp64 recurrence"
    return {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
        "config": {"workload": wl.name, "batch": wl.batch, "seq_len": wl.seqlen, "nheads": wl.nheads,
                   "headdim": wl.headdim, "dstate": wl.dstate, "ngroups": wl.ngroups, "chunk": wl.chunk},
        "impl": "reference",
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true",
                    help="skip the measurements of the decode step and the block steps around the SSD")
    ap.add_argument("--profile-target", choices=PROFILE_TARGETS, default=None,
                    help="only launch one entry point a few times (for one-kernel ncu captures) and exit")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload measurements (state-size and length sweeps, packed batch)")
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-heads", type=int, default=16)
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.profile_target:
        profile_target(args.profile_target)
        return

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
