#!/usr/bin/env python3
"""Benchmark of the fused attention forward (one JSON line on stdout).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1..5|decode]
                    [--pass fwd|bwd] [--dtype bf16|fp8] [--impl reference]

A step is one call of the fused forward (the whole hot path) over one batch of
the workload.  The default workload is the causal grouped-query forward at
N = 8192 (B=2, Hq=32, Hkv=8, d=128), the first pure causal d = 128 case with
N >= 8192.  Inputs are seeded synthetic normal bf16 tensors (workloads.py).

Metric: TFLOP/s = 4 * d * (visible query/key pairs) * Hq / time, counting only
unmasked pairs (diagonal included).  Device time comes from CUDA events on the
launching stream; L2 is flushed between timed steps (outside the events).
`e2e` repeats the measurement through the host-buffer C entry point
(attn_fwd_host) with pinned host buffers: host->device copies of q, k, v, the
kernel and device->host copies of o and lse are all inside the timed region.

With N > 1 (torchrun, one process per GPU) every rank runs one batch shard of
the workload's size on its own GPU (weak scaling: the global batch is N times
the workload's); the time is the max over ranks and the value is all ranks'
FLOPs over that time.  --split heads|sequences|auto instead splits ONE
workload over the ranks (strong scaling; exact_attention_142_b200/split.py):
whole GQA groups of heads, or contiguous sequence ranges balanced by their
visible pairs.  There is no collective on the data path either way.

The default run (workload 3) also times the other d = 128 workloads (2, 4, 5)
the same way ("other_workloads") and runs the headline workload back to back
for about 2.5 s with the SM clock sampled ("sustained"), to hold against the
sustained matmul peak; --no-extra skips both.

--impl reference times the CPU oracle (fp64, all host cores) on bounded
samples of the same workload (rank 0 only).

--pass bwd times attn_bwd (dQ, dK, dV) on the same workload instead, with O and
LSE from one untimed attn_fwd; the metric counts five products of 2 * d FLOPs
per visible pair (2.5x the forward's count).

--dtype fp8 times attn_fwd_fp8 (e4m3 inputs) on the same workload, against
the measured bf16 peak x 2 (the nominal fp8 / bf16 tensor-core ratio).

--workload ring times the context-parallel ring forward: one causal sequence of
8192 tokens per rank (B=2, Hq=32, Hkv=8, d=128) split in zigzag chunks, K/V
passed around the ranks with NCCL (weak scaling); on one GPU the ring is one
rank with two chunks.

--workload decode times the key/value-cache decode instead (attn_decode: one
new token for each of 64 sequences against 8192-token paged caches, 32 query
heads over 8 key/value heads, d = 128).  It is bound by HBM, so its metric is
GB/s of algorithmic bytes (every visible cached key and value read once, plus
q, o and lse) against the measured copy bandwidth; a step is one attn_decode
call (the slice kernel and, with more than one slice, the merge kernel).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as W  # noqa: E402

METRIC = "attn fwd TFLOP/s (bf16, causal, d=128) and % of B200 dense BF16 peak"
UNIT = "TFLOP/s"
SPEC_BF16_TFLOPS = 2250.0   # NVIDIA datasheet dense bf16, for context
FALLBACK_BF16_TFLOPS = 1590.0
DECODE_METRIC = "attn decode GB/s (bf16 paged KV cache, d=128) and % of measured HBM bandwidth"
DECODE_UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["exact_attention_142_b200/csrc/attn_fwd_kernel.cuh",
                  "exact_attention_142_b200/csrc/ptx.cuh",
                  "exact_attention_142_b200/csrc/attn_api.cu"]
DECODE_SOURCES = ["exact_attention_142_b200/csrc/attn_decode_kernel.cuh",
                  "exact_attention_142_b200/csrc/ptx.cuh",
                  "exact_attention_142_b200/csrc/attn_decode_api.cu"]


def visible_pairs(w: W.Workload) -> int:
    """Number of visible (query, key) pairs per head, summed over sequences."""
    right = 0 if w.causal else w.window_right
    left = w.window_left
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    total = 0
    for L in lengths:
        i = np.arange(L, dtype=np.int64)
        lo = np.zeros(L, np.int64) if left < 0 else np.maximum(0, i - left)
        hi = np.full(L, L - 1, np.int64) if right < 0 else np.minimum(L - 1, i + right)
        total += int((hi - lo + 1).sum())
    return total


def flops_of(w: W.Workload) -> float:
    return 4.0 * w.d * visible_pairs(w) * w.Hq


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {}, "fallback"


def kernel_sources_digest(sources=None) -> str:
    h = hashlib.sha256()
    for rel in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str, prefix: str = "attn_fwd", sources=None):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", f"{prefix}_{workload_name}_traffic.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", text)
    s = re.search(r"kernel_sources_sha256_16:\s*([0-9a-f]+)", text)
    if not m or not s or s.group(1) != kernel_sources_digest(sources):
        return None
    return float(m.group(1))


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.sw_power_cap,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.lines = []
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._thr = threading.Thread(target=self._read, daemon=True)
            self._thr.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark_begin(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sel = [l for (t, l) in self.lines if self.t0 is None or (self.t0 <= t <= (self.t1 or t) + 0.06)]
        if not sel:
            sel = [l for (_, l) in self.lines]
        sm, mx, pw = [], [], []
        reasons = set()
        names = ["sw_power_cap", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown"]
        for l in sel:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
                pw.append(float(parts[3]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "power_w_max": max(pw) if pw else None,
                "samples": len(sm),
                "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# CUDA arm
# ---------------------------------------------------------------------------
def run_cuda(args, w: W.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import exact_attention_142_b200 as ea

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ea.load_library()
    q, k, v = W.inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o = torch.empty_like(qd)
    if w.packed:
        cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=dev)
        lse = torch.empty((w.Hq, w.tokens), dtype=torch.float32, device=dev)
    else:
        cu = None
        lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ea.attn_fwd(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                    w.window_left, w.window_right, cu, w.max_seqlen, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a timeout during warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for i in range(args.steps):
        flush.zero_()  # evict L2 (outside the timed events)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    times = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    kernel_ms = sum(times) / len(times)
    status = ea.attn_device_status()
    if status != ea.ATTN_OK:
        raise RuntimeError(f"device status {status} during the timed region")

    # End to end through the host-buffer entry point, as a serving loop runs it:
    # two streams, each with its own device workspace and pinned output
    # buffers, take alternate steps, so one step's copies overlap the other's
    # kernel.  Every step still copies its inputs in and its O and LSE out; the
    # events bracket all the steps.
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    slots = 2
    ohs = [torch.empty_like(qh).pin_memory() for _ in range(slots)]
    lhs = [torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory() for _ in range(slots)]
    cuh = torch.tensor(w.cu_seqlens, dtype=torch.int32) if w.packed else None
    nbytes = ea.attn_fwd_host_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d, w.packed)
    del qd, kd, vd, o
    wss = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(slots)]
    streams = [torch.cuda.Stream(dev) for _ in range(slots)]

    def e2e_step(i):
        j = i % slots
        ea.attn_fwd_host(qh, kh, vh, ohs[j], lhs[j], w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                         w.window_left, w.window_right, cuh, w.max_seqlen, wss[j], nbytes, streams[j])

    for i in range(max(2, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_steps = max(4, min(args.steps, 20))
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    e_start.record(stream)
    for st in streams:
        st.wait_event(e_start)
    for i in range(e_steps):
        e2e_step(i)
    for st in streams:
        stream.wait_stream(st)
    e_end.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e_start.elapsed_time(e_end) / e_steps
    oh, lh = ohs[0], lhs[0]
    h2d = (q.numel() + k.numel() + v.numel()) * 2 + (4 * len(w.cu_seqlens) if w.packed else 0)
    d2h = oh.numel() * 2 + lh.numel() * 4

    clocks = sampler.stop() if sampler else None
    # max over ranks
    if world > 1:
        t = torch.tensor([kernel_ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        kernel_ms, e2e_ms = float(t[0]), float(t[1])
    run_cuda.step_times = sorted(times)
    return kernel_ms, e2e_ms, h2d, d2h, clocks


def time_forward(w: W.Workload, dev, steps: int, warmup: int, flush=None):
    """attn_fwd on one workload, timed like the benchmark's steps (L2 flushed
    between calls, outside the events): the per-call times in ms."""
    import torch

    import exact_attention_142_b200 as ea
    q, k, v = W.inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    del q, k, v
    o = torch.empty_like(qd)
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=dev) if w.packed else None
    lse = torch.empty((w.Hq, w.tokens) if w.packed else (w.B, w.Hq, w.N), dtype=torch.float32,
                      device=dev)
    if flush is None:
        flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: ea.attn_fwd(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale,  # noqa: E731
                               w.causal, w.window_left, w.window_right, cu, w.max_seqlen, stream)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize(dev)
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError(f"device status reported an error on {w.name}")
    return [a.elapsed_time(b) for a, b in ev]


def other_workloads(dev, steps: int, warmup: int, peak: float):
    """The other d = 128 workloads, each timed like the headline one."""
    out = {}
    for cfg in (2, 4, 5):
        w = W.workload(cfg)
        times = time_forward(w, dev, steps, warmup)
        ms = sum(times) / len(times)
        tf = flops_of(w) / (ms * 1e-3) / 1e12
        out[w.name] = {"ms_per_step": ms, "steps": steps, "value": tf, "unit": UNIT,
                       "frac": tf / peak, "frac_of_spec_2250": tf / SPEC_BF16_TFLOPS,
                       "step_ms": step_stats(times), "flop_per_step": flops_of(w),
                       "gpu_launches": steps, "l2": "flushed between timed steps"}
    return out


def sustained_forward(w: W.Workload, dev, seconds: float, peak_sustained: float):
    """Back-to-back calls (no flush; the inputs, 2x the L2, stream through it)
    for at least `seconds`, under the power cap, with the SM clock sampled
    over the loop: the figure to hold against the sustained matmul peak."""
    import torch

    import exact_attention_142_b200 as ea
    q, k, v = W.inputs(w)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    del q, k, v
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.Hq, w.N), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    call = lambda: ea.attn_fwd(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale,  # noqa: E731
                               w.causal, w.window_left, w.window_right, None, 0, stream)
    for _ in range(5):
        call()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(10):
        call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    n = max(20, int(seconds / (a.elapsed_time(b) / 10 * 1e-3)))
    sampler = ClockSampler(dev.index)
    sampler.start()
    time.sleep(0.3)
    sampler.mark_begin()
    a.record(stream)
    for _ in range(n):
        call()
    b.record(stream)
    torch.cuda.synchronize(dev)
    sampler.mark_end()
    clocks = sampler.stop()
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported an error in the sustained loop")
    ms = a.elapsed_time(b) / n
    tf = flops_of(w) / (ms * 1e-3) / 1e12
    return {"workload": w.name, "value": tf, "unit": UNIT, "ms_per_step": ms, "steps": n,
            "seconds": ms * n * 1e-3, "gpu_launches": n,
            "frac_of_sustained": (tf / peak_sustained) if peak_sustained else None,
            "peak_sustained": peak_sustained, "frac_of_spec_2250": tf / SPEC_BF16_TFLOPS,
            "clocks": clocks, "l2": "not flushed (back-to-back calls; inputs 2.7x L2)"}


# ---------------------------------------------------------------------------
# key/value-cache decode
# ---------------------------------------------------------------------------
def decode_visible_keys(w: W.DecodeWorkload) -> int:
    """Cached keys that at least one query row of a sequence sees, summed over
    sequences (each is read once per key/value head)."""
    right = 0 if w.causal else w.window_right
    total = 0
    for L in w.lengths:
        lo = 0 if w.window_left < 0 else max(0, L - w.Nq - w.window_left)
        hi = L - 1 if right < 0 else min(L - 1, L - 1 + right)
        total += max(0, hi - lo + 1)
    return total


def decode_bytes(w: W.DecodeWorkload) -> float:
    kv = 2.0 * decode_visible_keys(w) * w.Hkv * w.d * 2
    qo = 2.0 * w.B * w.Nq * w.Hq * w.d * 2
    return kv + qo + 4.0 * w.B * w.Hq * w.Nq


def run_decode(args, w: W.DecodeWorkload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import exact_attention_142_b200 as ea

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ea.load_library()
    q, kc, vc, seqlens, table = W.decode_inputs(w, device="cuda")
    sd, td = seqlens.to(dev), table.to(dev) if table is not None else None
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=dev)
    splits = args.splits or ea.attn_decode_default_splits(w.B, w.Hq, w.Hkv, w.Nq, w.max_len)
    nbytes = ea.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                                            w.pages_per_seq, splits)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ea.attn_decode(q, kc, vc, o, lse, sd, td, w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                       w.pages_per_seq, kc.shape[0], w.scale, w.causal, w.window_left,
                       w.window_right, splits, ws if nbytes else None, nbytes, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    kernel_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a failure during the timed region")

    # end to end: pinned host inputs copied in, result copied out, every step
    host = [t.cpu().pin_memory() for t in (q, kc, vc, seqlens)]
    host_table = table.pin_memory() if table is not None else None
    oh = torch.empty(tuple(o.shape), dtype=o.dtype).pin_memory()
    lh = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()
    devs = [q, kc, vc, sd]

    def e2e_step():
        for hsrc, ddst in zip(host, devs):
            ddst.copy_(hsrc, non_blocking=True)
        if host_table is not None:
            td.copy_(host_table, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e_steps = max(3, min(args.steps, 10))
    es = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps)]
    if world > 1:
        dist.barrier()
    for i in range(e_steps):
        es[i].record(stream)
        e2e_step()
        ee[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(s.elapsed_time(e) for s, e in zip(es, ee)) / e_steps
    h2d = sum(t.numel() * t.element_size() for t in host) + (
        host_table.numel() * 4 if host_table is not None else 0)
    d2h = oh.numel() * 2 + lh.numel() * 4
    clocks = sampler.stop() if sampler else None
    if world > 1:
        t = torch.tensor([kernel_ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        kernel_ms, e2e_ms = float(t[0]), float(t[1])
    launches = args.steps * (2 if nbytes else 1)
    return kernel_ms, e2e_ms, h2d, d2h, clocks, splits, launches


def decode_oracle_sample(w: W.DecodeWorkload, inputs, nseq: int, seed: int):
    """Time the oracle on `nseq` sequences drawn from the workload; returns
    (seconds, algorithmic bytes of those sequences, threads)."""
    import oracle
    q, kc, vc, seqlens, table = inputs
    rng = np.random.default_rng(seed)
    pick = np.sort(rng.choice(w.B, size=nseq, replace=False))
    sub = W.DecodeWorkload("sample", nseq, w.Hq, w.Hkv, w.Nq, w.d, w.page_size, w.pages_per_seq,
                           [w.lengths[b] for b in pick], w.paged, w.causal, w.window_left,
                           w.window_right, w.seed)
    t0 = time.perf_counter()
    oracle.attn_kvcache(W.bf16_bits(q[pick]), W.bf16_bits(kc), W.bf16_bits(vc),
                        seqlens.numpy()[pick], B=nseq, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, d=w.d,
                        page_size=w.page_size, pages_per_seq=w.pages_per_seq, scale=w.scale,
                        causal=w.causal, window_left=w.window_left, window_right=w.window_right,
                        block_table=None if table is None else table.numpy()[pick])
    return time.perf_counter() - t0, decode_bytes(sub), oracle.num_threads()


def decode_host_inputs(w: W.DecodeWorkload):
    """The benchmark's inputs (drawn with the CUDA generator) brought to the host."""
    return tuple(t.cpu() if t is not None else None for t in W.decode_inputs(w, device="cuda"))


def decode_cpu_baseline(w: W.DecodeWorkload, inputs, target_s: float = 12.0):
    """The oracle on whole batches of the workload, repeated until about
    target_s seconds of CPU work."""
    tot_t, tot_b, reps, thr = 0.0, 0.0, 0, 1
    while tot_t < target_s and reps < 1000:
        dt, by, thr = decode_oracle_sample(w, inputs, w.B, seed=2 + reps)
        tot_t += dt
        tot_b += by
        reps += 1
    return {"value": tot_b / tot_t / 1e9, "unit": DECODE_UNIT, "cores": thr, "kind": "oracle",
            "sample": f"{reps} passes over all {w.B} sequences (all heads, full caches), "
                      f"fp64 oracle, {tot_t:.1f} s on {thr} threads"}


def decode_config(w: W.DecodeWorkload, n_gpus: int, splits: int):
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "Nq": w.Nq, "d": w.d,
            "cache_len": max(w.lengths), "page_size": w.page_size, "paged": w.paged,
            "causal": w.causal, "window": [w.window_left, w.window_right],
            "num_splits": splits, "bytes_per_step": decode_bytes(w),
            "l2": "flushed between timed steps (the caches are 17x L2 as well)",
            "parallelism": f"replicas x{n_gpus} (no collective)"}


def main_decode(args, rank, world, local_rank):
    w = W.decode_workload(args.decode_batch)
    if args.impl == "reference":
        if rank != 0:
            return
        inputs = decode_host_inputs(w)
        budget_s = 150.0 / max(1, args.steps + args.warmup)
        dt, _, _ = decode_oracle_sample(w, inputs, 1, seed=1)
        nseq = int(max(1, min(w.B, round(min(budget_s, 30.0) / max(dt, 1e-6)))))
        for i in range(args.warmup):
            decode_oracle_sample(w, inputs, nseq, seed=10 + i)
        tot_t, tot_b, thr = 0.0, 0.0, 1
        for i in range(args.steps):
            dt, by, thr = decode_oracle_sample(w, inputs, nseq, seed=1000 + i)
            tot_t += dt
            tot_b += by
        value = tot_b / tot_t / 1e9
        print(json.dumps({
            "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": decode_config(w, args.gpus, 0), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": DECODE_UNIT, "cores": thr, "kind": "oracle",
                             "sample": f"{nseq} sequences per step; fp64 oracle on {thr} threads"},
            "e2e": {"value": value, "unit": DECODE_UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        kernel_ms, e2e_ms, h2d, d2h, clocks, splits, launches = run_decode(
            args, w, rank, world, local_rank)
    finally:
        if world > 1:
            dist.barrier()
    if rank == 0:
        by = decode_bytes(w)
        achieved = by / (kernel_ms * 1e-3) / 1e9
        peaks, src = measured_peaks()
        peak = float(peaks.get("hbm_gbs", FALLBACK_HBM_GBS))
        line = {
            "metric": DECODE_METRIC, "value": achieved * world, "unit": DECODE_UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": kernel_ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 q and caches, random page table)",
            "config": decode_config(w, world, splits),
            "e2e": {"value": by * world / (e2e_ms * 1e-3) / 1e9, "unit": DECODE_UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": launches,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak,
                         "traffic": recorded_traffic(w.name, "attn_decode", DECODE_SOURCES)
                         if splits == 1 else None,
                         "peak_source": f"{src} hbm_gbs (copy)" if src == "measured"
                         else "fallback 6650 GB/s",
                         "kernel": "attn_decode_tma<128,3>"
                                   + (" + attn_decode_combine<128>" if splits > 1 else ""),
                         "timed_as": "whole attn_decode call (both kernels)"},
            "clocks": clocks,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = decode_cpu_baseline(w, decode_host_inputs(w))
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# oracle (CPU) timing
# ---------------------------------------------------------------------------
def oracle_sample(w: W.Workload, q, k, v, nrows: int, seed: int):
    """Time the oracle on `nrows` (sequence, head, row) triples drawn uniformly
    from the workload; returns (seconds, flops of those rows, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    cum = np.cumsum([0] + lengths)
    flat = rng.integers(0, cum[-1], size=nrows)
    b = np.searchsorted(cum, flat, side="right") - 1
    i = flat - cum[b]
    h = rng.integers(0, w.Hq, size=nrows)
    rows = np.stack([b, h, i], axis=1).astype(np.int64)
    qb, kb, vb = W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v)
    t0 = time.perf_counter()
    _, _, nvis = oracle.attn_fwd(qb, kb, vb, B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d,
                                 scale=w.scale, causal=w.causal, window_left=w.window_left,
                                 window_right=w.window_right, cu_seqlens=w.cu_seqlens, rows=rows)
    dt = time.perf_counter() - t0
    return dt, 4.0 * w.d * float(nvis.sum()), oracle.num_threads()


def calibrate_rows(w, q, k, v, target_s: float) -> int:
    rows = 64
    dt, _, _ = oracle_sample(w, q, k, v, rows, seed=1)
    while dt < 0.5 and rows < (1 << 22):
        rows *= 4
        dt, _, _ = oracle_sample(w, q, k, v, rows, seed=1)
    return max(16, int(rows * target_s / max(dt, 1e-6)))


def run_torch_sdpa(args, w: W.Workload):
    """Context line: PyTorch's scaled_dot_product_attention on the same dense
    workload (inputs as [B, H, N, d] copies), each backend that accepts it,
    timed like the CUDA arm.  Sliding windows and packed sequences have no
    direct SDPA form, so those workloads are reported unavailable."""
    import torch
    import torch.nn.functional as F
    from torch.nn.attention import SDPBackend, sdpa_kernel

    base = {"metric": METRIC, "unit": UNIT, "impl": "torch_sdpa (context, not this library)",
            "config": config_dict(w, 1), "n_gpus": 1}
    if w.packed or w.window_left >= 0 or (not w.causal and w.window_right >= 0):
        return base | {"unavailable": "no sliding-window or packed form in scaled_dot_product_attention"}
    dev = torch.device("cuda", 0)
    q, k, v = W.inputs(w)
    qd, kd, vd = (t.to(dev).transpose(1, 2).contiguous() for t in (q, k, v))
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    fl = flops_of(w)
    results = {}
    backends = [("flash", SDPBackend.FLASH_ATTENTION), ("cudnn", SDPBackend.CUDNN_ATTENTION),
                ("efficient", SDPBackend.EFFICIENT_ATTENTION)]
    for name, be in backends:
        if args.sdpa_backend not in ("all", name):
            continue
        try:
            with sdpa_kernel([be]):
                def call():
                    return F.scaled_dot_product_attention(qd, kd, vd, is_causal=w.causal, scale=w.scale,
                                                          enable_gqa=w.Hq != w.Hkv)
                for _ in range(args.warmup):
                    call()
                torch.cuda.synchronize(dev)
                times = []
                for _ in range(min(args.steps, 20)):
                    flush.zero_()
                    a = torch.cuda.Event(enable_timing=True)
                    b = torch.cuda.Event(enable_timing=True)
                    a.record()
                    call()
                    b.record()
                    torch.cuda.synchronize(dev)
                    times.append(a.elapsed_time(b))
            ms = sum(times) / len(times)
            results[name] = {"ms": ms, "value": fl / (ms * 1e-3) / 1e12}
        except RuntimeError as e:  # backend not available for this shape or device
            results[name] = {"unavailable": str(e).splitlines()[0][:160]}
    ok = [r["value"] for r in results.values() if "value" in r]
    return base | {"value": max(ok) if ok else None, "backends": results,
                   "higher_is_better": True, "dtype": "bf16"}


def step_stats(times):
    """Median and minimum of the timed steps (rank 0), beside the mean that
    ms_per_step reports."""
    if not times:
        return None
    t = sorted(times)
    return {"mean": sum(t) / len(t), "median": t[len(t) // 2], "min": t[0], "max": t[-1],
            "rank": 0}


def host_cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w: W.Workload, target_s: float = 12.0):
    q, k, v = W.inputs(w)
    rows = calibrate_rows(w, q, k, v, target_s)
    dt, fl, thr = oracle_sample(w, q, k, v, rows, seed=2)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
            "cpu_model": host_cpu_model(),
            "sample": f"{rows} query rows drawn uniformly over (sequence, head, row) of the "
                      f"workload, fp64 oracle, {dt:.1f} s on {thr} threads"}


def run_reference(args, w: W.Workload):
    """The oracle as the reference arm: K timed steps, each a bounded sample."""
    q, k, v = W.inputs(w)
    budget_s = 150.0 / max(1, args.steps + args.warmup)
    rows = calibrate_rows(w, q, k, v, min(budget_s, 30.0))
    for i in range(args.warmup):
        oracle_sample(w, q, k, v, rows, seed=10 + i)
    tot_t, tot_f, thr = 0.0, 0.0, 1
    for i in range(args.steps):
        dt, fl, thr = oracle_sample(w, q, k, v, rows, seed=1000 + i)
        tot_t += dt
        tot_f += fl
    value = tot_f / tot_t / 1e12
    return {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(w, args.gpus), "impl": "reference",
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                         "sample": f"{rows} query rows per step, drawn uniformly over "
                                   f"(sequence, head, row); fp64 oracle on {thr} threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# backward pass
# ---------------------------------------------------------------------------
BWD_METRIC = "attn bwd TFLOP/s (bf16, dQ dK dV, 2.5x the forward's pair count) and % of B200 dense BF16 peak"


def bwd_flops_of(w: W.Workload) -> float:
    """Five products (S, dP, dV, dK, dQ) of 2 * d FLOPs per visible pair: 2.5x the forward."""
    return 10.0 * w.d * visible_pairs(w) * w.Hq


def draw_dout(w: W.Workload, q):
    import torch
    g = torch.Generator().manual_seed(w.seed + 1000)
    return torch.randn(tuple(q.shape), dtype=torch.float32, generator=g).to(torch.bfloat16)


def run_bwd(args, w: W.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    import exact_attention_142_b200 as ea

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ea.load_library()
    q, k, v = W.inputs(w)
    do = draw_dout(w, q)
    qd, kd, vd, dod = (t.to(dev) for t in (q, k, v, do))
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=dev) if w.packed else None
    o = torch.empty_like(qd)
    lse = torch.empty((w.Hq * w.tokens,), dtype=torch.float32, device=dev)
    ea.attn_fwd(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                w.window_left, w.window_right, cu, w.max_seqlen)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    nbytes = ea.attn_bwd_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d, w.packed)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ea.attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale,
                    w.causal, w.window_left, w.window_right, cu, w.max_seqlen, ws, nbytes, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a timeout during warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    kernel_ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a timeout during the timed region")

    # end to end: the step's inputs (q, k, v, o, lse, dout) copied in from pinned
    # host memory and the three gradients copied out, every step
    host_in = [t.cpu().pin_memory() for t in (qd, kd, vd, o, lse, dod)]
    dev_in = [qd, kd, vd, o, lse, dod]
    host_out = [torch.empty(tuple(t.shape), dtype=t.dtype).pin_memory() for t in (dq, dk, dv)]

    def e2e_step():
        for h, d_ in zip(host_in, dev_in):
            d_.copy_(h, non_blocking=True)
        step()
        for h, d_ in zip(host_out, (dq, dk, dv)):
            h.copy_(d_, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize(dev)
    e_steps = max(3, min(args.steps, 20))
    es = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(e_steps)]
    if world > 1:
        dist.barrier()
    for i in range(e_steps):
        es[i].record(stream)
        e2e_step()
        ee[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(es, ee)) / e_steps
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        t = torch.tensor([kernel_ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        kernel_ms, e2e_ms = float(t[0]), float(t[1])
    return kernel_ms, e2e_ms, h2d, d2h, clocks


def bwd_oracle_sample(w: W.Workload, q, k, v, do, L: int, seed: int):
    """The oracle's backward on a prefix of L tokens of one sequence and one
    key/value head group; returns (seconds, algorithmic FLOPs of it, threads)."""
    import oracle
    rng = np.random.default_rng(seed)
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    b = int(rng.integers(len(lengths)))
    while lengths[b] == 0:
        b = int(rng.integers(len(lengths)))
    g = int(rng.integers(w.Hkv))
    L = min(L, lengths[b])
    grp = w.Hq // w.Hkv
    start = w.cu_seqlens[b] if w.packed else 0

    def cut(t, heads):
        if w.packed:
            x = t[start:start + L, heads]
        else:
            x = t[b, :L, heads]
        return x.unsqueeze(0).contiguous()

    hq = slice(g * grp, (g + 1) * grp)
    hk = slice(g, g + 1)
    sub = W.Workload("sample", 1, grp, 1, L, w.d, w.causal, w.window_left, w.window_right, 0)
    t0 = time.perf_counter()
    oracle.attn_bwd(W.bf16_bits(cut(q, hq)), W.bf16_bits(cut(k, hk)), W.bf16_bits(cut(v, hk)),
                    W.bf16_bits(cut(do, hq)), B=1, Hq=grp, Hkv=1, N=L, d=w.d, scale=w.scale,
                    causal=w.causal, window_left=w.window_left, window_right=w.window_right)
    return time.perf_counter() - t0, bwd_flops_of(sub), oracle.num_threads()


def bwd_calibrate(w, q, k, v, do, target_s):
    L = 256
    dt, _, _ = bwd_oracle_sample(w, q, k, v, do, L, seed=1)
    while dt < 0.5 and L < w.max_seqlen:
        L *= 2
        dt, _, _ = bwd_oracle_sample(w, q, k, v, do, L, seed=1)
    # cost grows with L^2 (causal) or L * window
    return max(64, min(w.max_seqlen, int(L * math.sqrt(target_s / max(dt, 1e-6)))))


def bwd_cpu_baseline(w: W.Workload, target_s: float = 12.0):
    q, k, v = W.inputs(w)
    do = draw_dout(w, q)
    L = bwd_calibrate(w, q, k, v, do, target_s)
    dt, fl, thr = bwd_oracle_sample(w, q, k, v, do, L, seed=2)
    return {"value": fl / dt / 1e12, "unit": UNIT, "cores": thr, "kind": "oracle",
            "sample": f"the first {L} tokens of one sequence, one key/value head group "
                      f"({w.Hq // w.Hkv} query heads), fp64 oracle backward, {dt:.1f} s "
                      f"on {thr} threads"}


def main_bwd(args, w: W.Workload, rank, world, local_rank):
    if args.impl == "reference":
        if rank != 0:
            return
        q, k, v = W.inputs(w)
        do = draw_dout(w, q)
        budget_s = 150.0 / max(1, args.steps + args.warmup)
        L = bwd_calibrate(w, q, k, v, do, min(budget_s, 30.0))
        for i in range(args.warmup):
            bwd_oracle_sample(w, q, k, v, do, L, seed=10 + i)
        tot_t, tot_f, thr = 0.0, 0.0, 1
        for i in range(args.steps):
            dt, fl, thr = bwd_oracle_sample(w, q, k, v, do, L, seed=1000 + i)
            tot_t += dt
            tot_f += fl
        value = tot_f / tot_t / 1e12
        print(json.dumps({
            "metric": BWD_METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": tot_t / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(config_dict(w, args.gpus), **{"pass": "bwd"}),
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": thr, "kind": "oracle",
                             "sample": f"a {L}-token prefix of one sequence and head group "
                                       f"per step; fp64 oracle on {thr} threads"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}), flush=True)
        return
    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        kernel_ms, e2e_ms, h2d, d2h, clocks = run_bwd(args, w, rank, world, local_rank)
    finally:
        if world > 1:
            dist.barrier()
    if rank == 0:
        fl = bwd_flops_of(w)
        achieved = fl / (kernel_ms * 1e-3) / 1e12
        peaks, src = measured_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        line = {
            "metric": BWD_METRIC, "value": achieved * world, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": kernel_ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 Q, K, V, dO; O and LSE from attn_fwd)",
            "config": dict(config_dict(w, world), **{"pass": "bwd", "flop_per_step": fl}),
            "e2e": {"value": fl * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": 3 * args.steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{src} bf16_tflops (burst, cuBLAS)" if src == "measured"
                         else "fallback 1590 TF/s",
                         "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                         "kernel": f"attn_bwd_dsum<{w.d}> + attn_bwd_dkv<{w.d}> + attn_bwd_dq<{w.d}>",
                         "timed_as": "whole attn_bwd call (three kernels)"},
            "clocks": clocks,
        }
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = bwd_cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# context-parallel ring forward
# ---------------------------------------------------------------------------
RING_METRIC = "attn ring fwd TFLOP/s (bf16, causal, d=128, sequence split across GPUs)"


def ring_workload(world: int) -> W.Workload:
    """8192 tokens per rank (two zigzag chunks of 4096) of one causal GQA
    sequence per batch entry: B=2, Hq=32, Hkv=8, d=128, N = 8192 * world."""
    return W.Workload(f"ring_causal_gqa_b2_hq32_hkv8_n{8192 * world}_d128", 2, 32, 8, 8192 * world,
                      128, True, -1, -1, 6)


def main_ring(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import exact_attention_142_b200 as ea
    from exact_attention_142_b200 import ring

    w = ring_workload(world)
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "unavailable":
                              "the ring's reference arm is the oracle forward on the whole "
                              "sequence; see --workload 3 --impl reference"}), flush=True)
        return
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    ea.load_library()
    # this rank's chunks only: draw the rank's slice of a seeded sequence
    C = w.N // (2 * world)
    g = torch.Generator(device="cuda").manual_seed(w.seed)
    full = [torch.randn((w.B, w.N, h, w.d), generator=g, device=dev).to(torch.bfloat16)
            for h in (w.Hq, w.Hkv, w.Hkv)]
    qs, ks, vs = (ring.shard_zigzag(t, world, rank) for t in full)
    del full
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def step():
        return ring.ring_attention_forward(qs, ks, vs, scale=w.scale, causal=True,
                                           group=None, stream=stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a timeout during the timed region")
    # end to end: this rank's chunks from pinned host memory, O and LSE back
    host_in = [t.cpu().pin_memory() for t in (*qs, *ks, *vs)]
    dev_in = [*qs, *ks, *vs]

    def e2e_step():
        for h, d_ in zip(host_in, dev_in):
            d_.copy_(h, non_blocking=True)
        outs, lses = step()
        return [x.to("cpu", non_blocking=True) for x in (*outs, *lses)]

    e2e_step()
    torch.cuda.synchronize(dev)
    es = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    if world > 1:
        dist.barrier()
    for i in range(5):
        es[i].record(stream)
        res = e2e_step()
        ee[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(es, ee)) / 5
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in res)
    clocks = sampler.stop() if sampler else None
    if world > 1:
        t = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms = float(t[0]), float(t[1])
    if rank == 0:
        fl = flops_of(w)
        achieved = fl / world / (ms * 1e-3) / 1e12
        peaks, src = measured_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        pairs = sum(len(pp) for _, _, pp in ring.ring_schedule(world, 0, True))
        print(json.dumps({
            "metric": RING_METRIC, "value": fl / (ms * 1e-3) / 1e12, "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 Q, K, V drawn on the device)",
            "config": {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N,
                       "d": w.d, "causal": True, "tokens_per_rank": 2 * C,
                       "chunk_pairs_per_rank": pairs, "flop_per_step": fl,
                       "l2": "flushed between timed steps",
                       "parallelism": f"context parallel x{world} (zigzag ring, NCCL send/recv)"},
            "e2e": {"value": fl / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d * world, "d2h_bytes_per_step": d2h * world},
            "gpu_launches": (pairs + 2) * args.steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": f"{src} bf16_tflops (burst, cuBLAS)" if src == "measured"
                         else "fallback 1590 TF/s",
                         "kernel": "attn_fwd_sm100<128,4,accumulate> + attn_acc_to_bf16",
                         "timed_as": "whole ring step per rank (all chunk pairs, transfers, cast)"},
            "clocks": clocks,
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# e4m3 inputs
# ---------------------------------------------------------------------------
FP8_METRIC = "attn fwd TFLOP/s (e4m3 inputs, causal, d=128) and % of B200 dense FP8 peak"


def main_fp8(args, w: W.Workload, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from datetime import timedelta

    import exact_attention_142_b200 as ea
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps({"impl": "reference", "unavailable":
                              "the e4m3 path's reference arm is the oracle on the widened "
                              "values; see --impl reference for the bf16 workload"}), flush=True)
        return
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)
    ea.load_library()
    if w.packed:
        q, k, v = W.draw_qkv_e4m3((w.tokens, w.Hq, w.d), (w.tokens, w.Hkv, w.d), w.seed)
    else:
        q, k, v = W.draw_qkv_e4m3((w.B, w.N, w.Hq, w.d), (w.B, w.N, w.Hkv, w.d), w.seed)
    qd, kd, vd = (t.view(torch.uint8).to(dev) for t in (q, k, v))
    cu = torch.tensor(w.cu_seqlens, dtype=torch.int32, device=dev) if w.packed else None
    o = torch.empty(tuple(q.shape), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.Hq * w.tokens,), dtype=torch.float32, device=dev)
    nbytes = ea.attn_fwd_fp8_workspace_bytes(w.B, w.Hq, w.Hkv, w.N, w.d, w.packed)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        ea.attn_fwd_fp8(qd, kd, vd, o, lse, w.B, w.Hq, w.Hkv, w.N, w.d, w.scale, w.causal,
                        w.window_left, w.window_right, cu, w.max_seqlen, ws, nbytes, stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for i in range(args.steps):
        flush.zero_()
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    ms = sum(a.elapsed_time(b) for a, b in zip(starts, ends)) / args.steps
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported a timeout during the timed region")
    host_in = [t.view(torch.uint8).pin_memory() for t in (q, k, v)]
    oh = torch.empty(tuple(o.shape), dtype=o.dtype).pin_memory()
    lh = torch.empty(tuple(lse.shape), dtype=torch.float32).pin_memory()

    def e2e_step():
        for h, d_ in zip(host_in, (qd, kd, vd)):
            d_.copy_(h, non_blocking=True)
        step()
        oh.copy_(o, non_blocking=True)
        lh.copy_(lse, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize(dev)
    es = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    ee = [torch.cuda.Event(enable_timing=True) for _ in range(10)]
    if world > 1:
        dist.barrier()
    for i in range(10):
        es[i].record(stream)
        e2e_step()
        ee[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(es, ee)) / 10
    clocks = sampler.stop() if sampler else None
    if world > 1:
        t = torch.tensor([ms, e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms, e2e_ms = float(t[0]), float(t[1])
    if rank == 0:
        fl = flops_of(w)
        achieved = fl / (ms * 1e-3) / 1e12
        peaks, src = measured_peaks()
        peak = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        print(json.dumps({
            "metric": FP8_METRIC, "value": achieved * world, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "e4m3",
            "data": "synthetic (seeded normal draws rounded to e4m3)",
            "config": dict(config_dict(w, world), **{"inputs": "e4m3"}),
            "e2e": {"value": fl * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": sum(t.numel() for t in host_in),
                    "d2h_bytes_per_step": oh.numel() * 2 + lh.numel() * 4},
            "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": None,
                         "peak_source": (f"{src} bf16_tflops x 2 (nominal fp8 / bf16 ratio)"
                                         if src == "measured" else "fallback 1590 x 2"),
                         "frac_of_bf16_peak": achieved / (peak / 2),
                         "kernel": "attn_vt_transpose_kernel + attn_fwd_fp8_sm100",
                         "timed_as": "whole attn_fwd_fp8 call (transpose + kernel)"},
            "clocks": clocks,
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()


def config_dict(w: W.Workload, n_gpus: int, split_mode: str = "none"):
    par = (f"one batch shard per rank x{n_gpus} (no collective)" if split_mode == "none"
           else f"{split_mode} split of one workload over {n_gpus} ranks (no collective)")
    return {"workload": w.name, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
            "N": w.N if not w.packed else None, "tokens": w.tokens, "d": w.d,
            "causal": w.causal, "window": [w.window_left, w.window_right],
            "packed_sequences": len(w.cu_seqlens) - 1 if w.packed else None,
            "flop_per_step": flops_of(w), "l2": "flushed between timed steps",
            "parallelism": par}


def main_split(args, w: W.Workload, rank, world, local_rank):
    """One workload split over the ranks (heads or sequences): each rank runs
    attn_fwd on its shard; the time is the slowest rank's, the value the whole
    workload's FLOPs over it (strong scaling)."""
    import torch
    import torch.distributed as dist

    import exact_attention_142_b200 as ea
    from exact_attention_142_b200 import split

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    ea.load_library()
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    shards = split.plan(world, args.split, B=w.B, Hq=w.Hq, Hkv=w.Hkv, lengths=lengths,
                        causal=w.causal, left=w.window_left, right=w.window_right)
    sh = shards[rank]
    q, k, v = W.inputs(w)
    qs, ks, vs, cu, B, Hq, Hkv = split.shard_inputs(q, k, v, sh, w.cu_seqlens if w.packed else None)
    del q, k, v
    my_flops = 0.0
    if not sh.empty:
        my_lengths = lengths[sh.seqs[0]:sh.seqs[1]]
        my_flops = 4.0 * w.d * Hq * sum(split.visible_pairs(L, w.causal, w.window_left,
                                                            w.window_right) for L in my_lengths)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    times = [0.0] * args.steps
    if not sh.empty:
        qd, kd, vd = qs.to(dev), ks.to(dev), vs.to(dev)
        N = qd.shape[0] if cu is not None else w.N
        o = torch.empty_like(qd)
        lse = torch.empty((Hq, N) if cu is not None else (B, Hq, N), dtype=torch.float32, device=dev)
        cud = torch.tensor(cu, dtype=torch.int32, device=dev) if cu is not None else None
        max_len = max(lengths[sh.seqs[0]:sh.seqs[1]])

        def step():
            ea.attn_fwd(qd, kd, vd, o, lse, B, Hq, Hkv, N, w.d, w.scale, w.causal, w.window_left,
                        w.window_right, cud, max_len, stream)
    else:
        def step():
            pass
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    sampler = ClockSampler(dev.index) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_begin()
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.mark_end()
    times = [a.elapsed_time(b) for a, b in ev]
    if ea.attn_device_status() != ea.ATTN_OK:
        raise RuntimeError("device status reported an error during the timed region")
    ms = sum(times) / len(times)
    clocks = sampler.stop() if sampler else None
    t = torch.tensor([ms], dtype=torch.float64, device=dev)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    ms_max = float(t[0])
    if rank == 0:
        fl = flops_of(w)
        value = fl / (ms_max * 1e-3) / 1e12
        peaks, src = measured_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 Q, K, V)",
            "config": config_dict(w, world, args.split) | {
                "shards": [{"rank": s.rank, "heads": list(s.heads), "kv_heads": list(s.kv_heads),
                            "seqs": list(s.seqs)} for s in shards]},
            "gpu_launches": args.steps,
            "rank0": {"ms_per_step": ms, "flop_per_step": my_flops},
            "roofline": {"bound": "tensor", "achieved": value / world, "peak": peak, "unit": UNIT,
                         "frac": value / world / peak,
                         "note": "per GPU: the whole workload's FLOPs / slowest rank / ranks"},
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="3", choices=["1", "2", "3", "4", "5", "decode", "ring"])
    ap.add_argument("--splits", type=int, default=0,
                    help="decode only: cache slices (0 = attn_decode_default_splits)")
    ap.add_argument("--decode-batch", type=int, default=64,
                    help="decode only: sequences (64 is the benchmark; smaller for profiling)")
    ap.add_argument("--pass", dest="pass_", default="fwd", choices=["fwd", "bwd"],
                    help="fwd: attn_fwd (the benchmark); bwd: attn_bwd on the same workload")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "fp8"],
                    help="fp8: the forward on e4m3 inputs (attn_fwd_fp8); d = 128 workloads")
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference", "torch_sdpa"],
                    help="torch_sdpa: context only, PyTorch's scaled_dot_product_attention on the "
                         "same dense workload (not this library; one GPU)")
    ap.add_argument("--sdpa-backend", default="all", choices=["all", "cudnn", "flash", "efficient"],
                    help="--impl torch_sdpa only: the backends to time")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the other d = 128 workloads and the sustained loop (default "
                         "workload only)")
    ap.add_argument("--split", default="none", choices=["none", "heads", "sequences", "auto"],
                    help="with --gpus N: split ONE workload over the ranks (strong scaling) "
                         "instead of one batch shard per rank (weak scaling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.workload == "decode":
        main_decode(args, rank, world, local_rank)
        return
    if args.workload == "ring":
        main_ring(args, rank, world, local_rank)
        return
    w = W.workload(int(args.workload))
    if args.pass_ == "bwd":
        main_bwd(args, w, rank, world, local_rank)
        return
    if args.dtype == "fp8":
        main_fp8(args, w, rank, world, local_rank)
        return

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args, w)), flush=True)
        return
    if args.impl == "torch_sdpa":
        if rank == 0:
            print(json.dumps(run_torch_sdpa(args, w)), flush=True)
        return

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    if args.split != "none":
        try:
            main_split(args, w, rank, world, local_rank)
        finally:
            if world > 1:
                dist.destroy_process_group()
        return
    extra = sustained_run = None
    try:
        kernel_ms, e2e_ms, h2d, d2h, clocks = run_cuda(args, w, rank, world, local_rank)
        if rank == 0 and args.workload == "3" and not args.no_extra:
            dev = torch.device("cuda", local_rank)
            peaks, _ = measured_peaks()
            extra = other_workloads(dev, args.steps, args.warmup,
                                    float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS)))
            sustained_run = sustained_forward(w, dev, 2.5,
                                          float(peaks.get("bf16_tflops_sustained", 0.0)) or None)
    finally:
        if world > 1:
            dist.barrier()
    if rank == 0:
        fl = flops_of(w)
        value = fl * world / (kernel_ms * 1e-3) / 1e12
        achieved = fl / (kernel_ms * 1e-3) / 1e12
        peaks, src = measured_peaks()
        peak = float(peaks.get("bf16_tflops", FALLBACK_BF16_TFLOPS))
        sustained = float(peaks.get("bf16_tflops_sustained", 0.0)) or None
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": kernel_ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded normal bf16 Q, K, V)",
            "config": config_dict(w, world),
            "e2e": {"value": fl * world / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms, "streams": 2,
                    "how": "attn_fwd_host on pinned host buffers; two streams with their own "
                           "workspaces take alternate steps (copies overlap the other step's kernel)"},
            "gpu_launches": args.steps,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": UNIT,
                         "frac": achieved / peak, "traffic": recorded_traffic(w.name),
                         "peak_source": f"{src} bf16_tflops (burst, cuBLAS)" if src == "measured"
                         else "fallback 1590 TF/s",
                         "frac_of_sustained": (achieved / sustained) if sustained else None,
                         "frac_of_spec_2250": achieved / SPEC_BF16_TFLOPS,
                         "kernel": "attn_fwd_sm100<128,4>" if w.d == 128 else "attn_fwd_sm100<64,8>"},
            "clocks": clocks,
            "step_ms": step_stats(run_cuda.step_times),
        }
        if extra is not None:
            line["other_workloads"] = extra
        if sustained_run is not None:
            line["sustained"] = sustained_run
        if not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(w)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
