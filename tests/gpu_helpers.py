"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same host bytes, and compare."""
from __future__ import annotations

import math

import numpy as np
import torch

import exact_attention_142_b200 as ea
import oracle
import workloads as W

# Tolerances against the fp64 oracle (bf16 O, fp32 LSE).
TOL_O = 1e-2
TOL_LSE = 1e-3


def gpu_run(q, k, v, *, B, Hq, Hkv, N, d, scale, causal, window_left=-1, window_right=-1,
            cu_seqlens=None, max_seqlen=0):
    """q/k/v CPU bf16 tensors -> (o CPU bf16 tensor, lse CPU fp32 tensor)."""
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    if cu_seqlens is not None:
        cu = torch.tensor(cu_seqlens, dtype=torch.int32, device=dev)
        lse = torch.full((Hq, N), float("nan"), dtype=torch.float32, device=dev)
        if max_seqlen == 0:
            max_seqlen = max(b - a for a, b in zip(cu_seqlens[:-1], cu_seqlens[1:]))
    else:
        cu = None
        lse = torch.full((B, Hq, N), float("nan"), dtype=torch.float32, device=dev)
    o = torch.full_like(qd, float("nan"))
    ea.attn_fwd(qd, kd, vd, o, lse, B, Hq, Hkv, N, d, scale, causal, window_left, window_right,
                cu, max_seqlen)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return o.cpu(), lse.cpu()


def oracle_run(q, k, v, rows=None, **kw):
    kw = dict(kw)
    kw.pop("max_seqlen", None)
    return oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), rows=rows, **kw)


def compare_full(o_gpu, lse_gpu, o_ref, lse_ref, tol_o=TOL_O, tol_lse=TOL_LSE):
    og = o_gpu.to(torch.float64).numpy().reshape(o_ref.shape)
    lg = lse_gpu.to(torch.float64).numpy().reshape(lse_ref.shape)
    assert np.isfinite(og).all(), "non-finite O"
    dO = float(np.abs(og - o_ref).max()) if og.size else 0.0
    dL = float(np.abs(lg - lse_ref).max()) if lg.size else 0.0
    assert dO <= tol_o, f"max|dO| = {dO}"
    assert dL <= tol_lse, f"max|dLSE| = {dL}"
    return dO, dL


def lse_index(w_cu, b, h, i, Hq, N):
    """Flat index of (sequence b, head h, row i) in the LSE output."""
    if w_cu is not None:
        return h * N + w_cu[b] + i
    return (b * Hq + h) * N + i


def o_index(w_cu, b, i, N):
    return (w_cu[b] + i) if w_cu is not None else b * N + i


def sample_rows(lengths, Hq, n_random, seed):
    """(sequence, head, row) triples: tile boundaries, both ends, random rows."""
    rng = np.random.default_rng(seed)
    rows = set()
    B = len(lengths)
    special_b = sorted({0, B - 1, int(rng.integers(B))})
    for b in special_b:
        L = lengths[b]
        if L == 0:
            continue
        for i in (0, 1, 2, 126, 127, 128, 129, 255, 256, L // 2, L - 129, L - 128, L - 2, L - 1):
            if 0 <= i < L:
                rows.add((b, int(rng.integers(Hq)), i))
                rows.add((b, 0, i))
                rows.add((b, Hq - 1, i))
    nonempty = [b for b in range(B) if lengths[b] > 0]
    for _ in range(n_random):
        b = nonempty[int(rng.integers(len(nonempty)))]
        rows.add((b, int(rng.integers(Hq)), int(rng.integers(lengths[b]))))
    return np.array(sorted(rows), dtype=np.int64)


def visible_counts(lengths, causal, left, right):
    """Closed-form count of visible keys for every row of every sequence
    (the count the oracle returns, per the window definition)."""
    if causal:
        right = 0
    out = []
    for L in lengths:
        i = np.arange(L, dtype=np.int64)
        lo = np.zeros(L, np.int64) if left < 0 else np.maximum(0, i - left)
        hi = np.full(L, L - 1, np.int64) if right < 0 else np.minimum(L - 1, i + right)
        out.append(hi - lo + 1)
    return out


def default_scale(d):
    return float(np.float32(1.0 / math.sqrt(d)))
