"""Seeded synthetic inputs, shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic: only shapes, seeds and random draws.
Both sides receive the very same host bytes from it.

Recipe (one fixed rule for every workload):
  torch.manual_seed(seed); q, k, v = torch.randn(shape, float32) drawn in that
  order on the CPU, each then rounded to bfloat16.
  Dense shapes are [B, N, H, d] ("Flash Attention" skill page (skillmd.com),
  Workflow 2: input [batch_size, seq_len, num_heads, head_dim]); packed
  variable-length shapes are [tokens, H, d] with int32 cumulative boundaries.
  The pages time normal-random bf16/fp16 tensors of this kind ("FlashAttention"
  explainer page, "A simple benchmark script"); no dataset is involved.

The five named workloads are the ones the benchmark and the parity tests use.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional

import numpy as np
import torch


@dataclass
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    N: int  # dense: sequence length; packed: total tokens
    d: int
    causal: bool
    window_left: int
    window_right: int
    seed: int
    cu_seqlens: Optional[List[int]] = None
    max_seqlen: int = 0
    scale: float = field(default=0.0)

    def __post_init__(self):
        if self.scale == 0.0:
            self.scale = default_scale(self.d)
        if self.max_seqlen == 0:
            if self.cu_seqlens is None:
                self.max_seqlen = self.N
            else:
                self.max_seqlen = max(b - a for a, b in zip(self.cu_seqlens[:-1], self.cu_seqlens[1:]))

    @property
    def tokens(self) -> int:
        return self.cu_seqlens[-1] if self.cu_seqlens is not None else self.B * self.N

    @property
    def packed(self) -> bool:
        return self.cu_seqlens is not None


def default_scale(d: int) -> float:
    """1/sqrt(d) as the fp32 value that is passed to both sides."""
    return float(np.float32(1.0 / math.sqrt(d)))


def packed_lengths(seed: int = 4, total: int = 65536, lo: int = 128, hi: int = 4096) -> List[int]:
    """Sequence lengths drawn uniform in [lo, hi] until `total` tokens; the last
    one is truncated so the lengths sum to exactly `total`."""
    rng = np.random.default_rng(seed)
    out: List[int] = []
    acc = 0
    while acc < total:
        L = int(rng.integers(lo, hi + 1))
        L = min(L, total - acc)
        out.append(L)
        acc += L
    return out


def cumulative(lengths: List[int]) -> List[int]:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return cu


def workload(cfg: int) -> Workload:
    """The five named workloads (1 is small enough for a full oracle run)."""
    if cfg == 1:
        return Workload("noncausal_b1_h2_n256_d64", 1, 2, 2, 256, 64, False, -1, -1, 0)
    if cfg == 2:
        return Workload("causal_mha_b4_h16_n2048_d128", 4, 16, 16, 2048, 128, True, -1, -1, 1)
    if cfg == 3:
        return Workload("causal_gqa_b2_hq32_hkv8_n8192_d128", 2, 32, 8, 8192, 128, True, -1, -1, 2)
    if cfg == 4:
        return Workload("swa_b1_h32_n16384_d128_left4096", 1, 32, 32, 16384, 128, True, 4096, 0, 3)
    if cfg == 5:
        cu = cumulative(packed_lengths(4))
        return Workload("varlen_causal_t65536_hq32_hkv8_d128", len(cu) - 1, 32, 8, cu[-1], 128,
                        True, -1, -1, 4, cu_seqlens=cu)
    raise ValueError(f"unknown workload {cfg}")


def draw_qkv(shape_q, shape_kv, seed: int):
    """q, k, v as CPU bf16 tensors (fp32 normal draws rounded to bf16)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(shape_q, dtype=torch.float32, generator=g).to(torch.bfloat16)
    k = torch.randn(shape_kv, dtype=torch.float32, generator=g).to(torch.bfloat16)
    v = torch.randn(shape_kv, dtype=torch.float32, generator=g).to(torch.bfloat16)
    return q, k, v


def inputs(w: Workload):
    """(q, k, v) CPU bf16 tensors for a workload; packed workloads are [T, H, d]."""
    if w.packed:
        return draw_qkv((w.tokens, w.Hq, w.d), (w.tokens, w.Hkv, w.d), w.seed)
    return draw_qkv((w.B, w.N, w.Hq, w.d), (w.B, w.N, w.Hkv, w.d), w.seed)


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """View a CPU bf16 tensor as its uint16 bit patterns (no copy of values)."""
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def from_bits(a: np.ndarray) -> torch.Tensor:
    """Inverse of bf16_bits."""
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


# --------------------------------------------------------------------------
# key/value-cache decode
# --------------------------------------------------------------------------
@dataclass
class DecodeWorkload:
    """Nq newest tokens per sequence against a paged key/value cache.

    Caches are [B * pages_per_seq, page_size, Hkv, d]; the page table, when
    `paged`, is a seeded random permutation of all pages (so logical neighbours
    sit far apart in memory, as in a serving pool); otherwise sequence b owns
    pages b * pages_per_seq ... contiguously.
    """
    name: str
    B: int
    Hq: int
    Hkv: int
    Nq: int
    d: int
    page_size: int
    pages_per_seq: int
    lengths: List[int]
    paged: bool
    causal: bool
    window_left: int
    window_right: int
    seed: int
    scale: float = field(default=0.0)

    def __post_init__(self):
        if self.scale == 0.0:
            self.scale = default_scale(self.d)

    @property
    def max_len(self) -> int:
        return self.page_size * self.pages_per_seq


def decode_workload(B: int = 64) -> DecodeWorkload:
    """The decode benchmark: B (64) sequences, each with a full 8192-token
    cache, one new token, the grouped-query head layout of the 8192-token
    causal workload (32 query heads over 8 key/value heads, d = 128), 64-token
    pages.  Smaller B gives the same shape at a smaller size (B = 8: 268 MB of
    cache, still twice the L2)."""
    return DecodeWorkload(f"decode_gqa_b{B}_hq32_hkv8_l8192_d128_page64", B, 32, 8, 1, 128, 64,
                          128, [8192] * B, True, True, -1, -1, 5)


def decode_inputs(w: DecodeWorkload, device: str = "cpu"):
    """(q [B,Nq,Hq,d], k_cache, v_cache, cache_seqlens int32 [B],
    block_table int32 [B, pages_per_seq] or None).  The draws follow the same
    rule as draw_qkv (fp32 normal, rounded to bf16; q, k, v in that order),
    then the page permutation; `device="cuda"` draws with a CUDA generator
    (faster for multi-GB caches; different bytes than the CPU draw)."""
    g = torch.Generator(device=device)
    g.manual_seed(w.seed)
    pages = w.B * w.pages_per_seq
    q = torch.randn((w.B, w.Nq, w.Hq, w.d), dtype=torch.float32, generator=g,
                    device=device).to(torch.bfloat16)
    kc = torch.empty((pages, w.page_size, w.Hkv, w.d), dtype=torch.bfloat16, device=device)
    vc = torch.empty_like(kc)
    for c in (kc, vc):  # page by page to bound the fp32 temporary
        step = max(1, (1 << 26) // (w.page_size * w.Hkv * w.d))
        for p0 in range(0, pages, step):
            p1 = min(pages, p0 + step)
            c[p0:p1] = torch.randn((p1 - p0, w.page_size, w.Hkv, w.d), dtype=torch.float32,
                                   generator=g, device=device).to(torch.bfloat16)
    seqlens = torch.tensor(w.lengths, dtype=torch.int32)
    table = None
    if w.paged:
        perm = torch.randperm(pages, generator=torch.Generator().manual_seed(w.seed))
        table = perm.to(torch.int32).reshape(w.B, w.pages_per_seq)
    return q, kc, vc, seqlens, table


# --------------------------------------------------------------------------
# 8-bit (e4m3) inputs
# --------------------------------------------------------------------------
def draw_qkv_e4m3(shape_q, shape_kv, seed: int):
    """q, k, v as CPU float8_e4m3fn tensors: the same normal draws as draw_qkv,
    converted to e4m3 (round to nearest even, as torch's .to(float8_e4m3fn))."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn(shape_q, dtype=torch.float32, generator=g).to(torch.float8_e4m3fn)
    k = torch.randn(shape_kv, dtype=torch.float32, generator=g).to(torch.float8_e4m3fn)
    v = torch.randn(shape_kv, dtype=torch.float32, generator=g).to(torch.float8_e4m3fn)
    return q, k, v


def e4m3_as_bf16(t: torch.Tensor) -> torch.Tensor:
    """Every finite e4m3 value is exact in bf16 (3 mantissa bits into 7, exponents
    2^-9 .. 2^8 inside bf16's range): the oracle's bf16 input for e4m3 data."""
    return t.to(torch.bfloat16)
