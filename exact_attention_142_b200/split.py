"""One attention forward split over several GPUs, with no collective.

"FlashAttention" explainer page (ozercemkelahmet.com/tools/flashattention), How
it works, Step 7: the work is spread over (query block, batch, head), and the
forward pass has no exchange step -- every (sequence, head) is independent of
every other.  Across GPUs the same independence gives two splits of one
workload, each rank running the single-GPU kernel on its own shard:

* heads: rank r takes a contiguous range of key/value heads together with the
  query heads that read them (whole GQA groups, so no key/value head is held
  by two ranks), over every sequence;
* sequences: rank r takes a contiguous range of the batch's sequences (dense
  batch entries or packed sequences), all heads; the ranges are chosen so that
  the largest rank's attention work (visible query/key pairs) is as small as a
  contiguous split allows -- causal and packed batches are far from uniform.

A shard's tensors are contiguous copies of its slice (in tensor parallelism a
rank already holds just its heads); its outputs are the same slice of the full
o and lse, so `unshard` only places them.  Nothing crosses between GPUs on the
data path.  `step` can be replaced (the CPU tests pass the oracle); by default
it is the CUDA entry point through the package's `attention`, with no fallback.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence, Tuple


@dataclass(frozen=True)
class Shard:
    rank: int
    heads: Tuple[int, int]     # query heads [h0, h1)
    kv_heads: Tuple[int, int]  # key/value heads [g0, g1)
    seqs: Tuple[int, int]      # sequences [b0, b1)

    @property
    def empty(self) -> bool:
        return self.heads[0] >= self.heads[1] or self.seqs[0] >= self.seqs[1]


def visible_pairs(L: int, causal: bool, left: int = -1, right: int = -1) -> int:
    """Visible (query, key) pairs of one sequence of L tokens: for row i the
    keys [max(0, i - left), min(L - 1, i + right)] (inclusive; -1 = unlimited,
    causal forces right = 0)."""
    if causal:
        right = 0
    total = 0
    for i in range(L):
        lo = 0 if left < 0 else max(0, i - left)
        hi = L - 1 if right < 0 else min(L - 1, i + right)
        total += hi - lo + 1
    return total


def split_heads(world: int, B: int, Hq: int, Hkv: int) -> List[Shard]:
    """Key/value heads dealt out in contiguous runs, as evenly as possible;
    ranks beyond Hkv get nothing."""
    if world <= 0 or Hkv <= 0 or Hq % Hkv:
        raise ValueError("need world >= 1 and Hq a multiple of Hkv")
    group = Hq // Hkv
    base, extra = divmod(Hkv, world)
    shards, g = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        shards.append(Shard(r, (g * group, (g + n) * group), (g, g + n), (0, B)))
        g += n
    return shards


def split_sequences(world: int, lengths: Sequence[int], Hq: int, Hkv: int, causal: bool,
                    left: int = -1, right: int = -1) -> List[Shard]:
    """Contiguous runs of sequences minimising the largest run's visible
    pairs (binary search on that maximum with a greedy fill); ranks left over
    get nothing."""
    if world <= 0:
        raise ValueError("need world >= 1")
    cost = [visible_pairs(L, causal, left, right) for L in lengths]

    def fill(limit):
        cuts, acc = [0], 0
        for b, c in enumerate(cost):
            if acc + c > limit and acc > 0:
                cuts.append(b)
                acc = 0
            acc += c
        return cuts

    lo, hi = max(cost, default=0), sum(cost)
    while lo < hi:
        mid = (lo + hi) // 2
        if len(fill(mid)) <= world:
            hi = mid
        else:
            lo = mid + 1
    cuts = fill(lo) if cost else [0]
    cuts = cuts + [len(lengths)] * (world + 1 - len(cuts))
    return [Shard(r, (0, Hq), (0, Hkv), (cuts[r], cuts[r + 1])) for r in range(world)]


def plan(world: int, mode: str, *, B: int, Hq: int, Hkv: int, lengths: Sequence[int],
         causal: bool, left: int = -1, right: int = -1) -> List[Shard]:
    """mode 'heads', 'sequences' or 'auto' (heads when the key/value heads
    divide evenly over the ranks, else sequences)."""
    if mode == "auto":
        mode = "heads" if Hkv % world == 0 else "sequences"
    if mode == "heads":
        return split_heads(world, B, Hq, Hkv)
    if mode == "sequences":
        return split_sequences(world, lengths, Hq, Hkv, causal, left, right)
    raise ValueError(f"unknown split mode {mode!r}")


def shard_inputs(q, k, v, shard: Shard, cu_seqlens: Optional[Sequence[int]] = None):
    """Contiguous copies of a shard's slice.  Dense q [B, N, Hq, d] (k, v with
    Hkv); packed q [T, Hq, d] with host cu_seqlens.  Returns (q, k, v, local
    cu_seqlens or None, local B, local Hq, local Hkv)."""
    (h0, h1), (g0, g1), (b0, b1) = shard.heads, shard.kv_heads, shard.seqs
    if cu_seqlens is None:
        return (q[b0:b1, :, h0:h1].contiguous(), k[b0:b1, :, g0:g1].contiguous(),
                v[b0:b1, :, g0:g1].contiguous(), None, b1 - b0, h1 - h0, g1 - g0)
    t0, t1 = cu_seqlens[b0], cu_seqlens[b1]
    cu = [c - t0 for c in cu_seqlens[b0:b1 + 1]]
    return (q[t0:t1, h0:h1].contiguous(), k[t0:t1, g0:g1].contiguous(),
            v[t0:t1, g0:g1].contiguous(), cu, b1 - b0, h1 - h0, g1 - g0)


def run_shard(q, k, v, shard: Shard, *, causal: bool, scale: float, left: int = -1,
              right: int = -1, cu_seqlens: Optional[Sequence[int]] = None,
              step: Optional[Callable] = None):
    """This rank's part of the forward: (o, lse) of its slice, laid out like
    attn_fwd's outputs for the local sizes (None for an empty shard).
    step(q, k, v, cu_seqlens, B, Hq, Hkv) -> (o, lse); by default the CUDA path
    on q's device."""
    if shard.empty:
        return None
    qs, ks, vs, cu, B, Hq, Hkv = shard_inputs(q, k, v, shard, cu_seqlens)
    if step is None:
        step = _cuda_step(causal, scale, left, right)
    return step(qs, ks, vs, cu, B, Hq, Hkv)


def _cuda_step(causal, scale, left, right):
    def step(q, k, v, cu, B, Hq, Hkv):
        import torch

        from . import attention
        cud = None if cu is None else torch.tensor(cu, dtype=torch.int32, device=q.device)
        max_seqlen = 0 if cu is None else max(b - a for a, b in zip(cu[:-1], cu[1:]))
        return attention(q, k, v, causal=causal, window_left=left, window_right=right,
                         scale=scale, cu_seqlens=cud, max_seqlen=max_seqlen)
    return step


def unshard(parts, shards: List[Shard], *, B: int, Hq: int, d: int,
            cu_seqlens: Optional[Sequence[int]] = None, N: int = 0):
    """Place every rank's (o, lse) into full-size arrays (numpy or torch
    tensors on the CPU).  Dense: o [B, N, Hq, d], lse [B, Hq, N]; packed:
    o [T, Hq, d], lse [Hq, T]."""
    import numpy as np
    T = cu_seqlens[-1] if cu_seqlens is not None else 0
    if cu_seqlens is None:
        o = np.full((B, N, Hq, d), np.nan)
        lse = np.full((B, Hq, N), np.nan)
    else:
        o = np.full((T, Hq, d), np.nan)
        lse = np.full((Hq, T), np.nan)
    for part, sh in zip(parts, shards):
        if part is None or sh.empty:
            continue
        po, pl = (np.asarray(x.cpu().double() if hasattr(x, "cpu") else x, dtype=np.float64)
                  for x in part)
        (h0, h1), (b0, b1) = sh.heads, sh.seqs
        if cu_seqlens is None:
            o[b0:b1, :, h0:h1] = po.reshape(b1 - b0, N, h1 - h0, d)
            lse[b0:b1, h0:h1] = pl.reshape(b1 - b0, h1 - h0, N)
        else:
            t0, t1 = cu_seqlens[b0], cu_seqlens[b1]
            o[t0:t1, h0:h1] = po.reshape(t1 - t0, h1 - h0, d)
            lse[h0:h1, t0:t1] = pl.reshape(h1 - h0, t1 - t0)
    return o, lse
