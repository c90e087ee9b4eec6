"""Context-parallel (ring) attention forward across ranks.

"FlashAttention" explainer page (ozercemkelahmet.com/tools/flashattention),
"Long context beyond a single GPU": the sequence is split across devices, blocks
of keys and values travel around the group, every device computes partial
attention with the fused kernel and merges the partial results with the
online-softmax rule.  Here:

* Sharding ("zigzag"): a sequence of N = 2 P C tokens is cut into 2P chunks of
  C tokens; rank r holds chunks r and 2P - 1 - r of Q, K and V.  Under a causal
  mask every rank then has the same amount of work.
* Step t = 0 .. P-1: rank r holds the K/V chunks of rank (r - t) mod P.  For
  each of its two query chunks a and each visiting key chunk c: c < a is full
  (unmasked) attention, c == a is the causal diagonal, c > a is skipped.
  Without a causal mask every pair is full.
* Each computed pair is merged into an fp32 accumulator by the CUDA kernel's
  accumulating epilogue (attn_fwd_accumulate), so no separate merge pass runs;
  the accumulator is rounded to bf16 once at the end (attn_acc_to_bf16).
* K/V move with torch.distributed point-to-point sends to rank r + 1 and
  receives from rank r - 1 (NCCL on GPUs), posted before the step's compute
  so that the transfer overlaps it; the next step waits for them.

Dense batches [B, C, H, d] per chunk; sliding windows and packed sequences are
not part of the ring (a window would make the per-chunk masks position
dependent).  `accumulate` can be replaced (the CPU tests pass an oracle-based
one); by default it is the CUDA entry point, and there is no fallback.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence, Tuple


def zigzag_chunks(world: int, rank: int) -> Tuple[int, int]:
    """The two chunk indices (of 2 * world) that a rank holds."""
    return rank, 2 * world - 1 - rank


def chunk_pair(q_chunk: int, k_chunk: int, causal: bool) -> str:
    """'full', 'diag' (causal within the chunk) or 'skip' for a chunk pair."""
    if not causal or k_chunk < q_chunk:
        return "full"
    return "diag" if k_chunk == q_chunk else "skip"


def ring_schedule(world: int, rank: int, causal: bool = True):
    """[(step, source rank, [(query slot, key slot, 'full' | 'diag'), ...]), ...]"""
    mine = zigzag_chunks(world, rank)
    out = []
    for t in range(world):
        src = (rank - t) % world
        theirs = zigzag_chunks(world, src)
        pairs = []
        for a in range(2):
            for c in range(2):
                rel = chunk_pair(mine[a], theirs[c], causal)
                if rel != "skip":
                    pairs.append((a, c, rel))
        out.append((t, src, pairs))
    return out


def cuda_accumulate(scale: float, stream=None) -> Callable:
    """The default step: attn_fwd_accumulate on device buffers."""
    from . import _binding as b

    def step(q, k, v, o_acc, lse_acc, causal: bool):
        B, C, Hq, d = q.shape
        Hkv = k.shape[2]
        b.attn_fwd_accumulate(q, k, v, o_acc, lse_acc, B, Hq, Hkv, C, d, scale, causal, -1, -1,
                              None, 0, stream)
    return step


def ring_attention_forward(q_chunks: Sequence, k_chunks: Sequence, v_chunks: Sequence, *,
                           scale: float, causal: bool = True, group=None,
                           accumulate: Optional[Callable] = None, finalize: Optional[Callable] = None,
                           stream=None):
    """This rank's part of ring attention.

    q_chunks, k_chunks, v_chunks: this rank's two zigzag chunks, each a
    contiguous [B, C, H, d] bf16 tensor (q with Hq heads, k and v with Hkv).
    Returns ((o_a, o_b), (lse_a, lse_b)): O as bf16 [B, C, Hq, d] and the fp32
    LSE [B, Hq, C] of each query chunk over the whole sequence.
    """
    import torch
    import torch.distributed as dist

    distributed = dist.is_available() and dist.is_initialized()
    world = dist.get_world_size(group) if distributed else 1
    rank = dist.get_rank(group) if distributed else 0
    if accumulate is None:
        accumulate = cuda_accumulate(scale, stream)
    q_chunks = list(q_chunks)
    B, C, Hq, d = q_chunks[0].shape
    # rows whose LSE is -inf are empty: their O is neither read nor needs zeroing
    o_acc = [torch.empty((B, C, Hq, d), dtype=torch.float32, device=q.device) for q in q_chunks]
    lse_acc = [torch.full((B, Hq, C), float("-inf"), dtype=torch.float32, device=q.device)
               for q in q_chunks]
    cur_k, cur_v = list(k_chunks), list(v_chunks)
    nxt = ([torch.empty_like(t) for t in cur_k], [torch.empty_like(t) for t in cur_v])
    for t, src, pairs in ring_schedule(world, rank, causal):
        reqs = []
        if t < world - 1:
            to, frm = (rank + 1) % world, (rank - 1) % world
            if group is not None:
                to, frm = dist.get_global_rank(group, to), dist.get_global_rank(group, frm)
            ops = []
            for i in range(2):
                ops.append(dist.P2POp(dist.isend, cur_k[i], to, group))
                ops.append(dist.P2POp(dist.isend, cur_v[i], to, group))
                ops.append(dist.P2POp(dist.irecv, nxt[0][i], frm, group))
                ops.append(dist.P2POp(dist.irecv, nxt[1][i], frm, group))
            reqs = dist.batch_isend_irecv(ops)
        for a, c, rel in pairs:
            accumulate(q_chunks[a], cur_k[c], cur_v[c], o_acc[a], lse_acc[a], rel == "diag")
        for r in reqs:
            r.wait()
        if t < world - 1:
            # the buffers just sent become the next receive buffers
            old = (cur_k, cur_v)
            cur_k, cur_v = nxt
            nxt = old
    if finalize is None:
        from . import _binding as b

        def finalize(acc):
            out = torch.empty(acc.shape, dtype=torch.bfloat16, device=acc.device)
            b.attn_acc_to_bf16(acc, out, acc.numel(), stream)
            return out
    return tuple(finalize(o) for o in o_acc), tuple(lse_acc)


def shard_zigzag(x, world: int, rank: int, dim: int = 1):
    """This rank's two chunks of a full [B, N, H, d] tensor (contiguous copies)."""
    n = x.shape[dim]
    assert n % (2 * world) == 0, "sequence length must be a multiple of 2 * world"
    c = n // (2 * world)
    return tuple(x.narrow(dim, i * c, c).contiguous() for i in zigzag_chunks(world, rank))


def unshard_zigzag(chunks_by_rank, world: int, dim: int = 1):
    """Inverse of shard_zigzag: chunks_by_rank[r] = (chunk r, chunk 2P-1-r)."""
    import torch
    order = [None] * (2 * world)
    for r, (a, b) in enumerate(chunks_by_rank):
        i, j = zigzag_chunks(world, r)
        order[i], order[j] = a, b
    return torch.cat(order, dim=dim)
