"""One forward split over several ranks (heads or sequences, no collective on
the data path): the split plans on CPU, and world_size 2 and 3 gloo runs whose
per-rank attention is the fp64 oracle (passed in as the step function),
gathered on rank 0 and checked against the oracle on the whole workload."""
from __future__ import annotations

import os
import pickle
import socket
import tempfile

import numpy as np
import pytest
import torch.multiprocessing as mp

from exact_attention_142_b200 import split


def brute_pairs(L, causal, left, right):
    if causal:
        right = 0
    n = 0
    for i in range(L):
        for j in range(L):
            if (left < 0 or j >= i - left) and (right < 0 or j <= i + right):
                n += 1
    return n


@pytest.mark.parametrize("L,causal,left,right", [(0, True, -1, -1), (1, True, -1, -1),
                                                 (37, True, -1, -1), (37, False, -1, -1),
                                                 (50, True, 7, -1), (50, False, 3, 9),
                                                 (20, False, -1, 0), (20, False, 0, 0)])
def test_visible_pairs_closed_count(L, causal, left, right):
    assert split.visible_pairs(L, causal, left, right) == brute_pairs(L, causal, left, right)


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8, 16])
@pytest.mark.parametrize("Hq,Hkv", [(32, 8), (16, 16), (8, 1), (6, 2)])
def test_head_split_is_group_aligned_and_covers_every_head_once(world, Hq, Hkv):
    shards = split.split_heads(world, 3, Hq, Hkv)
    assert len(shards) == world
    group = Hq // Hkv
    seen_q, seen_kv = [], []
    for s in shards:
        (h0, h1), (g0, g1) = s.heads, s.kv_heads
        assert h0 == g0 * group and h1 == g1 * group  # whole groups only
        seen_q += list(range(h0, h1))
        seen_kv += list(range(g0, g1))
        assert s.seqs == (0, 3)
    assert seen_q == list(range(Hq)) and seen_kv == list(range(Hkv))
    sizes = [s.kv_heads[1] - s.kv_heads[0] for s in shards]
    assert max(sizes) - min(sizes) <= 1


def brute_best_max(costs, world):
    """Smallest possible largest run over all contiguous splits (brute force)."""
    import itertools
    n = len(costs)
    best = sum(costs)
    for k in range(min(world, n + 1)):
        for cuts in itertools.combinations(range(1, n), k):
            bounds = (0,) + cuts + (n,)
            best = min(best, max(sum(costs[a:b]) for a, b in zip(bounds, bounds[1:])))
    return best


@pytest.mark.parametrize("world", [1, 2, 3, 4, 7])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_sequence_split_is_contiguous_and_optimal(world, seed):
    rng = np.random.default_rng(seed)
    lengths = [int(x) for x in rng.integers(0, 60, size=int(rng.integers(1, 9)))]
    shards = split.split_sequences(world, lengths, 4, 2, causal=True)
    assert len(shards) == world
    assert shards[0].seqs[0] == 0 and shards[-1].seqs[1] == len(lengths)
    for a, b in zip(shards, shards[1:]):
        assert a.seqs[1] == b.seqs[0]
    costs = [brute_pairs(L, True, -1, -1) for L in lengths]
    worst = max(sum(costs[s.seqs[0]:s.seqs[1]]) for s in shards)
    assert worst == brute_best_max(costs, world)


def test_workload_splits_balance():
    """The 65 536-token packed workload over 2 and 4 ranks: the largest rank
    holds at most 1/world of the work plus one sequence."""
    import workloads as W
    w = W.workload(5)
    lengths = [b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])]
    costs = [split.visible_pairs(L, True) for L in lengths]
    for world in (2, 4, 8):
        shards = split.split_sequences(world, lengths, w.Hq, w.Hkv, True)
        worst = max(sum(costs[s.seqs[0]:s.seqs[1]]) for s in shards)
        assert worst <= sum(costs) / world + max(costs)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


CASES = {
    "heads_dense_causal": dict(mode="heads", lengths=[40, 40], packed=False, Hq=8, Hkv=4, d=16,
                               causal=True, left=-1, right=-1),
    "heads_packed_window": dict(mode="heads", lengths=[30, 0, 57, 5], packed=True, Hq=6, Hkv=3,
                                d=16, causal=True, left=9, right=-1),
    "sequences_packed_causal": dict(mode="sequences", lengths=[70, 3, 0, 41, 22, 9], packed=True,
                                    Hq=4, Hkv=2, d=16, causal=True, left=-1, right=-1),
    "sequences_dense_noncausal": dict(mode="sequences", lengths=[33, 33, 33], packed=False, Hq=2,
                                      Hkv=1, d=8, causal=False, left=4, right=6),
}


def _oracle_step(d, scale, causal, left, right):
    import oracle
    import workloads as W

    def step(q, k, v, cu, B, Hq, Hkv):
        N = q.shape[0] if cu is not None else q.shape[1]
        o, lse, _ = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), B=B, Hq=Hq,
                                    Hkv=Hkv, N=N, d=d, scale=scale, causal=causal,
                                    window_left=left, window_right=right, cu_seqlens=cu)
        return o, lse
    return step


def _worker(rank, world, port, name, out_dir):
    import torch.distributed as dist

    import oracle
    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = CASES[name]
        lengths, Hq, Hkv, d = c["lengths"], c["Hq"], c["Hkv"], c["d"]
        scale = 0.3
        B = len(lengths)
        if c["packed"]:
            cu = W.cumulative(lengths)
            N = cu[-1]
            q, k, v = W.draw_qkv((N, Hq, d), (N, Hkv, d), seed=90 + world)
        else:
            cu = None
            N = lengths[0]
            q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed=90 + world)
        shards = split.plan(world, c["mode"], B=B, Hq=Hq, Hkv=Hkv, lengths=lengths,
                            causal=c["causal"], left=c["left"], right=c["right"])
        mine = split.run_shard(q, k, v, shards[rank], causal=c["causal"], scale=scale,
                               left=c["left"], right=c["right"], cu_seqlens=cu,
                               step=_oracle_step(d, scale, c["causal"], c["left"], c["right"]))
        parts = [None] * world
        dist.all_gather_object(parts, mine)
        if rank == 0:
            o, lse = split.unshard(parts, shards, B=B, Hq=Hq, d=d, cu_seqlens=cu, N=N)
            o_ref, lse_ref, _ = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v),
                                                B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                                                causal=c["causal"], window_left=c["left"],
                                                window_right=c["right"], cu_seqlens=cu)
            nonempty = [s.rank for s in shards if not s.empty]
            with open(os.path.join(out_dir, "result.pkl"), "wb") as f:
                pickle.dump((o, lse, o_ref.reshape(o.shape), lse_ref.reshape(lse.shape),
                             nonempty), f)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,name", [(2, "heads_dense_causal"), (3, "heads_packed_window"),
                                        (2, "sequences_packed_causal"),
                                        (3, "sequences_packed_causal"),
                                        (2, "sequences_dense_noncausal")])
def test_split_gloo_matches_whole_workload(world, name):
    with tempfile.TemporaryDirectory() as out:
        mp.spawn(_worker, args=(world, _free_port(), name, out), nprocs=world, join=True)
        with open(os.path.join(out, "result.pkl"), "rb") as f:
            o, lse, o_ref, lse_ref, nonempty = pickle.load(f)
    assert len(nonempty) >= 2  # the work really was split
    # an empty sequence has no rows; everything else was written by some rank
    assert not np.isnan(o).any() and not np.isnan(lse).any()
    # the same fp64 arithmetic on each slice: equal to the whole-workload run
    assert np.abs(o - o_ref).max() <= 1e-12
    assert np.abs(lse - lse_ref).max() <= 1e-12
