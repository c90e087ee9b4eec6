"""The ring (context-parallel) forward's host logic on CPU: the zigzag schedule,
and world_size 2 and 3 gloo runs of ring_attention_forward whose per-step
attention is the fp64 oracle (passed in as the step function), checked against
the oracle on the whole sequence."""
from __future__ import annotations

import os
import socket
import tempfile

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

from exact_attention_142_b200 import ring


@pytest.mark.parametrize("world", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("causal", [True, False])
def test_schedule_covers_every_pair_once(world, causal):
    work = []
    for r in range(world):
        mine = ring.zigzag_chunks(world, r)
        seen = {}
        n = 0
        for t, src, pairs in ring.ring_schedule(world, r, causal):
            assert src == (r - t) % world
            theirs = ring.zigzag_chunks(world, src)
            for a, c, rel in pairs:
                key = (mine[a], theirs[c])
                assert key not in seen
                seen[key] = rel
                n += 1
        for qc in mine:
            for kc in range(2 * world):
                want = ring.chunk_pair(qc, kc, causal)
                assert seen.get((qc, kc), "skip") == want
        work.append(n)
    if causal:
        assert len(set(work)) == 1  # zigzag: every rank does the same number of chunk pairs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_step(B, Hq, Hkv, d, scale):
    import oracle
    import workloads as W

    def step(q, k, v, o_acc, lse_acc, causal):
        C = q.shape[1]
        o, lse, _ = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), B=B, Hq=Hq,
                                    Hkv=Hkv, N=C, d=d, scale=scale, causal=causal)
        o = o.reshape(B, C, Hq, d)
        old_l = lse_acc.to(torch.float64).numpy()
        L = np.logaddexp(old_l, lse)
        w_old = np.where(np.isneginf(old_l), 0.0, np.exp(old_l - L))
        w_new = np.where(np.isneginf(lse), 0.0, np.exp(lse - L))
        # weights [B, Hq, C] -> [B, C, Hq, 1]
        wo = np.transpose(w_old, (0, 2, 1))[..., None]
        wn = np.transpose(w_new, (0, 2, 1))[..., None]
        # a row whose accumulator LSE is -inf is empty: its O is not read
        empty = np.transpose(np.isneginf(old_l), (0, 2, 1))[..., None]
        acc = np.where(empty, 0.0, o_acc.to(torch.float64).numpy())
        o_acc.copy_(torch.from_numpy(wo * acc + wn * o))
        lse_acc.copy_(torch.from_numpy(L))
    return step


def _worker(rank, world, port, causal, out_dir):
    import torch.distributed as dist

    import oracle
    import workloads as W
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        B, Hq, Hkv, d, C = 2, 4, 2, 16, 24
        N = 2 * world * C
        scale = 0.3
        q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed=60 + world)
        qs, ks, vs = (ring.shard_zigzag(t, world, rank) for t in (q, k, v))
        outs, lses = ring.ring_attention_forward(
            qs, ks, vs, scale=scale, causal=causal, accumulate=_oracle_step(B, Hq, Hkv, d, scale),
            finalize=lambda acc: acc.clone())
        mine = torch.stack([torch.cat([outs[0], outs[1]], dim=1),
                            torch.cat([lses[0], lses[1]], dim=2).transpose(1, 2).unsqueeze(-1)
                            .expand(-1, -1, -1, d)], dim=0)
        got = [torch.empty_like(mine) for _ in range(world)]
        dist.all_gather(got, mine)
        if rank == 0:
            parts = [(g[0][:, :C], g[0][:, C:]) for g in got]
            lparts = [(g[1][:, :C, :, 0], g[1][:, C:, :, 0]) for g in got]
            o_full = ring.unshard_zigzag(parts, world).to(torch.float64).numpy()
            l_full = ring.unshard_zigzag(lparts, world).to(torch.float64).numpy()  # [B, N, Hq]
            o_ref, lse_ref, _ = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v),
                                                B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                                                causal=causal)
            o_ref = o_ref.reshape(B, N, Hq, d)
            dO = float(np.abs(o_full - o_ref).max())
            dL = float(np.abs(l_full - np.transpose(lse_ref, (0, 2, 1))).max())
            with open(os.path.join(out_dir, "result.txt"), "w") as f:
                f.write(f"{dO} {dL}\n")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,causal", [(2, True), (3, True), (2, False)])
def test_ring_gloo_matches_whole_sequence(world, causal):
    with tempfile.TemporaryDirectory() as out:
        mp.spawn(_worker, args=(world, _free_port(), causal, out), nprocs=world, join=True)
        dO, dL = map(float, open(os.path.join(out, "result.txt")).read().split())
    # fp32 accumulators of fp64 partial results: rounding only
    assert dO <= 1e-5 and dL <= 1e-5, (dO, dL)
