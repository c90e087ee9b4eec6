"""GPU parity of the ring (context-parallel) forward's kernels: attn_fwd_accumulate
and attn_acc_to_bf16, through the C ABI.  The ranks of a ring are emulated one
after the other on this GPU (no rank waits on another), each step merging its
chunk pairs into the accumulators exactly as ring_attention_forward does; the
result must match the oracle on the whole sequence."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import oracle
import workloads as W
from exact_attention_142_b200 import ring
from gpu_helpers import TOL_LSE, TOL_O, default_scale

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def ref(q, k, v, *, B, Hq, Hkv, N, d, scale, causal):
    o, lse, _ = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), B=B, Hq=Hq,
                                Hkv=Hkv, N=N, d=d, scale=scale, causal=causal)
    return o.reshape(B, N, Hq, d), lse  # lse [B, Hq, N]


def emulate_ring(q, k, v, world, *, scale, causal):
    """Every rank's ring_attention_forward, one rank at a time on this GPU."""
    outs, lses = [], []
    for r in range(world):
        qs = [t.to(DEV) for t in ring.shard_zigzag(q, world, r)]
        B, C, Hq, d = qs[0].shape
        o_acc = [torch.zeros((B, C, Hq, d), dtype=torch.float32, device=DEV) for _ in range(2)]
        l_acc = [torch.full((B, Hq, C), float("-inf"), dtype=torch.float32, device=DEV)
                 for _ in range(2)]
        step = ring.cuda_accumulate(scale)
        for t, src, pairs in ring.ring_schedule(world, r, causal):
            ks = [x.to(DEV) for x in ring.shard_zigzag(k, world, src)]
            vs = [x.to(DEV) for x in ring.shard_zigzag(v, world, src)]
            for a, c, rel in pairs:
                step(qs[a], ks[c], vs[c], o_acc[a], l_acc[a], rel == "diag")
        o16 = []
        for acc in o_acc:
            out = torch.empty(acc.shape, dtype=torch.bfloat16, device=DEV)
            ea.attn_acc_to_bf16(acc, out, acc.numel())
            o16.append(out.cpu())
        outs.append(tuple(o16))
        lses.append(tuple(x.cpu() for x in l_acc))
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o = ring.unshard_zigzag(outs, world)
    lse = ring.unshard_zigzag(lses, world, dim=2)
    return o, lse


@pytest.mark.parametrize("world,B,Hq,Hkv,C,d,causal", [
    (2, 2, 4, 2, 192, 128, True),
    (4, 1, 8, 2, 128, 128, True),
    (3, 1, 4, 4, 100, 64, True),      # chunks that are not a multiple of the 128-row tile
    (3, 2, 4, 1, 96, 128, False),
])
def test_emulated_ring_matches_whole_sequence(world, B, Hq, Hkv, C, d, causal):
    N = 2 * world * C
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed=90 + world)
    scale = default_scale(d)
    o, lse = emulate_ring(q, k, v, world, scale=scale, causal=causal)
    o_ref, lse_ref = ref(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=causal)
    dO = float(np.abs(o.to(torch.float64).numpy() - o_ref).max())
    dL = float(np.abs(lse.to(torch.float64).numpy() - lse_ref).max())
    assert dO <= TOL_O and dL <= TOL_LSE, (dO, dL)


def test_accumulate_two_key_halves_equals_one_call():
    """Non-causal attention over keys [0, N) accumulated as two halves equals
    one attn_fwd over all keys: same LSE, O within the bf16 rounding of the
    single-call output."""
    B, N, Hq, Hkv, d = 2, 256, 4, 2, 128
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, 2 * N, Hkv, d), seed=3)
    scale = default_scale(d)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o_acc = torch.zeros((B, N, Hq, d), dtype=torch.float32, device=DEV)
    l_acc = torch.full((B, Hq, N), float("-inf"), dtype=torch.float32, device=DEV)
    for half in range(2):
        kh = kd[:, half * N:(half + 1) * N].contiguous()
        vh = vd[:, half * N:(half + 1) * N].contiguous()
        ea.attn_fwd_accumulate(qd, kh, vh, o_acc, l_acc, B, Hq, Hkv, N, d, scale, False)
    torch.cuda.synchronize()
    # oracle: each query over all 2N keys (non-causal), via a 2N-token problem
    q2 = torch.cat([q, torch.zeros_like(q)], dim=1)
    o_ref, lse_ref = ref(q2, k, v, B=B, Hq=Hq, Hkv=Hkv, N=2 * N, d=d, scale=scale, causal=False)
    assert float(np.abs(o_acc.cpu().double().numpy() - o_ref[:, :N]).max()) <= 2e-3
    assert float(np.abs(l_acc.cpu().double().numpy() - lse_ref[:, :, :N]).max()) <= TOL_LSE


def test_single_rank_ring_forward():
    """ring_attention_forward without a process group (one rank, two chunks)."""
    B, Hq, Hkv, C, d = 1, 4, 2, 160, 128
    N = 2 * C
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed=11)
    scale = default_scale(d)
    qs, ks, vs = ([x.to(DEV) for x in ring.shard_zigzag(t, 1, 0)] for t in (q, k, v))
    outs, lses = ring.ring_attention_forward(qs, ks, vs, scale=scale, causal=True)
    torch.cuda.synchronize()
    o = ring.unshard_zigzag([tuple(x.cpu() for x in outs)], 1).double().numpy()
    lse = ring.unshard_zigzag([tuple(x.cpu() for x in lses)], 1, dim=2).double().numpy()
    o_ref, lse_ref = ref(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=True)
    assert float(np.abs(o - o_ref).max()) <= TOL_O
    assert float(np.abs(lse - lse_ref).max()) <= TOL_LSE


def test_acc_to_bf16_rounds_to_nearest_even():
    x = torch.tensor([1.0, 1.00390625, 1.01171875, -2.5, 3.0e38, 1.5e-30, 0.0, -0.0, 7.0],
                     dtype=torch.float32)
    n = x.numel()
    xd = x.to(DEV)
    out = torch.empty(16, dtype=torch.bfloat16, device=DEV)
    ea.attn_acc_to_bf16(xd, out, n)
    torch.cuda.synchronize()
    assert torch.equal(out[:n].cpu().view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


def test_accumulate_ignores_empty_rows_contents():
    """A row whose accumulator LSE is -inf is empty: whatever its O holds (NaN
    here) is not read, so an unzeroed accumulator gives the attention output."""
    B, N, Hq, Hkv, d = 1, 300, 4, 2, 128
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed=9)
    scale = default_scale(d)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o_acc = torch.full((B, N, Hq, d), float("nan"), dtype=torch.float32, device=DEV)
    l_acc = torch.full((B, Hq, N), float("-inf"), dtype=torch.float32, device=DEV)
    ea.attn_fwd_accumulate(qd, kd, vd, o_acc, l_acc, B, Hq, Hkv, N, d, scale, True)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, lse_ref = ref(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=True)
    got = o_acc.cpu().double().numpy()
    assert np.isfinite(got).all()
    assert float(np.abs(got - o_ref).max()) <= 5e-3
    assert float(np.abs(l_acc.cpu().double().numpy() - lse_ref).max()) <= TOL_LSE
