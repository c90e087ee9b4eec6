"""GPU parity of attn_bwd (dQ, dK, dV) with the fp64 oracle's gradients, through
the C ABI.  The GPU backward takes o and lse from the GPU forward (as a caller
would); the oracle computes its own weights from q, k, v.

Tolerance: max|dX_gpu - dX_ref| <= 1e-2 * max|dX_ref| + 1e-4 for each of dQ,
dK, dV.  The outputs are rounded once to bf16 (half an ulp: 2^-9 of the
element), and the products take P and dS rounded to bf16 (2^-9 relative per
term, largely cancelling over the sums), with fp32 accumulation.  The absolute
floor covers gradients that are exactly zero (a row with a single visible
key has dS = P (dP - D) = 0): there dP and D, each ~|dO||v| ~ 10, cancel in
fp32 (2^-24 relative), and dK = scale * dS^T q carries that ~1e-6."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import oracle
import workloads as W
from gpu_helpers import default_scale

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
REL_TOL = 1e-2
ABS_FLOOR = 1e-4


def draw(shape_q, shape_kv, seed):
    q, k, v = W.draw_qkv(shape_q, shape_kv, seed)
    g = torch.Generator().manual_seed(seed + 1000)
    do = torch.randn(shape_q, dtype=torch.float32, generator=g).to(torch.bfloat16)
    return q, k, v, do


def gpu_bwd(q, k, v, do, *, B, Hq, Hkv, N, d, scale, causal, left=-1, right=-1, cu=None):
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    packed = cu is not None
    cud = torch.tensor(cu, dtype=torch.int32, device=DEV) if packed else None
    max_seqlen = max(b - a for a, b in zip(cu[:-1], cu[1:])) if packed else 0
    o = torch.empty_like(qd)
    lse = torch.empty((Hq * N,) if packed else (B * Hq * N,), dtype=torch.float32, device=DEV)
    ea.attn_fwd(qd, kd, vd, o, lse, B, Hq, Hkv, N, d, scale, causal, left, right, cud, max_seqlen)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(vd, float("nan"))
    nbytes = ea.attn_bwd_workspace_bytes(B, Hq, Hkv, N, d, packed)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV)
    ea.attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal, left, right,
                cud, max_seqlen, ws, nbytes)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return dq.cpu(), dk.cpu(), dv.cpu()


def ref_bwd(q, k, v, do, *, B, Hq, Hkv, N, d, scale, causal, left=-1, right=-1, cu=None):
    return oracle.attn_bwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), W.bf16_bits(do), B=B,
                           Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=causal,
                           window_left=left, window_right=right, cu_seqlens=cu)


def compare(got, ref):
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        gf = g.to(torch.float64).numpy().reshape(r.shape)
        assert np.isfinite(gf).all(), f"{name}: non-finite"
        err = float(np.abs(gf - r).max())
        scale = float(np.abs(r).max())
        assert err <= REL_TOL * scale + ABS_FLOOR, f"{name}: max|d| = {err}, max|ref| = {scale}"


CASES = [
    # B, Hq, Hkv, N, d, causal, left, right
    (2, 4, 4, 256, 128, True, -1, -1),
    (2, 8, 2, 300, 128, True, -1, -1),     # GQA, ragged tail
    (1, 4, 1, 200, 64, False, -1, -1),     # MQA, d = 64
    (1, 4, 2, 400, 128, True, 100, 0),     # sliding window
    (2, 2, 2, 333, 64, False, 50, 30),     # two-sided window
    (1, 2, 1, 1, 128, True, -1, -1),
    (1, 2, 2, 127, 128, True, -1, -1),
    (1, 2, 2, 129, 64, True, -1, -1),
    (1, 6, 3, 520, 128, False, -1, -1),    # group 2, several full blocks
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_h{}x{}_n{}_d{}_c{}_w{}_{}".format(*c))
def test_bwd_parity(case):
    B, Hq, Hkv, N, d, causal, left, right = case
    q, k, v, do = draw((B, N, Hq, d), (B, N, Hkv, d), seed=N + Hq)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=causal, left=left,
              right=right)
    compare(gpu_bwd(q, k, v, do, **kw), ref_bwd(q, k, v, do, **kw))


@pytest.mark.parametrize("d", [128, 64])
def test_bwd_packed(d):
    lens = [100, 1, 257, 130, 0, 64]
    cu = W.cumulative(lens)
    T, Hq, Hkv = cu[-1], 4, 2
    q, k, v, do = draw((T, Hq, d), (T, Hkv, d), seed=77)
    kw = dict(B=len(lens), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=default_scale(d), causal=True, cu=cu)
    compare(gpu_bwd(q, k, v, do, **kw), ref_bwd(q, k, v, do, **kw))


def test_bwd_deterministic():
    B, Hq, Hkv, N, d = 1, 4, 2, 384, 128
    q, k, v, do = draw((B, N, Hq, d), (B, N, Hkv, d), seed=5)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=True)
    a = gpu_bwd(q, k, v, do, **kw)
    b = gpu_bwd(q, k, v, do, **kw)
    for x, y in zip(a, b):
        assert torch.equal(x.view(torch.int16), y.view(torch.int16))


def test_bwd_causal_mha_workload_one_head():
    """The causal MHA workload (B=4, H=16, N=2048, d=128) on the GPU; the oracle
    checks sequence 2, head 5 (a sub-problem whose gradients depend only on
    its own q, k, v, dout)."""
    w = W.workload(2)
    q, k, v = W.inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1000)
    do = torch.randn(q.shape, dtype=torch.float32, generator=g).to(torch.bfloat16)
    kw = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, scale=w.scale, causal=True)
    dq, dk, dv = gpu_bwd(q, k, v, do, **kw)
    b, h = 2, 5
    sub = lambda t: t[b:b + 1, :, h:h + 1].contiguous()
    ref = ref_bwd(sub(q), sub(k), sub(v), sub(do), B=1, Hq=1, Hkv=1, N=w.N, d=w.d,
                  scale=w.scale, causal=True)
    compare((dq[b:b + 1, :, h:h + 1], dk[b:b + 1, :, h:h + 1], dv[b:b + 1, :, h:h + 1]), ref)


def test_bwd_causal_gqa_workload_one_group():
    """The benchmark's causal GQA workload (B=2, Hq=32, Hkv=8, N=8192, d=128) on
    the GPU; the oracle checks sequence 1, K/V head 5 with its four query heads
    (a sub-problem whose gradients depend only on its own q, k, v, dout)."""
    w = W.workload(3)
    q, k, v = W.inputs(w)
    g = torch.Generator().manual_seed(w.seed + 1000)
    do = torch.randn(q.shape, dtype=torch.float32, generator=g).to(torch.bfloat16)
    kw = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, scale=w.scale, causal=True)
    dq, dk, dv = gpu_bwd(q, k, v, do, **kw)
    b, gkv = 1, 5
    grp = w.Hq // w.Hkv
    hs = slice(gkv * grp, (gkv + 1) * grp)
    subq = lambda t: t[b:b + 1, :, hs].contiguous()
    subk = lambda t: t[b:b + 1, :, gkv:gkv + 1].contiguous()
    ref = ref_bwd(subq(q), subk(k), subk(v), subq(do), B=1, Hq=grp, Hkv=1, N=w.N, d=w.d,
                  scale=w.scale, causal=True)
    compare((dq[b:b + 1, :, hs], dk[b:b + 1, :, gkv:gkv + 1], dv[b:b + 1, :, gkv:gkv + 1]), ref)


def test_bwd_packed_max_seqlen_too_small_is_reported():
    """A sequence longer than max_seqlen (rounded up to 128) is skipped by the
    gradient kernels -- its rows of dq, dk, dv are left as they were -- and the
    status word reports it; the other sequences match a call with the right
    max_seqlen.  Every address stays inside the tensors."""
    lens = [300, 129, 50]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 128
    q, k, v, do = draw((T, Hq, d), (T, Hkv, d), 81)
    scale = default_scale(d)
    good = gpu_bwd(q, k, v, do, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=scale, causal=True, cu=cu)
    qd, kd, vd, dod = (t.to(DEV) for t in (q, k, v, do))
    cud = torch.tensor(cu, dtype=torch.int32, device=DEV)
    o = torch.empty_like(qd)
    lse = torch.empty((Hq * T,), dtype=torch.float32, device=DEV)
    ea.attn_fwd(qd, kd, vd, o, lse, 3, Hq, Hkv, T, d, scale, True, -1, -1, cud, 300)
    dq = torch.full_like(qd, float("nan"))
    dk = torch.full_like(kd, float("nan"))
    dv = torch.full_like(vd, float("nan"))
    nbytes = ea.attn_bwd_workspace_bytes(3, Hq, Hkv, T, d, True)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV)
    ea.attn_bwd(qd, kd, vd, o, lse, dod, dq, dk, dv, 3, Hq, Hkv, T, d, scale, True, -1, -1, cud, 200,
                ws, nbytes)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_SEQLENS
    assert ea.attn_device_status() == ea.ATTN_OK
    for got, ref in zip((dq.cpu(), dk.cpu(), dv.cpu()), good):
        assert torch.isnan(got[:300].float()).all()
        g, r = got[300:].double(), ref[300:].double()
        assert float((g - r).abs().max()) <= REL_TOL * float(r.abs().max()) + ABS_FLOOR
