"""attn_decode_noalloc: the key/value-cache decode for callers that must not
allocate device memory while they run (a serving loop whose page pool holds
nearly all of HBM, or a latency-bound step loop, where cudaMalloc / cudaFree can
block on the device or fail).  It keeps its slice partials in a fixed 8 MiB
array inside the library instead of a caller-provided workspace.

Checked through the C ABI against attn_decode with a torch-allocated workspace,
on two calls in a row with different shapes and slice counts, so the second
call runs on whatever the first left in the shared array.  This file is named
to be collected last; it also passes alone in a fresh process."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import workloads as W

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL_O = 1e-2
TOL_LSE = 1e-3


def _inputs(w: W.DecodeWorkload):
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    return (q.to(DEV), kc.to(DEV), vc.to(DEV), seqlens.to(DEV),
            table.to(DEV) if table is not None else None)


def _outputs(w):
    o = torch.full((w.B, w.Nq, w.Hq, w.d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((w.B, w.Hq, w.Nq), float("nan"), dtype=torch.float32, device=DEV)
    return o, lse


def _with_workspace(w, ins, splits):
    q, kc, vc, sd, td = ins
    o, lse = _outputs(w)
    nbytes = ea.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                                            w.pages_per_seq, splits)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    ea.attn_decode(q, kc, vc, o, lse, sd, td, w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                   w.pages_per_seq, kc.shape[0], w.scale, w.causal, w.window_left,
                   w.window_right, splits, ws, nbytes)
    return o, lse


def _no_alloc(w, ins, splits):
    q, kc, vc, sd, td = ins
    o, lse = _outputs(w)
    ea.attn_decode_noalloc(q, kc, vc, o, lse, sd, td, w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                           w.pages_per_seq, kc.shape[0], w.scale, w.causal, w.window_left,
                           w.window_right, splits)
    return o, lse


def _close(a, b):
    (oa, la), (ob, lb) = a, b
    assert torch.isfinite(oa.float()).all() and torch.isfinite(la).all()
    assert float((oa.float() - ob.float()).abs().max()) <= TOL_O
    assert float((la - lb).abs().max()) <= TOL_LSE


def test_no_alloc_matches_workspace_entry_two_calls_in_a_row():
    first = W.DecodeWorkload("first", 3, 16, 4, 2, 128, 32, 40, [1280, 77, 900], True, True,
                             -1, -1, 21)
    second = W.DecodeWorkload("second", 2, 8, 2, 3, 64, 16, 64, [1000, 333], True, True, 200,
                              -1, 22)
    cases = [(first, _inputs(first), 6), (second, _inputs(second), 4)]
    for w, _, splits in cases:
        need = ea.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                                              w.pages_per_seq, splits)
        assert 0 < need <= ea.ATTN_DECODE_NOALLOC_SCRATCH_BYTES  # really uses the scratch
    refs = [_with_workspace(w, ins, s) for w, ins, s in cases]
    got = [_no_alloc(w, ins, s) for w, ins, s in cases]  # two calls in a row
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for g, r in zip(got, refs):
        _close(g, r)
    # and once more on the first shape, after the second call changed the array
    again = _no_alloc(*cases[0])
    torch.cuda.synchronize()
    _close(again, refs[0])


def test_no_alloc_rejects_a_call_beyond_the_scratch():
    # 256 sequences x 32 heads x 128 columns x 16 slices of fp32 partials: 64 MiB
    B, Hq, Hkv, Nq, d, page, pps, splits = 256, 32, 8, 1, 128, 64, 128, 16
    need = ea.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, page, pps, splits)
    assert need > ea.ATTN_DECODE_NOALLOC_SCRATCH_BYTES
    fake = 1 << 20  # never touched: the size check comes first
    rc = ea.attn_decode_noalloc(fake, fake, fake, fake, fake, fake, fake, B, Hq, Hkv, Nq, d, page,
                                pps, B * pps, 0.1, True, -1, -1, splits, check=False)
    assert rc == ea.ATTN_ERR_WORKSPACE
    # a single slice needs no scratch at all, whatever the size
    assert ea.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, page, pps, 1) == 0
