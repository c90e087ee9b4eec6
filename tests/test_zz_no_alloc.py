"""attn_decode_noalloc: the key/value-cache decode for callers that must not
allocate device memory while they run (a serving loop whose page pool holds
nearly all of HBM, or a latency-bound step loop, where cudaMalloc / cudaFree can
block on the device or fail).  It keeps its slice partials in a fixed array
inside the library instead of a caller-provided workspace.

Checked through the C ABI against the fp64 oracle's key/value-cache entry and
against attn_decode with a torch-allocated workspace, on two calls in a row with
different shapes and slice counts, so the second call runs on whatever the
first left in the shared array.  A call whose partials would not fit the array
is rejected; that check is exercised in a child process that sees no GPU
(tests/test_abi.py), so no kernel can ever run on it.  This file is named to be
collected last; it also passes alone in a fresh process."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import oracle
import workloads as W

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")
TOL_O = 1e-2
TOL_LSE = 1e-3


def _inputs(w: W.DecodeWorkload):
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    host = (q, kc, vc, seqlens, table)
    dev = (q.to(DEV), kc.to(DEV), vc.to(DEV), seqlens.to(DEV),
           table.to(DEV) if table is not None else None)
    return host, dev


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


def _oracle(w, host):
    q, kc, vc, seqlens, table = host
    o, lse, _ = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc),
                                    seqlens.numpy(), B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, d=w.d,
                                    page_size=w.page_size, pages_per_seq=w.pages_per_seq,
                                    scale=w.scale, causal=w.causal, window_left=w.window_left,
                                    window_right=w.window_right,
                                    block_table=None if table is None else table.numpy())
    return o, lse


def _close_to_oracle(got, ref):
    (o, lse), (o_ref, lse_ref) = got, ref
    og = o.cpu().to(torch.float64).numpy()
    lg = lse.cpu().to(torch.float64).numpy()
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    assert float(np.abs(og - o_ref).max()) <= TOL_O
    assert float(np.abs(lg - lse_ref).max()) <= TOL_LSE


def _close(a, b):
    (oa, la), (ob, lb) = a, b
    assert torch.isfinite(oa.float()).all() and torch.isfinite(la).all()
    assert float((oa.float() - ob.float()).abs().max()) <= TOL_O
    assert float((la - lb).abs().max()) <= TOL_LSE


def test_no_alloc_matches_oracle_two_calls_in_a_row():
    first = W.DecodeWorkload("first", 3, 16, 4, 2, 128, 32, 40, [1280, 77, 900], True, True,
                             -1, -1, 21)
    second = W.DecodeWorkload("second", 2, 8, 2, 3, 64, 16, 64, [1000, 333], True, True, 200,
                              -1, 22)
    scratch = ea.attn_decode_noalloc_scratch_bytes()
    cases = []
    for w, splits in ((first, 6), (second, 4)):
        need = ea.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                                              w.pages_per_seq, splits)
        assert 0 < need <= scratch  # really uses the scratch
        host, dev = _inputs(w)
        cases.append((w, host, dev, splits))
    refs = [_oracle(w, host) for w, host, _, _ in cases]
    with_ws = [_with_workspace(w, dev, s) for w, _, dev, s in cases]
    got = [_no_alloc(w, dev, s) for w, _, dev, s in cases]  # two calls in a row
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    for g, r, ws in zip(got, refs, with_ws):
        _close_to_oracle(g, r)
        _close(g, ws)
    # and once more on the first shape, after the second call changed the array
    w, _, dev, splits = cases[0]
    again = _no_alloc(w, dev, splits)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    _close_to_oracle(again, refs[0])


def test_no_alloc_rejects_bad_arguments_before_touching_the_scratch():
    """A NULL query pointer is reported as attn_decode reports it, before the
    library looks up or touches its array."""
    w = W.DecodeWorkload("bad", 2, 8, 2, 1, 128, 32, 8, [100, 200], True, True, -1, -1, 23)
    _, (q, kc, vc, sd, td) = _inputs(w)
    o, lse = _outputs(w)
    rc = ea.attn_decode_noalloc(None, kc, vc, o, lse, sd, td, w.B, w.Hq, w.Hkv, w.Nq, w.d,
                                w.page_size, w.pages_per_seq, kc.shape[0], w.scale, True, -1, -1,
                                2, check=False)
    assert rc == ea.ATTN_ERR_NULL
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
