"""Pins that tie the fp64 oracle to something other than itself.

Each pin is a plain function taking a loaded oracle library (ctypes handle) and
raising AssertionError on a mismatch.  ``test_oracle_pins.py`` runs them on the
real oracle; ``test_oracle_mutants.py`` runs them on copies of the oracle with a
planted mistake and requires that at least one pin fails for every mistake.

What pins what:
  * worked example  -- the numbers printed on the "FlashAttention" explainer
    page (ozercemkelahmet.com), "A worked example" / "Online softmax by hand"
    (tests/golden/worked_example.json): exponent values, normaliser, and the
    block-merge rule, all in the page's notation.
  * uniform scores  -- Q = 0 makes every visible weight equal, so O is the mean
    of V over the visible key range and LSE = ln(count): a closed form that pins
    the mask (inclusive window bounds, causal override, sequence boundaries).
  * two keys        -- softmax of two scores is the logistic function
    (scipy.special.expit) and the LSE is numpy.logaddexp.
  * hard limit      -- a very large scale turns softmax into argmax.
  * single key / causal row 0 -- O = v_0, LSE = scale * q.k_0.
  * invariants      -- constant V, rows summing to one, key permutation
    (non-causal), window >= N-1 equals causal, packed == separate calls,
    grouped-query == key/value heads repeated per query head.
  * library routine -- torch.nn.functional.scaled_dot_product_attention in
    float64 on the CPU with a band mask built by torch.triu / torch.tril (the
    page's own causal-mask recipe in "Checking correctness"), and
    torch.logsumexp for the LSE.
  * gradients       -- central finite differences of sum(dO * O) computed by a
    numpy forward written in the pin; torch autograd through float64
    scaled_dot_product_attention; the zero-sum of key gradients and the
    value-gradient sum; packed == separate; grouped == repeated with the
    gradients summed.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _bf16(x) -> torch.Tensor:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    return t.to(torch.bfloat16)


def _run(lib, q, k, v, **kw):
    """q [B,N,Hq,d] / k,v [B,N,Hkv,d] (or packed [T,H,d]) bf16 tensors."""
    return oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), lib=lib, **kw)


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.to(torch.float64).numpy()


# --------------------------------------------------------------------------
# worked example from the page
# --------------------------------------------------------------------------
def pin_worked_example(lib):
    g = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    s = g["scores"]
    n = len(s)
    half_ulp = 0.5 * 10.0 ** (-g["printed_decimals"])
    d = 4
    # q = e_0, k_j = s_j e_0 so that q.k_j = s_j; v_j = e_j so that O = the weights.
    q = np.zeros((1, n, 1, d), np.float32)
    q[0, :, 0, 0] = 1.0
    k = np.zeros((1, n, 1, d), np.float32)
    k[0, :, 0, 0] = s
    v = np.zeros((1, n, 1, d), np.float32)
    for j in range(n):
        v[0, j, 0, j] = 1.0
    o, lse, nvis = _run(lib, _bf16(q), _bf16(k), _bf16(v), B=1, Hq=1, Hkv=1, N=n, d=d,
                        scale=1.0, causal=False)
    M = g["direct"]["max"]
    Z = math.exp(lse[0, 0, 0] - M)
    # direct computation: the normaliser and each exponent relative to the max
    assert abs(Z - g["direct"]["sum"]) <= half_ulp, (Z, g["direct"]["sum"])
    for j in range(n):
        assert abs(o[0, 0, j] * Z - g["direct"]["exps"][j]) <= half_ulp, (j, o[0, 0, j] * Z)
    # online: the page's final sum adds two rounded terms
    assert abs(Z - g["online_final_sum"]) <= 2 * half_ulp
    assert nvis[0, 0, 0] == n
    # block by block: run the oracle on each key block alone
    lse_blocks = []
    for blk, ref in zip(g["blocks"], (g["block1"], g["block2"])):
        nb = len(blk)
        kb = np.ascontiguousarray(k[:, blk])
        vb = np.zeros((1, nb, 1, d), np.float32)
        for jj in range(nb):
            vb[0, jj, 0, jj] = 1.0
        qb = np.ascontiguousarray(q[:, :nb])
        ob, lb, _ = _run(lib, _bf16(qb), _bf16(kb), _bf16(vb), B=1, Hq=1, Hkv=1, N=nb, d=d,
                         scale=1.0, causal=False)
        Zb = math.exp(lb[0, 0, 0] - ref["max"])
        assert abs(Zb - ref["sum"]) <= half_ulp, (Zb, ref["sum"])
        for jj in range(nb):
            assert abs(ob[0, 0, jj] * Zb - ref["exps"][jj]) <= half_ulp
        lse_blocks.append(lb[0, 0, 0])
    # the rescale step: block 1's sum times exp(m1 - m2) is the page's 0.154
    rescale = math.exp(g["block1"]["max"] - g["block2"]["max"])
    assert abs(rescale - g["rescale_factor"]) <= half_ulp
    assert abs(math.exp(lse_blocks[0] - M) - g["rescaled_block1_sum"]) <= half_ulp
    # merging the two partial results by the same rule gives the whole row
    merged = np.logaddexp(lse_blocks[0], lse_blocks[1])
    assert abs(merged - lse[0, 0, 0]) <= 1e-12


# --------------------------------------------------------------------------
# closed forms
# --------------------------------------------------------------------------
def _visible_range(i, L, left, right, causal):
    """Closed form of the visible key range of row i (inclusive ends)."""
    if causal:
        right = 0
    lo = 0 if left < 0 else max(0, i - left)
    hi = L - 1 if right < 0 else min(L - 1, i + right)
    return lo, hi


MASK_CASES = [
    # (N, causal, left, right)
    (13, False, -1, -1),
    (13, True, -1, -1),
    (13, True, 3, 0),
    (13, False, 2, 5),
    (13, False, 0, 0),
    (13, False, -1, 2),
    (13, False, 4, -1),
    (13, True, 4, 7),  # causal wins over a positive right window
    (1, True, -1, -1),
]


def pin_uniform_scores(lib):
    rng = np.random.default_rng(11)
    d = 8
    for (N, causal, left, right) in MASK_CASES:
        q = np.zeros((1, N, 2, d), np.float32)
        k = rng.standard_normal((1, N, 1, d)).astype(np.float32)
        v = rng.integers(-8, 9, size=(1, N, 1, d)).astype(np.float32)  # exact in bf16
        o, lse, nvis = _run(lib, _bf16(q), _bf16(k), _bf16(v), B=1, Hq=2, Hkv=1, N=N, d=d,
                            scale=0.7, causal=causal, window_left=left, window_right=right)
        for h in range(2):
            for i in range(N):
                lo, hi = _visible_range(i, N, left, right, causal)
                cnt = hi - lo + 1
                assert nvis[0, h, i] == cnt, ((N, causal, left, right), i, nvis[0, h, i], cnt)
                mean = v[0, lo:hi + 1, 0, :].astype(np.float64).mean(axis=0)
                assert np.allclose(o[i, h], mean, rtol=0, atol=1e-13), ((N, causal, left, right), i)
                assert abs(lse[0, h, i] - math.log(cnt)) <= 1e-13


def pin_uniform_scores_packed(lib):
    rng = np.random.default_rng(12)
    d = 4
    lens = [5, 1, 9, 3]
    cu = W.cumulative(lens)
    T = cu[-1]
    for (causal, left, right) in [(True, -1, -1), (False, -1, -1), (True, 2, 0), (False, 1, 3)]:
        q = np.zeros((T, 3, d), np.float32)
        k = rng.standard_normal((T, 3, d)).astype(np.float32)
        v = rng.integers(-8, 9, size=(T, 3, d)).astype(np.float32)
        o, lse, nvis = _run(lib, _bf16(q), _bf16(k), _bf16(v), B=len(lens), Hq=3, Hkv=3, N=T,
                            d=d, scale=1.0, causal=causal, window_left=left,
                            window_right=right, cu_seqlens=cu)
        for b, L in enumerate(lens):
            for h in range(3):
                for i in range(L):
                    lo, hi = _visible_range(i, L, left, right, causal)
                    t0 = cu[b]
                    mean = v[t0 + lo:t0 + hi + 1, h, :].astype(np.float64).mean(axis=0)
                    assert np.allclose(o[t0 + i, h], mean, rtol=0, atol=1e-13), (b, h, i)
                    assert nvis[h, t0 + i] == hi - lo + 1
                    assert abs(lse[h, t0 + i] - math.log(hi - lo + 1)) <= 1e-13


def pin_two_keys(lib):
    from scipy.special import expit
    rng = np.random.default_rng(13)
    d = 16
    q = _bf16(rng.standard_normal((1, 2, 1, d)))
    k = _bf16(rng.standard_normal((1, 2, 1, d)))
    v = _bf16(rng.standard_normal((1, 2, 1, d)))
    scale = 0.25
    o, lse, _ = _run(lib, q, k, v, B=1, Hq=1, Hkv=1, N=2, d=d, scale=scale, causal=False)
    qf, kf, vf = _f64(q)[0, :, 0], _f64(k)[0, :, 0], _f64(v)[0, :, 0]
    for i in range(2):
        s0 = scale * float(np.dot(qf[i], kf[0]))
        s1 = scale * float(np.dot(qf[i], kf[1]))
        w1 = float(expit(s1 - s0))
        expect = (1.0 - w1) * vf[0] + w1 * vf[1]
        assert np.allclose(o[i, 0], expect, rtol=0, atol=1e-12), i
        assert abs(lse[0, 0, i] - np.logaddexp(s0, s1)) <= 1e-12


def pin_hard_limit(lib):
    # distinct integer scores times a huge scale: softmax -> one-hot at argmax
    N, d = 6, 8
    rng = np.random.default_rng(14)
    q = np.zeros((1, N, 1, d), np.float32)
    q[..., 0] = 1.0
    perm = rng.permutation(N).astype(np.float32)
    k = np.zeros((1, N, 1, d), np.float32)
    k[0, :, 0, 0] = perm
    v = rng.integers(-5, 6, size=(1, N, 1, d)).astype(np.float32)
    o, lse, _ = _run(lib, _bf16(q), _bf16(k), _bf16(v), B=1, Hq=1, Hkv=1, N=N, d=d,
                     scale=80.0, causal=False)
    j = int(np.argmax(perm))
    for i in range(N):
        assert np.allclose(o[i, 0], v[0, j, 0], rtol=0, atol=1e-12)
        assert abs(lse[0, 0, i] - 80.0 * perm[j]) <= 1e-9


def pin_single_key_and_row0(lib):
    rng = np.random.default_rng(15)
    d = 32
    q = _bf16(rng.standard_normal((2, 5, 2, d)))
    k = _bf16(rng.standard_normal((2, 5, 2, d)))
    v = _bf16(rng.standard_normal((2, 5, 2, d)))
    scale = 0.3
    # causal: row 0 sees only key 0
    o, lse, _ = _run(lib, q, k, v, B=2, Hq=2, Hkv=2, N=5, d=d, scale=scale, causal=True)
    o = o.reshape(2, 5, 2, d)
    qf, kf, vf = _f64(q), _f64(k), _f64(v)
    for b in range(2):
        for h in range(2):
            assert np.array_equal(o[b, 0, h], vf[b, 0, h])
            assert abs(lse[b, h, 0] - scale * float(np.dot(qf[b, 0, h], kf[b, 0, h]))) <= 1e-12
    # N = 1
    o1, lse1, _ = _run(lib, q[:, :1].contiguous(), k[:, :1].contiguous(), v[:, :1].contiguous(),
                       B=2, Hq=2, Hkv=2, N=1, d=d, scale=scale, causal=False)
    o1 = o1.reshape(2, 1, 2, d)
    assert np.array_equal(o1[:, 0], vf[:, 0])


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------
def pin_constant_v_and_row_sums(lib):
    rng = np.random.default_rng(16)
    N, d = 40, 16
    q = _bf16(rng.standard_normal((1, N, 2, d)) * 2)
    k = _bf16(rng.standard_normal((1, N, 2, d)) * 2)
    c = rng.integers(-4, 5, size=(d,)).astype(np.float32)
    v = _bf16(np.broadcast_to(c, (1, N, 2, d)).copy())
    ones = _bf16(np.ones((1, N, 2, d), np.float32))
    for causal, left, right in [(False, -1, -1), (True, -1, -1), (False, 5, 3)]:
        o, _, _ = _run(lib, q, k, v, B=1, Hq=2, Hkv=2, N=N, d=d, scale=0.5, causal=causal,
                       window_left=left, window_right=right)
        assert np.allclose(o, np.broadcast_to(c, o.shape), rtol=0, atol=1e-12)
        o1, _, _ = _run(lib, q, k, ones, B=1, Hq=2, Hkv=2, N=N, d=d, scale=0.5, causal=causal,
                        window_left=left, window_right=right)
        assert np.abs(o1 - 1.0).max() <= 1e-12  # rows of P sum to one


def pin_key_permutation(lib):
    rng = np.random.default_rng(17)
    N, d = 33, 16
    q = _bf16(rng.standard_normal((1, N, 1, d)))
    k = _bf16(rng.standard_normal((1, N, 1, d)))
    v = _bf16(rng.standard_normal((1, N, 1, d)))
    perm = torch.as_tensor(rng.permutation(N))
    o, lse, _ = _run(lib, q, k, v, B=1, Hq=1, Hkv=1, N=N, d=d, scale=0.4, causal=False)
    op, lsep, _ = _run(lib, q, k[:, perm].contiguous(), v[:, perm].contiguous(), B=1, Hq=1,
                       Hkv=1, N=N, d=d, scale=0.4, causal=False)
    assert np.abs(o - op).max() <= 1e-12
    assert np.abs(lse - lsep).max() <= 1e-12


def pin_window_equals_causal(lib):
    rng = np.random.default_rng(18)
    N, d = 37, 8
    q = _bf16(rng.standard_normal((2, N, 2, d)))
    k = _bf16(rng.standard_normal((2, N, 1, d)))
    v = _bf16(rng.standard_normal((2, N, 1, d)))
    base, lb, _ = _run(lib, q, k, v, B=2, Hq=2, Hkv=1, N=N, d=d, scale=0.5, causal=True)
    for left in (N - 1, N, 5 * N):
        o, l, _ = _run(lib, q, k, v, B=2, Hq=2, Hkv=1, N=N, d=d, scale=0.5, causal=False,
                       window_left=left, window_right=0)
        assert np.array_equal(o, base) and np.array_equal(l, lb)


def pin_packed_equals_separate(lib):
    rng = np.random.default_rng(19)
    lens = [7, 1, 12, 4]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 8
    q = _bf16(rng.standard_normal((T, Hq, d)))
    k = _bf16(rng.standard_normal((T, Hkv, d)))
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    for causal, left, right in [(True, -1, -1), (False, -1, -1), (False, 2, 1)]:
        o, lse, _ = _run(lib, q, k, v, B=len(lens), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=0.6,
                         causal=causal, window_left=left, window_right=right, cu_seqlens=cu)
        for b, L in enumerate(lens):
            a = cu[b]
            ob, lb, _ = _run(lib, q[a:a + L].unsqueeze(0).contiguous(),
                             k[a:a + L].unsqueeze(0).contiguous(),
                             v[a:a + L].unsqueeze(0).contiguous(), B=1, Hq=Hq, Hkv=Hkv, N=L,
                             d=d, scale=0.6, causal=causal, window_left=left, window_right=right)
            assert np.array_equal(o[a:a + L], ob)
            assert np.array_equal(lse[:, a:a + L], lb[0])


def pin_gqa_equals_repeated(lib):
    rng = np.random.default_rng(20)
    B, N, Hq, Hkv, d = 2, 19, 6, 2, 8
    q = _bf16(rng.standard_normal((B, N, Hq, d)))
    k = _bf16(rng.standard_normal((B, N, Hkv, d)))
    v = _bf16(rng.standard_normal((B, N, Hkv, d)))
    o, lse, _ = _run(lib, q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=0.5, causal=True)
    kr = torch.repeat_interleave(k, Hq // Hkv, dim=2).contiguous()
    vr = torch.repeat_interleave(v, Hq // Hkv, dim=2).contiguous()
    o2, lse2, _ = _run(lib, q, kr, vr, B=B, Hq=Hq, Hkv=Hq, N=N, d=d, scale=0.5, causal=True)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


# --------------------------------------------------------------------------
# independent library routine
# --------------------------------------------------------------------------
def _band_mask(N, causal, left, right):
    """Visible-key matrix from torch.triu/torch.tril, as the page's recipe builds
    its causal mask with torch.triu(ones, 1)."""
    ones = torch.ones(N, N, dtype=torch.bool)
    if causal:
        right = 0
    allowed = ones.clone()
    if right >= 0:
        allowed &= ~torch.triu(ones, diagonal=right + 1)
    if left >= 0:
        allowed &= ~torch.tril(ones, diagonal=-left - 1)
    return allowed


def pin_torch_sdpa(lib):
    import torch.nn.functional as F
    rng = np.random.default_rng(21)
    cases = [
        # B, N, Hq, Hkv, d, causal, left, right, scale
        (2, 45, 4, 4, 32, False, -1, -1, 32 ** -0.5),
        (1, 70, 4, 2, 64, True, -1, -1, 64 ** -0.5),
        (2, 33, 6, 3, 16, True, 7, 0, 0.3),
        (1, 50, 2, 1, 8, False, 3, 9, 1.1),
    ]
    for (B, N, Hq, Hkv, d, causal, left, right, scale) in cases:
        q = _bf16(rng.standard_normal((B, N, Hq, d)))
        k = _bf16(rng.standard_normal((B, N, Hkv, d)))
        v = _bf16(rng.standard_normal((B, N, Hkv, d)))
        o, lse, _ = _run(lib, q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                         causal=causal, window_left=left, window_right=right)
        o = o.reshape(B, N, Hq, d)
        g = Hq // Hkv
        qt = q.to(torch.float64).transpose(1, 2)  # [B,H,N,d]
        kt = torch.repeat_interleave(k.to(torch.float64), g, dim=2).transpose(1, 2)
        vt = torch.repeat_interleave(v.to(torch.float64), g, dim=2).transpose(1, 2)
        mask = _band_mask(N, causal, left, right)
        ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
        ref = ref.transpose(1, 2).numpy()
        assert np.abs(o - ref).max() <= 1e-12, np.abs(o - ref).max()
        scores = (qt @ kt.transpose(-1, -2)) * scale
        ref_lse = torch.logsumexp(scores.masked_fill(~mask, float("-inf")), dim=-1).numpy()
        assert np.abs(lse - ref_lse).max() <= 1e-12


def pin_rows_mode_matches_full(lib):
    """The sampled-row entry (used at full workload sizes) equals the full run."""
    rng = np.random.default_rng(22)
    lens = [9, 30, 2]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 1, 16
    q = _bf16(rng.standard_normal((T, Hq, d)))
    k = _bf16(rng.standard_normal((T, Hkv, d)))
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    o, lse, nv = _run(lib, q, k, v, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=0.5, causal=True,
                      window_left=6, cu_seqlens=cu)
    rows = np.array([[1, 2, 17], [0, 0, 0], [2, 3, 1], [1, 1, 29]], dtype=np.int64)
    o2, lse2, nv2 = _run(lib, q, k, v, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=0.5, causal=True,
                         window_left=6, cu_seqlens=cu, rows=rows)
    for r, (b, h, i) in enumerate(rows):
        t = cu[b] + i
        assert np.array_equal(o2[r], o[t, h])
        assert lse2[r] == lse[h, t] and nv2[r] == nv[h, t]


# --------------------------------------------------------------------------
# key/value cache (decode) entry
# --------------------------------------------------------------------------
def _kvcache_inputs(rng, B, Hq, Hkv, Nq, d, lens, page_size, pages_per_seq, paged):
    """Random caches laid out in pages; returns q, kc, vc, block_table."""
    num_pages = B * pages_per_seq
    q = _bf16(rng.standard_normal((B, Nq, Hq, d)))
    kc = _bf16(rng.standard_normal((num_pages, page_size, Hkv, d)))
    vc = _bf16(rng.standard_normal((num_pages, page_size, Hkv, d)))
    bt = None
    if paged:
        bt = rng.permutation(num_pages).astype(np.int32).reshape(B, pages_per_seq)
    return q, kc, vc, bt


def _gather_cache(c, bt, b, L, page_size, pages_per_seq):
    """Logical [L, H, d] rows of sequence b from a paged cache (torch tensor)."""
    rows = []
    for j in range(L):
        page = bt[b, j // page_size] if bt is not None else b * pages_per_seq + j // page_size
        rows.append(c[int(page), j % page_size])
    return torch.stack(rows)


def pin_kvcache_matches_forward_last_rows(lib):
    """Decoding the newest tokens equals the last rows of full causal attention."""
    rng = np.random.default_rng(31)
    B, Hq, Hkv, d, page_size, pps = 2, 4, 2, 16, 8, 5
    lens = [37, 19]
    for Nq in (1, 3):
        q, kc, vc, _ = _kvcache_inputs(rng, B, Hq, Hkv, Nq, d, lens, page_size, pps, False)
        o, lse, _ = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc), lens,
                                        B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, page_size=page_size,
                                        pages_per_seq=pps, scale=0.4, causal=True, lib=lib)
        for b, L in enumerate(lens):
            kf = _gather_cache(kc, None, b, L, page_size, pps).unsqueeze(0).contiguous()
            vf = _gather_cache(vc, None, b, L, page_size, pps).unsqueeze(0).contiguous()
            qf = torch.zeros((1, L, Hq, d), dtype=torch.bfloat16)
            qf[0, L - Nq:] = q[b]
            of, lf, _ = _run(lib, qf, kf, vf, B=1, Hq=Hq, Hkv=Hkv, N=L, d=d, scale=0.4, causal=True)
            assert np.array_equal(o[b], of.reshape(L, Hq, d)[L - Nq:])
            assert np.array_equal(lse[b], lf[0][:, L - Nq:])


def pin_kvcache_paged_equals_contiguous(lib):
    rng = np.random.default_rng(32)
    B, Hq, Hkv, Nq, d, page_size, pps = 3, 4, 4, 2, 8, 4, 6
    lens = [24, 2, 13]
    q, kc, vc, bt = _kvcache_inputs(rng, B, Hq, Hkv, Nq, d, lens, page_size, pps, True)
    # contiguous copy of the same logical cache
    kcont = torch.zeros_like(kc)
    vcont = torch.zeros_like(vc)
    for b in range(B):
        for p_ in range(pps):
            kcont[b * pps + p_] = kc[int(bt[b, p_])]
            vcont[b * pps + p_] = vc[int(bt[b, p_])]
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, page_size=page_size, pages_per_seq=pps, scale=0.5,
              causal=True, window_left=7, lib=lib)
    o1, l1, _ = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc), lens,
                                    block_table=bt, **kw)
    o2, l2, _ = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kcont), W.bf16_bits(vcont), lens,
                                    **kw)
    assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def pin_kvcache_uniform_closed_form(lib):
    """Q = 0: O is the mean of V over the visible keys, aligned to the end of
    the cache; LSE = ln(count)."""
    rng = np.random.default_rng(33)
    B, Hq, Hkv, Nq, d, page_size, pps = 2, 2, 1, 3, 4, 4, 4
    lens = [11, 16]
    for causal, left, right in [(True, -1, -1), (True, 3, 0), (False, 2, 1), (False, -1, -1)]:
        q = torch.zeros((B, Nq, Hq, d), dtype=torch.bfloat16)
        kc = _bf16(rng.standard_normal((B * pps, page_size, Hkv, d)))
        vc = _bf16(rng.integers(-6, 7, size=(B * pps, page_size, Hkv, d)))
        o, lse, nv = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc), lens,
                                         B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, page_size=page_size,
                                         pages_per_seq=pps, scale=1.0, causal=causal,
                                         window_left=left, window_right=right, lib=lib)
        for b, L in enumerate(lens):
            vf = _gather_cache(vc, None, b, L, page_size, pps)[:, 0].to(torch.float64).numpy()
            for i in range(Nq):
                pos = L - Nq + i
                lo = 0 if left < 0 else max(0, pos - left)
                r_ = 0 if causal else right
                hi = L - 1 if r_ < 0 else min(L - 1, pos + r_)
                for h in range(Hq):
                    assert nv[b, h, i] == hi - lo + 1
                    assert np.allclose(o[b, i, h], vf[lo:hi + 1].mean(axis=0), rtol=0, atol=1e-13)
                    assert abs(lse[b, h, i] - math.log(hi - lo + 1)) <= 1e-13


def pin_kvcache_torch_sdpa(lib):
    import torch.nn.functional as F
    rng = np.random.default_rng(34)
    B, Hq, Hkv, Nq, d, page_size, pps = 2, 6, 2, 4, 32, 16, 4
    lens = [50, 37]
    q, kc, vc, bt = _kvcache_inputs(rng, B, Hq, Hkv, Nq, d, lens, page_size, pps, True)
    scale = d ** -0.5
    o, lse, _ = oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc), lens,
                                    B=B, Hq=Hq, Hkv=Hkv, Nq=Nq, d=d, page_size=page_size,
                                    pages_per_seq=pps, scale=scale, causal=True, window_left=20,
                                    block_table=bt, lib=lib)
    for b, L in enumerate(lens):
        kf = _gather_cache(kc, bt, b, L, page_size, pps).to(torch.float64)  # [L, Hkv, d]
        vf = _gather_cache(vc, bt, b, L, page_size, pps).to(torch.float64)
        g = Hq // Hkv
        kt = torch.repeat_interleave(kf, g, dim=1).transpose(0, 1)  # [Hq, L, d]
        vt = torch.repeat_interleave(vf, g, dim=1).transpose(0, 1)
        qt = q[b].to(torch.float64).transpose(0, 1)  # [Hq, Nq, d]
        # end-aligned causal band with a left window of 20, built from tril/triu
        full = _band_mask(L, True, 20, 0)  # [L, L] for queries at every position
        mask = full[L - Nq:]  # the newest Nq query positions
        ref = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
        assert np.abs(o[b] - ref.transpose(0, 1).numpy()).max() <= 1e-12
        sc = (qt @ kt.transpose(-1, -2)) * scale
        ref_lse = torch.logsumexp(sc.masked_fill(~mask, float("-inf")), dim=-1).numpy()
        assert np.abs(lse[b] - ref_lse).max() <= 1e-12


# --------------------------------------------------------------------------
# backward (gradients)
# --------------------------------------------------------------------------
def _bwd(lib, q, k, v, do, **kw):
    return oracle.attn_bwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), W.bf16_bits(do),
                           lib=lib, **kw)


def _np_forward_loss(qf, kf, vf, dof, scale, visible):
    """sum(dO * O) for one head, written out in numpy (fp64): the function
    whose gradient the oracle must return."""
    s = scale * qf @ kf.T
    s = np.where(visible, s, -np.inf)
    m = s.max(axis=1, keepdims=True)
    e = np.where(visible, np.exp(s - m), 0.0)
    o = (e / e.sum(axis=1, keepdims=True)) @ vf
    return float((dof * o).sum())


def pin_bwd_finite_differences(lib):
    """Central differences of sum(dO * O), computed by a numpy forward, match
    the oracle's gradients (independent of the oracle's formulas)."""
    rng = np.random.default_rng(40)
    for (N, d, causal, left, right, scale) in [(6, 4, True, -1, -1, 0.7),
                                               (7, 3, False, 2, 1, 0.9),
                                               (5, 4, False, -1, -1, 0.5)]:
        q = _bf16(rng.standard_normal((1, N, 1, d)))
        k = _bf16(rng.standard_normal((1, N, 1, d)))
        v = _bf16(rng.standard_normal((1, N, 1, d)))
        do = _bf16(rng.standard_normal((1, N, 1, d)))
        dq, dk, dv = _bwd(lib, q, k, v, do, B=1, Hq=1, Hkv=1, N=N, d=d, scale=scale,
                          causal=causal, window_left=left, window_right=right)
        vis = _band_mask(N, causal, left, right).numpy()
        base = [_f64(t).reshape(N, d) for t in (q, k, v, do)]
        eps = 1e-6
        for which, grad in ((0, dq), (1, dk), (2, dv)):
            g = grad.reshape(N, d)
            for i in range(N):
                for c in range(d):
                    plus = [a.copy() for a in base]
                    minus = [a.copy() for a in base]
                    plus[which][i, c] += eps
                    minus[which][i, c] -= eps
                    fd = (_np_forward_loss(*plus[:3], plus[3], scale, vis) -
                          _np_forward_loss(*minus[:3], minus[3], scale, vis)) / (2 * eps)
                    assert abs(fd - g[i, c]) <= 1e-6 * (1 + abs(fd)), (which, i, c, fd, g[i, c])


def pin_bwd_torch_autograd(lib):
    """torch autograd through float64 scaled_dot_product_attention with a band
    mask, grouped heads summed back onto their key/value head."""
    import torch.nn.functional as F
    rng = np.random.default_rng(41)
    cases = [
        # B, N, Hq, Hkv, d, causal, left, right, scale
        (2, 37, 4, 2, 16, True, -1, -1, 16 ** -0.5),
        (1, 29, 3, 3, 8, False, 5, 2, 0.4),
        (1, 41, 6, 1, 32, True, 9, 0, 32 ** -0.5),
    ]
    for (B, N, Hq, Hkv, d, causal, left, right, scale) in cases:
        q = _bf16(rng.standard_normal((B, N, Hq, d)))
        k = _bf16(rng.standard_normal((B, N, Hkv, d)))
        v = _bf16(rng.standard_normal((B, N, Hkv, d)))
        do = _bf16(rng.standard_normal((B, N, Hq, d)))
        dq, dk, dv = _bwd(lib, q, k, v, do, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                          causal=causal, window_left=left, window_right=right)
        g = Hq // Hkv
        qt = q.to(torch.float64).requires_grad_()
        kt = k.to(torch.float64).requires_grad_()
        vt = v.to(torch.float64).requires_grad_()
        kr = torch.repeat_interleave(kt, g, dim=2).transpose(1, 2)
        vr = torch.repeat_interleave(vt, g, dim=2).transpose(1, 2)
        o = F.scaled_dot_product_attention(qt.transpose(1, 2), kr, vr,
                                           attn_mask=_band_mask(N, causal, left, right),
                                           scale=scale).transpose(1, 2)
        (o * do.to(torch.float64)).sum().backward()
        for got, ref in ((dq, qt.grad), (dk, kt.grad), (dv, vt.grad)):
            ref = ref.numpy().reshape(got.shape)
            assert np.abs(got - ref).max() <= 1e-11 * (1 + np.abs(ref).max()), np.abs(got - ref).max()


def pin_bwd_invariants(lib):
    """Rows of dS sum to zero, so the key gradients of a sequence and head sum
    to zero; rows of P sum to one, so the value gradients sum to the output
    gradients of the rows that see any key."""
    rng = np.random.default_rng(42)
    lens = [13, 1, 22]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 8
    q = _bf16(rng.standard_normal((T, Hq, d)))
    k = _bf16(rng.standard_normal((T, Hkv, d)))
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    do = _bf16(rng.standard_normal((T, Hq, d)))
    for (causal, left, right) in [(True, -1, -1), (False, 3, 2), (True, 4, -1)]:
        dq, dk, dv = _bwd(lib, q, k, v, do, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=0.6,
                          causal=causal, window_left=left, window_right=right, cu_seqlens=cu)
        dof = _f64(do)
        for b in range(3):
            a, e = cu[b], cu[b + 1]
            for gh in range(Hkv):
                assert np.abs(dk[a:e, gh].sum(axis=0)).max() <= 1e-12
                heads = range(gh * (Hq // Hkv), (gh + 1) * (Hq // Hkv))
                want = sum(dof[a:e, h].sum(axis=0) for h in heads)
                assert np.abs(dv[a:e, gh].sum(axis=0) - want).max() <= 1e-12


def pin_bwd_packed_and_grouped(lib):
    """A packed batch equals separate calls per sequence, and grouped heads
    equal key/value heads repeated per query head with the gradients summed."""
    rng = np.random.default_rng(43)
    lens = [11, 4, 17]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 8
    q = _bf16(rng.standard_normal((T, Hq, d)))
    k = _bf16(rng.standard_normal((T, Hkv, d)))
    v = _bf16(rng.standard_normal((T, Hkv, d)))
    do = _bf16(rng.standard_normal((T, Hq, d)))
    kw = dict(scale=0.45, causal=True, window_left=5)
    dq, dk, dv = _bwd(lib, q, k, v, do, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, cu_seqlens=cu, **kw)
    for b, L in enumerate(lens):
        a = cu[b]
        sl = slice(a, a + L)
        r = _bwd(lib, q[sl].unsqueeze(0).contiguous(), k[sl].unsqueeze(0).contiguous(),
                 v[sl].unsqueeze(0).contiguous(), do[sl].unsqueeze(0).contiguous(), B=1, Hq=Hq,
                 Hkv=Hkv, N=L, d=d, **kw)
        for got, ref in zip((dq, dk, dv), r):
            assert np.array_equal(got[sl], ref)
    g = Hq // Hkv
    kr = torch.repeat_interleave(k, g, dim=1).contiguous()
    vr = torch.repeat_interleave(v, g, dim=1).contiguous()
    dq2, dk2, dv2 = _bwd(lib, q, kr, vr, do, B=3, Hq=Hq, Hkv=Hq, N=T, d=d, cu_seqlens=cu, **kw)
    assert np.abs(dq - dq2).max() <= 1e-12
    assert np.abs(dk - dk2.reshape(T, Hkv, g, d).sum(axis=2)).max() <= 1e-12
    assert np.abs(dv - dv2.reshape(T, Hkv, g, d).sum(axis=2)).max() <= 1e-12


# --------------------------------------------------------------------------
# e4m3 inputs
# --------------------------------------------------------------------------
def _e4m3_value(code: int) -> float:
    """E4M3FN from its definition: sign, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent 0 is subnormal (2^-6 * m/8); S.1111.111 is NaN (no inf)."""
    s = -1.0 if code & 0x80 else 1.0
    e = (code >> 3) & 0xF
    m = code & 0x7
    if e == 0xF and m == 0x7:
        return float("nan")
    if e == 0:
        return s * (m / 8.0) * 2.0 ** -6
    return s * (1.0 + m / 8.0) * 2.0 ** (e - 7)


def pin_e4m3_widening(lib):
    """The e4m3 -> bf16 widening that feeds the oracle is exact for all 256
    codes (checked against the format's definition)."""
    codes = torch.arange(256, dtype=torch.uint8)
    widened = W.e4m3_as_bf16(codes.view(torch.float8_e4m3fn)).to(torch.float64).numpy()
    for c in range(256):
        want = _e4m3_value(c)
        if math.isnan(want):
            assert math.isnan(widened[c])
        else:
            assert widened[c] == want, (c, widened[c], want)


ALL_PINS = [
    pin_worked_example,
    pin_uniform_scores,
    pin_uniform_scores_packed,
    pin_two_keys,
    pin_hard_limit,
    pin_single_key_and_row0,
    pin_constant_v_and_row_sums,
    pin_key_permutation,
    pin_window_equals_causal,
    pin_packed_equals_separate,
    pin_gqa_equals_repeated,
    pin_torch_sdpa,
    pin_rows_mode_matches_full,
    pin_kvcache_matches_forward_last_rows,
    pin_kvcache_paged_equals_contiguous,
    pin_kvcache_uniform_closed_form,
    pin_kvcache_torch_sdpa,
    pin_bwd_finite_differences,
    pin_bwd_torch_autograd,
    pin_bwd_invariants,
    pin_bwd_packed_and_grouped,
    pin_e4m3_widening,
]
