"""GPU parity of attn_decode (newest tokens against a paged key/value cache)
with the fp64 oracle's key/value-cache entry, through the C ABI.

Covers: single slice and split-and-merge, ragged cache lengths (including
L == Nq and a full cache), page sizes that are not multiples of the key tile,
contiguous and paged caches, MHA / GQA / MQA, ragged head chunks, Nq up to 16,
causal and sliding-window masks, the mask pattern bit-exact, determinism, and
sampled sequences of the full-size decode benchmark."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import oracle
import workloads as W
from gpu_helpers import TOL_LSE, TOL_O

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda:0")


def run_gpu(w: W.DecodeWorkload, q, kc, vc, seqlens, table, num_splits, *, q_dev=None):
    """Inputs on the CPU (or already on the device) -> (o, lse) on the CPU."""
    qd = q_dev if q_dev is not None else q.to(DEV)
    kd, vd = kc.to(DEV), vc.to(DEV)
    sd = seqlens.to(DEV)
    td = table.to(DEV) if table is not None else None
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((w.B, w.Hq, w.Nq), float("nan"), dtype=torch.float32, device=DEV)
    nbytes = ea.attn_decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                                            w.pages_per_seq, num_splits)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=DEV)
    ea.attn_decode(qd, kd, vd, o, lse, sd, td, w.B, w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                   w.pages_per_seq, kd.shape[0], w.scale, w.causal, w.window_left,
                   w.window_right, num_splits, ws if nbytes else None, nbytes)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return o.cpu(), lse.cpu()


def run_oracle(w: W.DecodeWorkload, q, kc, vc, seqlens, table):
    return oracle.attn_kvcache(W.bf16_bits(q), W.bf16_bits(kc), W.bf16_bits(vc),
                               seqlens.numpy(), B=w.B, Hq=w.Hq, Hkv=w.Hkv, Nq=w.Nq, d=w.d,
                               page_size=w.page_size, pages_per_seq=w.pages_per_seq,
                               scale=w.scale, causal=w.causal, window_left=w.window_left,
                               window_right=w.window_right,
                               block_table=None if table is None else table.numpy())


def compare(o, lse, o_ref, lse_ref):
    og = o.to(torch.float64).numpy()
    lg = lse.to(torch.float64).numpy()
    assert np.isfinite(og).all() and np.isfinite(lg).all()
    dO = float(np.abs(og - o_ref).max())
    dL = float(np.abs(lg - lse_ref).max())
    assert dO <= TOL_O, f"max|dO| = {dO}"
    assert dL <= TOL_LSE, f"max|dLSE| = {dL}"
    return dO, dL


def case(name, B, Hq, Hkv, Nq, d, page_size, pps, lengths, paged=True, causal=True, left=-1,
         right=-1, seed=11):
    return W.DecodeWorkload(name, B, Hq, Hkv, Nq, d, page_size, pps, list(lengths), paged,
                            causal, left, right, seed)


CASES = [
    # name, B, Hq, Hkv, Nq, d, page, pages/seq, lengths
    case("gqa4_nq1_d128", 3, 8, 2, 1, 128, 16, 40, [1, 333, 640]),
    case("gqa4_nq4_d128_rows16", 2, 16, 4, 4, 128, 64, 20, [4, 1200]),
    case("gqa8_nq3_chunks", 2, 16, 2, 3, 128, 32, 30, [517, 960]),     # 5 + 3 heads per chunk
    case("mqa_nq1_d128", 2, 16, 1, 1, 128, 64, 33, [2112, 700]),       # 16 rows per CTA
    case("mha_nq2_d128", 2, 4, 4, 2, 128, 16, 12, [2, 191]),
    case("nq16_mha_d128", 2, 2, 2, 16, 128, 128, 4, [16, 500]),
    case("gqa4_nq1_d64", 3, 8, 2, 1, 64, 16, 40, [64, 65, 639]),
    case("gqa8_nq2_d64", 2, 32, 4, 2, 64, 64, 10, [100, 640]),
    case("odd_page7_d128", 2, 8, 2, 2, 128, 7, 50, [349, 350]),       # gather kernel
    case("page100_d64", 2, 8, 2, 1, 64, 100, 6, [599, 301]),          # gather kernel
    case("page1_d128", 2, 4, 2, 2, 128, 1, 150, [150, 77]),            # gather kernel
    case("page24_d128", 2, 8, 2, 2, 128, 24, 30, [700, 31]),          # 8-key TMA copies
    case("page256_d128", 2, 8, 1, 1, 128, 256, 3, [700, 256]),        # 64-key copies
    case("contiguous_d128", 3, 8, 2, 2, 128, 64, 8, [2, 300, 512], paged=False),
    case("window_causal_d128", 2, 8, 2, 4, 128, 32, 20, [640, 200], left=100),
    case("window_noncausal_d64", 2, 8, 2, 4, 64, 32, 20, [640, 37], causal=False, left=50,
         right=-1),
    case("noncausal_d128", 2, 8, 4, 3, 128, 16, 16, [256, 3], causal=False),
    case("window0_d128", 2, 4, 1, 3, 128, 16, 16, [256, 30], left=0),  # each row sees itself
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
@pytest.mark.parametrize("splits", [1, 3, 8])
def test_decode_parity(w, splits):
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    o_ref, lse_ref, _ = run_oracle(w, q, kc, vc, seqlens, table)
    o, lse = run_gpu(w, q, kc, vc, seqlens, table, splits)
    compare(o, lse, o_ref, lse_ref)


def test_split_count_beyond_tiles_is_clamped():
    w = case("tiny", 2, 8, 2, 1, 128, 16, 4, [10, 64])
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    o_ref, lse_ref, _ = run_oracle(w, q, kc, vc, seqlens, table)
    # 64-key slices: at most one slice here, whatever is asked for
    assert ea.attn_decode_workspace_bytes(2, 8, 2, 1, 128, 16, 4, 1000) == 0
    o, lse = run_gpu(w, q, kc, vc, seqlens, table, 1000)
    compare(o, lse, o_ref, lse_ref)


def test_paged_equals_contiguous_bit_exact():
    """The same logical cache read through a permuted page table or in place
    gives identical bits (same values, same arithmetic order)."""
    w = case("paged", 3, 16, 4, 2, 128, 32, 12, [384, 17, 200], paged=True)
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    # contiguous copy: logical page p of sequence b at b * pps + p
    order = table.reshape(-1).long()
    kcont, vcont = kc[order].contiguous(), vc[order].contiguous()
    wc = case("contig", 3, 16, 4, 2, 128, 32, 12, [384, 17, 200], paged=False)
    for splits in (1, 4):
        o1, l1 = run_gpu(w, q, kc, vc, seqlens, table, splits)
        o2, l2 = run_gpu(wc, q, kcont, vcont, seqlens, None, splits)
        assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
        assert torch.equal(l1, l2)


def test_split_counts_agree():
    w = case("splits", 2, 32, 8, 1, 128, 64, 64, [4096, 3000])
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    o_ref, lse_ref, _ = run_oracle(w, q, kc, vc, seqlens, table)
    outs = [run_gpu(w, q, kc, vc, seqlens, table, s) for s in (1, 2, 5, 16, 64)]
    for o, lse in outs:
        compare(o, lse, o_ref, lse_ref)
    base = outs[0][0].float()
    for o, _ in outs[1:]:
        assert float((o.float() - base).abs().max()) <= 2 * TOL_O


@pytest.mark.parametrize("left,causal,right", [(-1, True, -1), (37, True, -1), (0, True, -1),
                                               (200, False, -1), (5, False, 3)])
def test_mask_pattern_bit_exact(left, causal, right):
    """Q = 0 makes every visible score 0, so exp(LSE) is the number of visible
    keys, which must equal the oracle's count for every row."""
    w = case("mask", 2, 4, 2, 5, 128, 16, 30, [470, 5], causal=causal, left=left, right=right)
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    q.zero_()
    _, _, nvis = run_oracle(w, q, kc, vc, seqlens, table)
    for splits in (1, 6):
        _, lse = run_gpu(w, q, kc, vc, seqlens, table, splits)
        count = np.rint(np.exp(lse.to(torch.float64).numpy()))
        assert np.array_equal(count.astype(np.int64), nvis)


def test_deterministic():
    w = case("det", 2, 16, 4, 2, 128, 64, 16, [1000, 777])
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    a = run_gpu(w, q, kc, vc, seqlens, table, 4)
    b = run_gpu(w, q, kc, vc, seqlens, table, 4)
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16))
    assert torch.equal(a[1], b[1])


def test_benchmark_workload_sampled():
    """The full decode benchmark (64 x 8192-token caches, paged) in the launch
    configuration the benchmark uses; the oracle checks 6 sequences."""
    w = W.decode_workload()
    q, kc, vc, seqlens, table = W.decode_inputs(w, device="cuda")
    splits = ea.attn_decode_default_splits(w.B, w.Hq, w.Hkv, w.Nq, w.max_len)
    o, lse = run_gpu(w, q.cpu(), kc, vc, seqlens, table, splits, q_dev=q)
    pick = [0, 1, 17, 40, 62, 63]
    sub = W.DecodeWorkload("sub", len(pick), w.Hq, w.Hkv, w.Nq, w.d, w.page_size,
                           w.pages_per_seq, [w.lengths[b] for b in pick], w.paged, w.causal,
                           w.window_left, w.window_right, w.seed)
    qc, kcc, vcc = q.cpu(), kc.cpu(), vc.cpu()
    o_ref, lse_ref, _ = run_oracle(sub, qc[pick], kcc, vcc, seqlens[pick], table[pick])
    compare(o[pick], lse[pick], o_ref, lse_ref)


@pytest.mark.parametrize("page_size", [32, 7])
def test_invalid_page_is_reported_not_followed(page_size):
    """A page-table entry outside [0, num_pages) is neither read nor followed:
    the call completes and attn_device_status reports ATTN_ERR_PAGE once."""
    w = case("badpage", 2, 8, 2, 1, 128, page_size, 10, [5 * page_size, 2 * page_size])
    q, kc, vc, seqlens, table = W.decode_inputs(w)
    bad = table.clone()
    bad[0, 1] = kc.shape[0] + 5
    bad[1, 0] = -3
    qd, kd, vd = q.to(DEV), kc.to(DEV), vc.to(DEV)
    o = torch.empty_like(qd)
    lse = torch.empty((w.B, w.Hq, w.Nq), dtype=torch.float32, device=DEV)
    ea.attn_decode(qd, kd, vd, o, lse, seqlens.to(DEV), bad.to(DEV), w.B, w.Hq, w.Hkv, w.Nq, w.d,
                   w.page_size, w.pages_per_seq, kd.shape[0], w.scale, True, -1, -1, 1)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_PAGE
    assert ea.attn_device_status() == ea.ATTN_OK  # read clears it
    # the context still works: a valid call afterwards matches the oracle
    o_ref, lse_ref, _ = run_oracle(w, q, kc, vc, seqlens, table)
    compare(*run_gpu(w, q, kc, vc, seqlens, table, 2), o_ref, lse_ref)
