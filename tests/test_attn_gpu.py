"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Small cases are compared element by element against a full oracle run; the
five named workloads are compared on sampled rows at full size, in the launch
configuration the benchmark times.  The visible-key pattern is checked
bit-exactly with a probe input (Q = 0 makes every visible weight equal, so
exp(LSE) is the integer number of visible keys and O counts residues of the
visible key indices)."""
import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import workloads as W
from gpu_helpers import (TOL_LSE, TOL_O, compare_full, default_scale, gpu_run, lse_index, o_index,
                         oracle_run, sample_rows, visible_counts)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_attention_142_b200 import build
    build.build()
    ea.load_library()


# (name, B, Hq, Hkv, N, d, causal, left, right, seed)
DENSE_CASES = [
    ("cfg1_noncausal_d64", 1, 2, 2, 256, 64, False, -1, -1, 0),
    ("mha_causal_ragged", 2, 4, 4, 300, 128, True, -1, -1, 5),
    ("gqa4_causal_ragged", 1, 8, 2, 520, 128, True, -1, -1, 6),
    ("gqa3_rowpairs", 2, 6, 2, 333, 64, True, -1, -1, 7),
    ("mqa_noncausal", 1, 4, 1, 257, 128, False, -1, -1, 8),
    ("swa_causal", 1, 2, 2, 700, 128, True, 100, 0, 9),
    ("window_both_sides", 1, 2, 2, 600, 64, False, 50, 70, 10),
    ("window_right_only", 1, 4, 2, 400, 128, False, -1, 5, 11),
    ("window_zero", 1, 2, 1, 300, 128, False, 0, 0, 12),
    ("window_left_huge", 1, 2, 2, 260, 128, False, 1 << 30, 3, 13),
    ("n1", 3, 2, 2, 1, 128, True, -1, -1, 14),
    ("n127", 1, 2, 2, 127, 64, True, -1, -1, 15),
    ("n128", 1, 4, 4, 128, 128, False, -1, -1, 16),
    ("n129", 1, 4, 2, 129, 128, True, -1, -1, 17),
    ("many_blocks", 1, 2, 2, 1100, 128, True, -1, -1, 18),
    ("large_scores", 1, 2, 2, 384, 128, False, -1, -1, 19),
]


@pytest.mark.parametrize("case", DENSE_CASES, ids=lambda c: c[0])
def test_dense_parity(case):
    name, B, Hq, Hkv, N, d, causal, left, right, seed = case
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed)
    if name == "large_scores":
        q = (q.float() * 4).to(torch.bfloat16)  # score spread of ~ +-50: exercises rescaling
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=causal,
              window_left=left, window_right=right)
    o, lse = gpu_run(q, k, v, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)


PACKED_CASES = [
    # (name, lengths, Hq, Hkv, d, causal, left, right, seed)
    ("packed_causal_gqa", [1, 0, 5, 128, 129, 300, 77], 4, 2, 128, True, -1, -1, 21),
    ("packed_noncausal", [200, 3, 0, 0, 256, 131], 2, 2, 64, False, -1, -1, 22),
    ("packed_window", [400, 129, 1, 600], 4, 1, 128, True, 64, 0, 23),
    ("packed_single", [513], 2, 2, 128, True, -1, -1, 24),
]


@pytest.mark.parametrize("case", PACKED_CASES, ids=lambda c: c[0])
def test_packed_parity(case):
    name, lengths, Hq, Hkv, d, causal, left, right, seed = case
    cu = W.cumulative(lengths)
    T = cu[-1]
    q, k, v = W.draw_qkv((T, Hq, d), (T, Hkv, d), seed)
    kw = dict(B=len(lengths), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=default_scale(d), causal=causal,
              window_left=left, window_right=right, cu_seqlens=cu)
    o, lse = gpu_run(q, k, v, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_workload_sampled_rows(cfg):
    """Full-size workloads in the benchmark's launch configuration; the oracle
    computes sampled rows one by one."""
    w = W.workload(cfg)
    q, k, v = W.inputs(w)
    kw = dict(B=w.B, Hq=w.Hq, Hkv=w.Hkv, N=w.N, d=w.d, scale=w.scale, causal=w.causal,
              window_left=w.window_left, window_right=w.window_right, cu_seqlens=w.cu_seqlens)
    o, lse = gpu_run(q, k, v, max_seqlen=w.max_seqlen, **kw)
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    rows = sample_rows(lengths, w.Hq, n_random=600, seed=100 + cfg)
    o_ref, lse_ref, _ = oracle_run(q, k, v, rows=rows, **kw)
    of = o.reshape(-1, w.Hq, w.d)
    lf = lse.reshape(-1)
    got_o = np.stack([of[o_index(w.cu_seqlens, b, i, w.N), h].to(torch.float64).numpy()
                      for b, h, i in rows])
    got_l = np.array([float(lf[lse_index(w.cu_seqlens, b, h, i, w.Hq, w.N)]) for b, h, i in rows])
    dO = np.abs(got_o - o_ref).max()
    dL = np.abs(got_l - lse_ref).max()
    assert dO <= TOL_O, dO
    assert dL <= TOL_LSE, dL
    # every row was written, and nothing is NaN/inf
    assert torch.isfinite(o.float()).all()
    assert torch.isfinite(lse).all()


def _mask_probe(lengths, Hq, Hkv, d, causal, left, right, packed):
    """Q = 0 and V[t, c] = [t mod d == c]: every visible weight is equal, so
    exp(LSE) is the number of visible keys and O[i, c] is the fraction of
    visible keys whose index is c modulo d."""
    B = len(lengths)
    if packed:
        cu = W.cumulative(lengths)
        T = cu[-1]
        shape_q, shape_kv = (T, Hq, d), (T, Hkv, d)
        N = T
    else:
        cu = None
        N = lengths[0]
        T = B * N
        shape_q, shape_kv = (B, N, Hq, d), (B, N, Hkv, d)
    g = torch.Generator().manual_seed(77)
    q = torch.zeros(shape_q, dtype=torch.bfloat16)
    k = torch.randn(shape_kv, generator=g).to(torch.bfloat16)
    t = torch.arange(T).reshape(-1, 1) % d
    onehot = (t == torch.arange(d).reshape(1, -1)).to(torch.bfloat16)  # [T, d]
    v = onehot.reshape(T, 1, d).expand(T, Hkv, d).reshape(shape_kv).contiguous()
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=causal,
              window_left=left, window_right=right, cu_seqlens=cu)
    o, lse = gpu_run(q, k, v, **kw)
    # 1) exact visible-key counts for every row, from exp(LSE)
    counts = visible_counts(lengths, causal, left, right)
    lse_np = lse.to(torch.float64).numpy()
    for b, L in enumerate(lengths):
        for h in range(Hq):
            if L == 0:
                continue
            if packed:
                row_lse = lse_np[h, cu[b]:cu[b] + L]
            else:
                row_lse = lse_np[b, h, :L]
            got = np.rint(np.exp(row_lse)).astype(np.int64)
            bad = np.nonzero(got != counts[b])[0]
            assert bad.size == 0, f"seq {b} head {h}: rows {bad[:8]} count {got[bad[:8]]} != {counts[b][bad[:8]]}"
    # 2) which keys: O equals the oracle's residue fractions on sampled rows
    rows = sample_rows(lengths, Hq, n_random=300, seed=5)
    o_ref, _, nvis = oracle_run(q, k, v, rows=rows, **kw)
    of = o.reshape(-1, Hq, d)
    for r, (b, h, i) in enumerate(rows):
        got = of[o_index(cu, b, i, N), h].to(torch.float64).numpy()
        # exact value count/n rounded once to bf16; allow one bf16 ulp
        ref = o_ref[r]
        ulp = np.where(ref > 0, 2.0 ** (np.floor(np.log2(np.maximum(ref, 1e-30))) - 7), 0.0)
        assert np.all(np.abs(got - ref) <= ulp + 1e-12), (b, h, i)


@pytest.mark.parametrize("probe", [
    ("causal_dense", [1000, 1000], 2, 2, 128, True, -1, -1, False),
    ("window_dense", [1500], 4, 2, 128, True, 300, 0, False),
    ("window_two_sided_d64", [900], 2, 1, 64, False, 129, 40, False),
    ("noncausal_dense", [700, 700], 2, 2, 64, False, -1, -1, False),
    ("packed_causal", [5, 0, 130, 1, 513, 255], 4, 2, 128, True, -1, -1, True),
    ("packed_window", [600, 129, 2], 2, 2, 128, True, 127, 0, True),
], ids=lambda p: p[0])
def test_mask_pattern_bit_exact(probe):
    _, lengths, Hq, Hkv, d, causal, left, right, packed = probe
    _mask_probe(lengths, Hq, Hkv, d, causal, left, right, packed)


@pytest.mark.parametrize("cfg", [2, 3, 4, 5])
def test_mask_pattern_workloads(cfg):
    """The same probe at the named workloads' full shapes and masks."""
    w = W.workload(cfg)
    lengths = ([b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])] if w.packed
               else [w.N] * w.B)
    Hq = min(w.Hq, 8)
    Hkv = max(1, Hq * w.Hkv // w.Hq)
    _mask_probe(lengths, Hq, Hkv, w.d, w.causal, w.window_left, w.window_right, w.packed)


def test_causal_row0_is_v0_exactly():
    B, N, H, d = 2, 300, 4, 128
    q, k, v = W.draw_qkv((B, N, H, d), (B, N, H, d), 31)
    o, _ = gpu_run(q, k, v, B=B, Hq=H, Hkv=H, N=N, d=d, scale=default_scale(d), causal=True)
    assert torch.equal(o[:, 0], v[:, 0])


def test_deterministic():
    B, N, Hq, Hkv, d = 1, 777, 8, 2, 128
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), 32)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=True)
    o1, l1 = gpu_run(q, k, v, **kw)
    o2, l2 = gpu_run(q, k, v, **kw)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_host_entry_matches_device_entry():
    lengths = [300, 1, 129]
    cu = W.cumulative(lengths)
    T, Hq, Hkv, d = cu[-1], 4, 2, 128
    q, k, v = W.draw_qkv((T, Hq, d), (T, Hkv, d), 33)
    kw = dict(B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=default_scale(d), causal=True,
              window_left=-1, window_right=-1, cu_seqlens=cu)
    o_dev, l_dev = gpu_run(q, k, v, **kw)
    qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
    oh = torch.empty_like(qh).pin_memory()
    lh = torch.empty((Hq, T), dtype=torch.float32).pin_memory()
    cuh = torch.tensor(cu, dtype=torch.int32)
    nbytes = ea.attn_fwd_host_workspace_bytes(3, Hq, Hkv, T, d, True)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    ea.attn_fwd_host(qh, kh, vh, oh, lh, 3, Hq, Hkv, T, d, default_scale(d), True, -1, -1, cuh,
                     0, ws, nbytes)
    torch.cuda.synchronize()
    assert torch.equal(oh, o_dev) and torch.equal(lh, l_dev)


def test_bounded_wait_reports_timeout_and_recovers():
    assert ea.attn_device_status() == ea.ATTN_OK
    assert ea.attn_selftest_bounded_wait(2_000_000) == ea.ATTN_OK  # 2 ms limit
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_DEVICE_TIMEOUT
    assert ea.attn_device_status() == ea.ATTN_OK  # read clears it
    # the context is healthy: a normal call still matches the oracle
    B, N, H, d = 1, 200, 2, 64
    q, k, v = W.draw_qkv((B, N, H, d), (B, N, H, d), 34)
    kw = dict(B=B, Hq=H, Hkv=H, N=N, d=d, scale=default_scale(d), causal=True)
    o, lse = gpu_run(q, k, v, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)


def test_empty_inputs_enqueue_nothing():
    z = torch.empty(0, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(0, dtype=torch.float32, device="cuda")
    assert ea.attn_fwd(z, z, z, z, lse, 2, 4, 2, 0, 128, 0.1, True) == ea.ATTN_OK
    cu = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert ea.attn_fwd(z, z, z, z, lse, 3, 4, 2, 0, 128, 0.1, True, cu_seqlens=cu,
                       max_seqlen=0) == ea.ATTN_OK
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK


def test_wrong_device_arch_is_not_silently_used():
    major, minor = torch.cuda.get_device_capability()
    assert (major, minor) == (10, 0), "these kernels are built for sm_100a only"


# The persistent schedule: one CTA per SM takes over the tile pairs of CTAs that
# have not started, so most CTAs compute many pairs in a row; per-pair state
# (running maximum and sums, barrier phases, the O hand-over between a pair's
# epilogue and the next pair's first P V) must not leak between pairs.  Pairs
# past a packed sequence's end are skipped by the producer.
SCHEDULE_CASES = [
    # (name, B, Hq, Hkv, N, d, causal, left, right, seed): a few hundred pairs each
    ("heads_paired_causal", 32, 8, 2, 300, 128, True, -1, -1, 31),
    ("rows_paired_noncausal_d64", 24, 6, 6, 520, 64, False, -1, -1, 32),
    ("heads_paired_window_d64", 16, 8, 4, 700, 64, True, 90, 0, 33),
]


@pytest.mark.parametrize("case", SCHEDULE_CASES, ids=lambda c: c[0])
def test_schedule_many_pairs_per_cta(case):
    name, B, Hq, Hkv, N, d, causal, left, right, seed = case
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=causal,
              window_left=left, window_right=right)
    o, lse = gpu_run(q, k, v, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)


@pytest.mark.parametrize("d", [128, 64])
def test_schedule_mostly_empty_packed(d):
    """Most tile pairs lie past their sequence's end (many empty and one-token
    sequences beside a long one); every row is still computed, once."""
    lengths = [0] * 40 + [1] * 20 + [700] + [0] * 30 + [129, 2, 0, 255]
    cu = W.cumulative(lengths)
    T, Hq, Hkv = cu[-1], 4, 2
    q, k, v = W.draw_qkv((T, Hq, d), (T, Hkv, d), 40 + d)
    kw = dict(B=len(lengths), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=default_scale(d), causal=True,
              cu_seqlens=cu)
    o, lse = gpu_run(q, k, v, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)


def test_schedule_accumulate_many_pairs():
    """The accumulating epilogue under the persistent schedule: one call into an
    empty accumulator (O = 0, LSE = -inf) gives the attention output itself."""
    B, Hq, Hkv, N, d = 24, 8, 2, 384, 128
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), 34)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o_acc = torch.zeros((B, N, Hq, d), dtype=torch.float32, device=dev)
    l_acc = torch.full((B, Hq, N), float("-inf"), dtype=torch.float32, device=dev)
    scale = default_scale(d)
    assert ea.attn_fwd_accumulate(qd, kd, vd, o_acc, l_acc, B, Hq, Hkv, N, d, scale,
                                  True) == ea.ATTN_OK
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o_ref, lse_ref, _ = oracle_run(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                                   causal=True)
    # fp32 output: only the weights' bf16 rounding remains (no output rounding)
    assert float(np.abs(o_acc.cpu().double().numpy() - o_ref.reshape(B, N, Hq, d)).max()) <= 5e-3
    assert float(np.abs(l_acc.cpu().double().numpy() - lse_ref.reshape(B, Hq, N)).max()) <= TOL_LSE


def test_long_sequence_sampled_rows():
    """A 131 072-token causal sequence (GQA 8:1): offsets past 2^31 bytes in O and
    the deepest key ranges, checked on sampled rows."""
    B, Hq, Hkv, N, d = 1, 8, 1, 131072, 128
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), 51)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=True)
    o, lse = gpu_run(q, k, v, **kw)
    rows = sample_rows([N], Hq, n_random=120, seed=52)
    rows = np.concatenate([rows, np.array([[0, Hq - 1, N - 1], [0, 0, N - 129], [0, 3, N // 2 + 127]])])
    o_ref, lse_ref, _ = oracle_run(q, k, v, rows=rows, **kw)
    of = o.reshape(-1, Hq, d)
    lf = lse.reshape(-1)
    got_o = np.stack([of[i, h].to(torch.float64).numpy() for b, h, i in rows])
    got_l = np.array([float(lf[(b * Hq + h) * N + i]) for b, h, i in rows])
    assert np.abs(got_o - o_ref).max() <= TOL_O
    assert np.abs(got_l - lse_ref).max() <= TOL_LSE
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_attention_convenience_dense_and_packed():
    """ea.attention allocates the outputs; packed batches without max_seqlen."""
    d, Hq, Hkv = 128, 4, 2
    q, k, v = W.draw_qkv((2, 200, Hq, d), (2, 200, Hkv, d), 61)
    o, lse = ea.attention(q.cuda(), k.cuda(), v.cuda(), causal=True)
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = oracle_run(q, k, v, B=2, Hq=Hq, Hkv=Hkv, N=200, d=d, scale=default_scale(d),
                                   causal=True)
    compare_full(o.cpu(), lse.cpu(), o_ref, lse_ref)
    lengths = [5, 0, 300, 130]
    cu = W.cumulative(lengths)
    T = cu[-1]
    q, k, v = W.draw_qkv((T, Hq, d), (T, Hkv, d), 62)
    o, lse = ea.attention(q.cuda(), k.cuda(), v.cuda(), causal=True,
                          cu_seqlens=torch.tensor(cu, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    o_ref, lse_ref, _ = oracle_run(q, k, v, B=len(lengths), Hq=Hq, Hkv=Hkv, N=T, d=d,
                                   scale=default_scale(d), causal=True, cu_seqlens=cu)
    compare_full(o.cpu(), lse.cpu(), o_ref, lse_ref)


# A key that the mask hides must weigh exactly 0 ("FlashAttention" explainer
# page, "Checking correctness": the reference fills masked scores with -inf).
# The same call runs twice, once with V = 1e37 (finite in bf16) on chosen keys:
# every row that sees none of them must come out bit-identical, which fails if a
# hidden key kept any weight at all (a weight of 2^-125 would add ~0.2 to O).
# The chosen keys sit in the columns 28-31 of every 32 of a key block, where the
# kernels take some exponentials from the FMA pipe, and past the end of a packed
# sequence.  The run with ordinary values is also checked against the oracle.
HUGE_V = 1e37


def _huge_masked_probe(lengths, Hq, Hkv, d, causal, left, right, packed, huge, seed):
    B = len(lengths)
    if packed:
        cu = W.cumulative(lengths)
        N = T = cu[-1]
        shape_q, shape_kv = (T, Hq, d), (T, Hkv, d)
        tok = lambda b, j: cu[b] + j  # noqa: E731
    else:
        cu = None
        N = lengths[0]
        T = B * N
        shape_q, shape_kv = (B, N, Hq, d), (B, N, Hkv, d)
        tok = lambda b, j: b * N + j  # noqa: E731
    q, k, v = W.draw_qkv(shape_q, shape_kv, seed)
    vf = v.reshape(T, Hkv, d).clone()
    hidden = {b: np.array([j for j in range(L) if huge(b, j)], dtype=np.int64)
              for b, L in enumerate(lengths)}
    for b, js in hidden.items():
        for j in js:
            vf[tok(b, int(j))] = HUGE_V
    v_huge = vf.reshape(shape_kv).contiguous()
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=default_scale(d), causal=causal,
              window_left=left, window_right=right, cu_seqlens=cu)
    o, lse = gpu_run(q, k, v, **kw)
    o_h, lse_h = gpu_run(q, k, v_huge, **kw)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    compare_full(o, lse, o_ref, lse_ref)
    r = 0 if causal else right
    rows, sensitive = [], 0
    for b, L in enumerate(lengths):
        js = hidden[b]
        for i in range(L):
            lo = 0 if left < 0 else max(0, i - left)
            hi = L - 1 if r < 0 else min(L - 1, i + r)
            if np.any((js >= lo) & (js <= hi)):
                continue  # this row sees a huge value
            # the key blocks the row's tile reads (128-key blocks from the
            # sequence start) hold a hidden huge key, or the next sequence does
            blk_lo, blk_hi = lo // 128 * 128, (hi // 128 + 1) * 128
            if np.any((js >= blk_lo) & (js < blk_hi)) or (packed and blk_hi > L and b + 1 < B and
                                                           hidden[b + 1].size):
                sensitive += 1
            rows.append(o_index(cu, b, i, N))
            for h in range(Hq):
                idx = lse_index(cu, b, h, i, Hq, N)
                assert lse_h.reshape(-1)[idx] == lse.reshape(-1)[idx], (b, h, i)
    assert sensitive > 0
    rows = torch.tensor(rows)
    of, ohf = o.reshape(-1, Hq, d), o_h.reshape(-1, Hq, d)
    assert torch.equal(ohf[rows], of[rows])


@pytest.mark.parametrize("probe", [
    # name, lengths, Hq, Hkv, d, causal, left, right, packed, huge(b, j)
    ("causal_diagonal_block", [384, 384], 2, 2, 128, True, -1, -1, False,
     lambda b, j: j % 128 >= 92 and j % 32 >= 28),
    ("window_left_causal", [700], 4, 2, 128, True, 16, 0, False, lambda b, j: j % 32 >= 28),
    ("window_two_sided_d64", [600], 2, 1, 64, False, 8, 8, False, lambda b, j: j % 32 >= 28),
    ("packed_neighbour_noncausal", [200, 300, 150], 2, 2, 128, False, -1, -1, True,
     lambda b, j: b == 1),
    ("packed_neighbour_causal_gqa", [200, 300, 150], 4, 2, 128, True, -1, -1, True,
     lambda b, j: b == 1),
], ids=lambda p: p[0])
def test_masked_keys_weigh_exactly_zero(probe):
    _, lengths, Hq, Hkv, d, causal, left, right, packed, huge = probe
    _huge_masked_probe(lengths, Hq, Hkv, d, causal, left, right, packed, huge, seed=71)


def test_packed_max_seqlen_too_small_is_reported():
    """A sequence longer than max_seqlen (rounded up to 128 rows) does not fit
    the launch: it is skipped -- its rows are left as they were -- and the
    status word reports it; the other sequences are computed, and the next call
    is clean.  Every address stays inside the tensors."""
    lengths = [300, 129, 50]
    cu = W.cumulative(lengths)
    T, Hq, Hkv, d = cu[-1], 4, 2, 128
    q, k, v = W.draw_qkv((T, Hq, d), (T, Hkv, d), 72)
    dev = torch.device("cuda:0")
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    cud = torch.tensor(cu, dtype=torch.int32, device=dev)
    o = torch.full_like(qd, float("nan"))
    lse = torch.full((Hq, T), float("nan"), dtype=torch.float32, device=dev)
    assert ea.attn_device_status() == ea.ATTN_OK
    ea.attn_fwd(qd, kd, vd, o, lse, 3, Hq, Hkv, T, d, default_scale(d), True, -1, -1, cud, 200)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_SEQLENS
    assert ea.attn_device_status() == ea.ATTN_OK  # read clears it
    o, lse = o.cpu(), lse.cpu()
    assert torch.isnan(o[:300].float()).all() and torch.isnan(lse[:, :300]).all()
    kw = dict(B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=default_scale(d), causal=True, cu_seqlens=cu)
    o_ref, lse_ref, _ = oracle_run(q, k, v, **kw)
    o_ref = o_ref.reshape(T, Hq, d)
    assert np.abs(o[300:].double().numpy() - o_ref[300:]).max() <= TOL_O
    assert np.abs(lse[:, 300:].double().numpy() - lse_ref.reshape(Hq, T)[:, 300:]).max() <= TOL_LSE
    o2, lse2 = gpu_run(q, k, v, max_seqlen=300, **kw)  # asserts a clean status
    compare_full(o2, lse2, o_ref, lse_ref)
