"""GPU parity of attn_fwd_fp8 (e4m3 inputs) with the fp64 oracle on the same
values, through the C ABI.  The oracle takes the e4m3 values widened exactly to
bf16 (pinned by pin_e4m3_widening).

Tolerance, derived from the arithmetic.  With exact scores s_j, weights
p_j = exp(s_j - max) and O = sum p_j v_j / sum p_j, the kernel uses e4m3-rounded
weights p'_j with |p'_j - p_j| <= delta_j = max(2^-4 p_j, 2^-10) (three
mantissa bits: half an ulp is 2^-4 of a normal value; below 2^-6 the spacing is
2^-9) and divides by their sum, so
    |O' - O| <= sum_j delta_j |v_j - O| / (sum_j p_j (1 - 2^-4)).
The kernel's lazy maximum only scales every p_j up by the same power of two,
which shrinks the 2^-10 term, so the bound with the true maximum holds.  Added:
the bf16 rounding of O (2^-9 |O'|, taken as 2^-8 |O|) and 2e-3 for the exp2
approximations and fp32 sums.  Each element must satisfy
    |O_gpu - O_ref| <= 1.07 * bound + 2^-8 |O_ref| + 2e-3.
The LSE comes from the fp32 weights: |dLSE| <= 1e-3 as for bf16 inputs, and
the mask pattern must be bit-exact."""
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
TOL_LSE = 1e-3


def gpu_fp8(q, k, v, *, B, Hq, Hkv, N, d, scale, causal, left=-1, right=-1, cu=None):
    qd, kd, vd = (t.view(torch.uint8).to(DEV) for t in (q, k, v))
    packed = cu is not None
    cud = torch.tensor(cu, dtype=torch.int32, device=DEV) if packed else None
    max_seqlen = max(b - a for a, b in zip(cu[:-1], cu[1:])) if packed else 0
    tokens = N if packed else B * N
    o = torch.full((tokens, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((Hq * N,) if packed else (B * Hq * N,), float("nan"), dtype=torch.float32,
                     device=DEV)
    nbytes = ea.attn_fwd_fp8_workspace_bytes(B, Hq, Hkv, N, d, packed)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    ea.attn_fwd_fp8(qd, kd, vd, o, lse, B, Hq, Hkv, N, d, scale, causal, left, right, cud,
                    max_seqlen, ws, nbytes)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    return o.cpu(), lse.cpu()


def widened(t):
    return W.bf16_bits(W.e4m3_as_bf16(t))


def oracle_fp8(q, k, v, rows=None, **kw):
    kw = {k_: v_ for k_, v_ in kw.items() if k_ not in ("left", "right", "cu")} | {
        "window_left": kw.get("left", -1), "window_right": kw.get("right", -1),
        "cu_seqlens": kw.get("cu")}
    return oracle.attn_fwd(widened(q), widened(k), widened(v), rows=rows, **kw)


def row_bound(qf, kf, vf, o_row, i, lo, hi, scale):
    """The derived error bound for one query row (visible keys lo..hi)."""
    ks = kf[lo:hi + 1]
    vs = vf[lo:hi + 1]
    s = scale * (ks @ qf)
    p = np.exp(s - s.max())
    delta = np.maximum(2.0 ** -4 * p, 2.0 ** -10)
    spread = np.abs(vs - o_row[None, :])  # [keys, d]
    return (delta @ spread) / (p.sum() * (1 - 2.0 ** -4))


def visible_range(i, L, causal, left, right):
    r = 0 if causal else right
    lo = max(0, i - left) if left >= 0 else 0
    hi = min(L - 1, i + r) if r >= 0 else L - 1
    return lo, hi


def check_rows(o_gpu, lse_gpu, o_ref, lse_ref, qf, kf, vf, rows, scale, causal, left, right,
               lengths, group):
    """rows: (sequence, head, row, index into o_ref / lse_ref, token) tuples."""
    for (b, h, i, r_idx, tok) in rows:
        lo, hi = visible_range(i, lengths[b], causal, left, right)
        start = tok - i
        bound = row_bound(qf[tok, h], kf[start:start + lengths[b], h // group],
                          vf[start:start + lengths[b], h // group], o_ref[r_idx], i, lo, hi, scale)
        tol = 1.07 * bound + 2.0 ** -8 * np.abs(o_ref[r_idx]) + 2e-3
        err = np.abs(o_gpu[tok, h] - o_ref[r_idx])
        assert (err <= tol).all(), (b, h, i, float(err.max()), float(tol[err.argmax()]))
        assert abs(lse_gpu[r_idx] - lse_ref[r_idx]) <= TOL_LSE


CASES = [
    # B, Hq, Hkv, N, causal, left, right
    (2, 4, 2, 256, True, -1, -1),
    (1, 4, 4, 300, True, -1, -1),     # ragged tail, MHA (row pairs)
    (2, 8, 1, 200, False, -1, -1),    # MQA
    (1, 4, 2, 400, True, 100, 0),     # sliding window
    (1, 2, 2, 129, False, 20, 40),
    (1, 2, 1, 1, True, -1, -1),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "b{}_h{}x{}_n{}_c{}_w{}_{}".format(*c))
def test_fp8_parity(case):
    B, Hq, Hkv, N, causal, left, right = case
    d = 128
    q, k, v = W.draw_qkv_e4m3((B, N, Hq, d), (B, N, Hkv, d), seed=N + 7)
    scale = default_scale(d)
    o_gpu, lse_gpu = gpu_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=causal,
                             left=left, right=right)
    o_ref, lse_ref, _ = oracle_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale,
                                   causal=causal, left=left, right=right)
    T = B * N
    qf = W.e4m3_as_bf16(q).double().numpy().reshape(T, Hq, d)
    kf = W.e4m3_as_bf16(k).double().numpy().reshape(T, Hkv, d)
    vf = W.e4m3_as_bf16(v).double().numpy().reshape(T, Hkv, d)
    og = o_gpu.double().numpy().reshape(T, Hq, d)
    lg = lse_gpu.double().numpy().reshape(B, Hq, N)
    assert np.isfinite(og).all()
    o_ref = o_ref.reshape(T, Hq, d)
    rows = []
    o_rows, l_rows = [], []
    for b in range(B):
        for h in range(Hq):
            for i in range(N):
                tok = b * N + i
                rows.append((b, h, i, len(rows), tok))
                o_rows.append(o_ref[tok, h])
                l_rows.append((lg[b, h, i], lse_ref[b, h, i]))
    check_rows(og, np.array([a for a, _ in l_rows]), np.array(o_rows), np.array([r for _, r in l_rows]),
               qf, kf, vf, rows, scale, causal, left, right, [N] * B, Hq // Hkv)


def test_fp8_packed():
    lens = [100, 1, 257, 0, 130]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 128
    q, k, v = W.draw_qkv_e4m3((T, Hq, d), (T, Hkv, d), seed=17)
    scale = default_scale(d)
    o_gpu, lse_gpu = gpu_fp8(q, k, v, B=len(lens), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=scale,
                             causal=True, cu=cu)
    o_ref, lse_ref, _ = oracle_fp8(q, k, v, B=len(lens), Hq=Hq, Hkv=Hkv, N=T, d=d, scale=scale,
                                   causal=True, cu=cu)
    qf = W.e4m3_as_bf16(q).double().numpy()
    kf = W.e4m3_as_bf16(k).double().numpy()
    vf = W.e4m3_as_bf16(v).double().numpy()
    og = o_gpu.double().numpy()
    lg = lse_gpu.double().numpy().reshape(Hq, T)
    rows, o_rows, lg_rows, lr_rows = [], [], [], []
    for b, L in enumerate(lens):
        for h in range(Hq):
            for i in range(L):
                tok = cu[b] + i
                rows.append((b, h, i, len(rows), tok))
                o_rows.append(o_ref[tok, h])
                lg_rows.append(lg[h, tok])
                lr_rows.append(lse_ref[h, tok])
    check_rows(og, np.array(lg_rows), np.array(o_rows), np.array(lr_rows), qf, kf, vf, rows, scale,
               True, -1, -1, lens, Hq // Hkv)


@pytest.mark.parametrize("left,causal,right", [(-1, True, -1), (50, True, -1), (30, False, 20)])
def test_fp8_mask_pattern_bit_exact(left, causal, right):
    B, Hq, Hkv, N, d = 1, 2, 1, 333, 128
    q, k, v = W.draw_qkv_e4m3((B, N, Hq, d), (B, N, Hkv, d), seed=3)
    q.zero_()
    _, lse = gpu_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=0.1, causal=causal, left=left,
                     right=right)
    _, _, nvis = oracle_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=0.1, causal=causal,
                            left=left, right=right)
    count = np.rint(np.exp(lse.double().numpy().reshape(nvis.shape))).astype(np.int64)
    assert np.array_equal(count, nvis)


def test_fp8_gqa_workload_sampled_rows():
    """The 8192-token causal GQA shape (B=2, Hq=32, Hkv=8) in e4m3, checked on
    sampled rows (first, last, tile boundaries, random)."""
    B, Hq, Hkv, N, d = 2, 32, 8, 8192, 128
    q, k, v = W.draw_qkv_e4m3((B, N, Hq, d), (B, N, Hkv, d), seed=2)
    scale = default_scale(d)
    o_gpu, lse_gpu = gpu_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=True)
    rng = np.random.default_rng(8)
    picks = [(0, 0, 0), (1, 31, N - 1), (0, 5, 127), (0, 6, 128), (1, 17, 4095)]
    picks += [(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(40)]
    rows_arr = np.array(picks, dtype=np.int64)
    o_ref, lse_ref, _ = oracle_fp8(q, k, v, rows=rows_arr, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d,
                                   scale=scale, causal=True)
    T = B * N
    qf = W.e4m3_as_bf16(q).double().numpy().reshape(T, Hq, d)
    kf = W.e4m3_as_bf16(k).double().numpy().reshape(T, Hkv, d)
    vf = W.e4m3_as_bf16(v).double().numpy().reshape(T, Hkv, d)
    og = o_gpu.double().numpy().reshape(T, Hq, d)
    lg = lse_gpu.double().numpy().reshape(B, Hq, N)
    rows = [(b, h, i, r, b * N + i) for r, (b, h, i) in enumerate(picks)]
    check_rows(og, np.array([lg[b, h, i] for b, h, i in picks]), o_ref, lse_ref, qf, kf, vf, rows,
               scale, True, -1, -1, [N] * B, Hq // Hkv)


def test_fp8_schedule_many_pairs_per_cta():
    """Several hundred tile pairs (many per CTA under the persistent schedule),
    ragged tail, GQA."""
    B, Hq, Hkv, N, d = 16, 8, 2, 300, 128
    q, k, v = W.draw_qkv_e4m3((B, N, Hq, d), (B, N, Hkv, d), seed=35)
    scale = default_scale(d)
    o_gpu, lse_gpu = gpu_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=True)
    o_ref, lse_ref, _ = oracle_fp8(q, k, v, B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=scale, causal=True)
    T = B * N
    qf = W.e4m3_as_bf16(q).double().numpy().reshape(T, Hq, d)
    kf = W.e4m3_as_bf16(k).double().numpy().reshape(T, Hkv, d)
    vf = W.e4m3_as_bf16(v).double().numpy().reshape(T, Hkv, d)
    og = o_gpu.double().numpy().reshape(T, Hq, d)
    lg = lse_gpu.double().numpy().reshape(B, Hq, N)
    o_ref = o_ref.reshape(T, Hq, d)
    rng = np.random.default_rng(36)
    picks = [(b, h, i) for b in (0, B - 1) for h in (0, Hq - 1) for i in (0, 127, 128, 255, 256, N - 1)]
    picks += [(int(rng.integers(B)), int(rng.integers(Hq)), int(rng.integers(N))) for _ in range(200)]
    rows = [(b, h, i, r, b * N + i) for r, (b, h, i) in enumerate(picks)]
    check_rows(og, np.array([lg[b, h, i] for b, h, i in picks]),
               np.array([o_ref[b * N + i, h] for b, h, i in picks]),
               np.array([lse_ref[b, h, i] for b, h, i in picks]), qf, kf, vf, rows, scale, True,
               -1, -1, [N] * B, Hq // Hkv)
    # every row of every pair was written
    assert np.isfinite(og).all() and np.isfinite(lg).all()


def test_fp8_packed_max_seqlen_too_small_is_reported():
    """As attn_fwd: a sequence longer than max_seqlen (rounded up to 128 rows)
    is skipped, nothing of it is read or written, and the status word reports
    it; the other sequences equal a call with the right max_seqlen."""
    lens = [300, 129, 50]
    cu = W.cumulative(lens)
    T, Hq, Hkv, d = cu[-1], 4, 2, 128
    q, k, v = W.draw_qkv_e4m3((T, Hq, d), (T, Hkv, d), seed=18)
    scale = default_scale(d)
    good_o, good_l = gpu_fp8(q, k, v, B=3, Hq=Hq, Hkv=Hkv, N=T, d=d, scale=scale, causal=True,
                             cu=cu)
    qd, kd, vd = (t.view(torch.uint8).to(DEV) for t in (q, k, v))
    cud = torch.tensor(cu, dtype=torch.int32, device=DEV)
    o = torch.full((T, Hq, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((Hq, T), float("nan"), dtype=torch.float32, device=DEV)
    nbytes = ea.attn_fwd_fp8_workspace_bytes(3, Hq, Hkv, T, d, True)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=DEV)
    ea.attn_fwd_fp8(qd, kd, vd, o, lse, 3, Hq, Hkv, T, d, scale, True, -1, -1, cud, 200, ws, nbytes)
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_ERR_SEQLENS
    assert ea.attn_device_status() == ea.ATTN_OK
    o, lse = o.cpu(), lse.cpu()
    assert torch.isnan(o[:300].float()).all() and torch.isnan(lse[:, :300]).all()
    assert torch.equal(o[300:], good_o[300:])
    assert torch.equal(lse[:, 300:], good_l.reshape(Hq, T)[:, 300:])
