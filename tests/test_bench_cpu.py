"""Host-side pieces of bench.py: the FLOP and byte counts behind the reported
TFLOP/s and GB/s (against closed forms), the traffic record's digest guard,
and the step statistics.  No GPU."""
from __future__ import annotations

import bench
import workloads as W


def pairs_closed_form(L: int, left: int, right: int) -> int:
    """Visible (i, j) pairs of one length-L sequence, i - left <= j <= i + right,
    summed row by row with the window clipped to [0, L)."""
    total = 0
    for i in range(L):
        lo = 0 if left < 0 else max(0, i - left)
        hi = L - 1 if right < 0 else min(L - 1, i + right)
        total += hi - lo + 1
    return total


def test_causal_pairs_are_triangular():
    w = W.workload(3)  # causal, N = 8192
    assert bench.visible_pairs(w) == w.B * w.N * (w.N + 1) // 2


def test_forward_flops_of_the_named_workloads():
    # 4 d flops per visible pair and query head (two products of 2 d each)
    w2, w3 = W.workload(2), W.workload(3)
    assert bench.flops_of(w2) == 4 * 128 * 16 * 4 * (2048 * 2049 // 2)
    assert bench.flops_of(w3) == 4 * 128 * 32 * 2 * (8192 * 8193 // 2)
    assert abs(bench.flops_of(w3) - 1.0996e12) / 1.0996e12 < 1e-4


def test_window_pairs_match_the_row_by_row_count():
    w = W.workload(4)  # left 4096, causal
    # first 4096 rows see i + 1 keys, the rest 4097
    closed = 4096 * 4097 // 2 + (w.N - 4096) * 4097
    assert bench.visible_pairs(w) == closed
    small = W.Workload("t", 1, 1, 1, 300, 64, False, 20, 7, 0)
    assert bench.visible_pairs(small) == pairs_closed_form(300, 20, 7)


def test_packed_pairs_sum_over_sequences():
    w = W.workload(5)
    lengths = [b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])]
    assert bench.visible_pairs(w) == sum(L * (L + 1) // 2 for L in lengths)


def test_backward_flops_are_two_and_a_half_forwards():
    w = W.workload(3)
    assert bench.bwd_flops_of(w) == 2.5 * bench.flops_of(w)


def test_decode_bytes_count_each_cached_key_once():
    w = W.decode_workload(64)
    keys = sum(w.lengths)  # causal, no window: every cached key is visible
    assert bench.decode_visible_keys(w) == keys
    expect = 2 * keys * w.Hkv * w.d * 2 + 2 * w.B * w.Nq * w.Hq * w.d * 2 + 4 * w.B * w.Hq * w.Nq
    assert bench.decode_bytes(w) == expect


def test_traffic_record_requires_matching_sources(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cuh"
    src.write_text("version 1\n")
    (tmp_path / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    digest = bench.kernel_sources_digest(["kernel.cuh"])
    (tmp_path / "profiles" / "attn_fwd_wl_traffic.md").write_text(
        f"traffic_bytes_per_launch: 12345\nkernel_sources_sha256_16: {digest}\n")
    assert bench.recorded_traffic("wl", sources=["kernel.cuh"]) == 12345.0
    src.write_text("version 2\n")  # the kernel changed since the counters were taken
    assert bench.recorded_traffic("wl", sources=["kernel.cuh"]) is None
    assert bench.recorded_traffic("missing", sources=["kernel.cuh"]) is None


def test_step_stats():
    st = bench.step_stats([3.0, 1.0, 2.0, 4.0])
    assert st["min"] == 1.0 and st["max"] == 4.0 and st["mean"] == 2.5 and st["median"] == 3.0
    assert bench.step_stats([]) is None
