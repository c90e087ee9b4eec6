"""One forward split over ranks (exact_attention_142_b200/split.py) on the real
kernel.  With a single GPU visible, each rank's shard runs in turn on it; the
parts are placed back with `unshard` and must equal the whole-workload call
bit for bit: every (sequence, head) is computed independently of the others
("FlashAttention" explainer page, How it works, Step 7), with the same
arithmetic whichever CTA or launch computes it.  The whole-workload result
itself is pinned to the oracle by test_attn_gpu.py."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import exact_attention_142_b200 as ea
import workloads as W
from exact_attention_142_b200 import split
from gpu_helpers import default_scale

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_attention_142_b200 import build
    build.build()
    ea.load_library()


# (name, world, mode, dense (B, N) or packed lengths, Hq, Hkv, d, causal, left, right, seed)
CASES = [
    ("heads_dense_causal", 2, "heads", (2, 600), 8, 4, 128, True, -1, -1, 31),
    ("heads_gqa_window", 4, "heads", (1, 1000), 16, 4, 128, True, 200, 0, 32),
    ("heads_rowpairs_d64", 3, "heads", (2, 333), 6, 3, 64, True, -1, -1, 33),
    ("sequences_packed_causal", 3, "sequences", [300, 5, 700, 129, 1000, 64], 4, 2, 128, True, -1, -1, 34),
    ("sequences_dense_noncausal", 2, "sequences", (3, 256), 2, 1, 64, False, -1, -1, 35),
    ("sequences_packed_window", 4, "sequences", [513, 0, 77, 1200, 300, 31], 4, 4, 128, False, 64, 64, 36),
]


def _run_case(world, mode, shape, Hq, Hkv, d, causal, left, right, seed):
    dev = torch.device("cuda:0")
    scale = default_scale(d)
    if isinstance(shape, tuple):
        B, N = shape
        q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), seed)
        cu, lengths, cud = None, [N] * B, None
    else:
        lengths = list(shape)
        cu = W.cumulative(lengths)
        B, N = len(lengths), cu[-1]
        q, k, v = W.draw_qkv((N, Hq, d), (N, Hkv, d), seed)
        cud = torch.tensor(cu, dtype=torch.int32, device=dev)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    o_whole, lse_whole = ea.attention(qd, kd, vd, causal=causal, window_left=left, window_right=right,
                                      scale=scale, cu_seqlens=cud, max_seqlen=max(lengths))
    shards = split.plan(world, mode, B=B, Hq=Hq, Hkv=Hkv, lengths=lengths, causal=causal, left=left,
                        right=right)
    parts = [split.run_shard(qd, kd, vd, s, causal=causal, scale=scale, left=left, right=right,
                             cu_seqlens=cu) for s in shards]
    torch.cuda.synchronize()
    assert ea.attn_device_status() == ea.ATTN_OK
    o, lse = split.unshard(parts, shards, B=B, Hq=Hq, d=d, cu_seqlens=cu, N=N)
    return shards, o, lse, o_whole.cpu().double().numpy(), lse_whole.cpu().double().numpy()


@pytest.mark.parametrize("case", CASES, ids=lambda c: c[0])
def test_split_shards_equal_whole_call(case):
    _, world, mode, shape, Hq, Hkv, d, causal, left, right, seed = case
    shards, o, lse, o_ref, lse_ref = _run_case(world, mode, shape, Hq, Hkv, d, causal, left, right, seed)
    assert sum(not s.empty for s in shards) >= 2  # the work really was split
    assert np.array_equal(o, o_ref)
    assert np.array_equal(lse, lse_ref)


@pytest.mark.parametrize("cfg,world,mode", [(3, 8, "heads"), (5, 4, "sequences")])
def test_split_full_workloads(cfg, world, mode):
    """The benchmark's GQA workload split over eight ranks by heads, and the
    packed one over four by sequences (bench.py --split)."""
    w = W.workload(cfg)
    shape = (w.B, w.N) if not w.packed else [b - a for a, b in zip(w.cu_seqlens[:-1], w.cu_seqlens[1:])]
    shards, o, lse, o_ref, lse_ref = _run_case(world, mode, shape, w.Hq, w.Hkv, w.d, w.causal,
                                               w.window_left, w.window_right, w.seed)
    assert sum(not s.empty for s in shards) == world
    assert np.array_equal(o, o_ref)
    assert np.array_equal(lse, lse_ref)
