"""The oracle's results do not depend on how many host threads compute them:
every row (forward, cache decode) and every gradient sum (backward) is
accumulated in a fixed order by one thread.  No GPU."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import workloads as W


@pytest.mark.parametrize("causal,left,right", [(True, -1, -1), (False, 40, 9)])
def test_forward_independent_of_threads(causal, left, right):
    B, Hq, Hkv, N, d = 2, 4, 2, 150, 64
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), 71)
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=d ** -0.5, causal=causal, window_left=left,
              window_right=right)
    a = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), nthreads=1, **kw)
    b = oracle.attn_fwd(W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), nthreads=5, **kw)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_backward_independent_of_threads():
    B, Hq, Hkv, N, d = 1, 4, 2, 130, 64
    q, k, v = W.draw_qkv((B, N, Hq, d), (B, N, Hkv, d), 72)
    g = torch.Generator().manual_seed(73)
    do = torch.randn((B, N, Hq, d), dtype=torch.float32, generator=g).to(torch.bfloat16)
    args = (W.bf16_bits(q), W.bf16_bits(k), W.bf16_bits(v), W.bf16_bits(do))
    kw = dict(B=B, Hq=Hq, Hkv=Hkv, N=N, d=d, scale=d ** -0.5, causal=True)
    a = oracle.attn_bwd(*args, nthreads=1, **kw)
    b = oracle.attn_bwd(*args, nthreads=3, **kw)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
