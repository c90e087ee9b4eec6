"""Exact fused attention forward for NVIDIA B200 (sm_100a).

The computation runs in hand-written CUDA (tcgen05 tensor cores, TMEM, TMA)
behind the C ABI declared in include/attn.h; this package is a thin ctypes
binding over it.  ``attention`` is a convenience wrapper that allocates the
outputs with torch and calls ``attn_fwd``.
"""
from ._binding import (  # noqa: F401
    ATTN_ERR_ALIGN, ATTN_ERR_CUDA, ATTN_ERR_DEVICE_TIMEOUT, ATTN_ERR_NULL, ATTN_ERR_SCALE,
    ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED, ATTN_ERR_WINDOW, ATTN_ERR_WORKSPACE, ATTN_OK, AttnError,
    attn_device_status, attn_fwd, attn_fwd_host, attn_fwd_host_workspace_bytes,
    attn_selftest_bounded_wait, attn_status_string, library_path, load_library)


def attention(q, k, v, *, causal=False, window_left=-1, window_right=-1, scale=None,
              cu_seqlens=None, max_seqlen=0, stream=None):
    """Allocate O and LSE on q's device and run attn_fwd.

    Dense: q [B, N, Hq, d], k/v [B, N, Hkv, d] -> o [B, N, Hq, d], lse [B, Hq, N].
    Packed: q [T, Hq, d], k/v [T, Hkv, d], cu_seqlens int32 [B+1] on the device
    -> o [T, Hq, d], lse [Hq, T].
    """
    import math

    import torch
    if cu_seqlens is None:
        B, N, Hq, d = q.shape
        Hkv = k.shape[2]
        lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device)
    else:
        N, Hq, d = q.shape
        Hkv = k.shape[1]
        B = cu_seqlens.numel() - 1
        lse = torch.empty((Hq, N), dtype=torch.float32, device=q.device)
    o = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window_left, window_right,
             cu_seqlens, max_seqlen, stream)
    return o, lse
