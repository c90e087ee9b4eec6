"""Exact fused attention forward for NVIDIA B200 (sm_100a).

The computation runs in hand-written CUDA (tcgen05 tensor cores, TMEM, TMA)
behind the C ABI declared in include/attn.h; this package is a thin ctypes
binding over it.  ``attention`` is a convenience wrapper that allocates the
outputs with torch and calls ``attn_fwd``.
"""
from ._binding import (  # noqa: F401
    ATTN_ERR_ALIGN, ATTN_ERR_CUDA, ATTN_ERR_DEVICE_TIMEOUT, ATTN_ERR_NULL, ATTN_ERR_PAGE, ATTN_ERR_SCALE,
    ATTN_ERR_SEQLENS, ATTN_ERR_SHAPE, ATTN_ERR_UNSUPPORTED, ATTN_ERR_WINDOW, ATTN_ERR_WORKSPACE,
    ATTN_OK, AttnError, attn_bwd, attn_bwd_workspace_bytes, attn_decode,
    attn_decode_default_splits,
    attn_decode_noalloc, attn_decode_noalloc_scratch_bytes, attn_decode_workspace_bytes,
    attn_device_status,
    attn_acc_to_bf16, attn_fwd, attn_fwd_accumulate, attn_fwd_fp8, attn_fwd_fp8_workspace_bytes,
    attn_fwd_host, attn_fwd_host_workspace_bytes,
    attn_selftest_bounded_wait, attn_selftest_exp2_poly, attn_status_string, library_path,
    load_library)


def attention(q, k, v, *, causal=False, window_left=-1, window_right=-1, scale=None,
              cu_seqlens=None, max_seqlen=0, stream=None):
    """Allocate O and LSE on q's device and run attn_fwd.

    Dense: q [B, N, Hq, d], k/v [B, N, Hkv, d] -> o [B, N, Hq, d], lse [B, Hq, N].
    Packed: q [T, Hq, d], k/v [T, Hkv, d], cu_seqlens int32 [B+1] on the device
    -> o [T, Hq, d], lse [Hq, T].  Without max_seqlen the longest sequence is
    read back from cu_seqlens (a device-to-host copy); attn_fwd itself never
    reads cu_seqlens on the host.
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
        if max_seqlen <= 0 and B > 0:
            max_seqlen = int((cu_seqlens[1:] - cu_seqlens[:-1]).max().item())
    o = torch.empty_like(q)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal, window_left, window_right,
             cu_seqlens, max_seqlen, stream)
    return o, lse


def attention_with_kvcache(q, k_cache, v_cache, cache_seqlens, *, block_table=None, causal=True,
                           window_left=-1, window_right=-1, scale=None, num_splits=0,
                           stream=None):
    """Newest-token attention against a (paged) key/value cache via attn_decode.

    q [B, Nq, Hq, d]; caches [num_pages, page_size, Hkv, d]; cache_seqlens int32
    [B] and block_table int32 [B, pages_per_seq] (or None: contiguous cache, then
    num_pages = B * pages_per_seq) on the device.  num_splits <= 0 picks
    attn_decode_default_splits.  Returns o [B, Nq, Hq, d], lse [B, Hq, Nq].
    """
    import math

    import torch
    B, Nq, Hq, d = q.shape
    page_size, Hkv = k_cache.shape[1], k_cache.shape[2]
    pages_per_seq = block_table.shape[1] if block_table is not None else k_cache.shape[0] // B
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if num_splits <= 0:
        num_splits = attn_decode_default_splits(B, Hq, Hkv, Nq, page_size * pages_per_seq)
    o = torch.empty_like(q)
    lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=q.device)
    nbytes = attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, page_size, pages_per_seq, num_splits)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=q.device) if nbytes else None
    attn_decode(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv, Nq, d,
                page_size, pages_per_seq, k_cache.shape[0], scale, causal, window_left,
                window_right, num_splits, ws, nbytes, stream)
    return o, lse
