"""ctypes binding of the C ABI in include/attn.h (argument marshalling only).

Every entry point keeps the C name.  Tensors may be passed as torch tensors
(their data pointer is used) or as raw integer addresses; streams as
torch.cuda.Stream, a raw handle, or None for torch's current stream.  All
computation happens in the CUDA library; there is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
import threading

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libattn_b200.so")
_lib = None
_lock = threading.Lock()

ATTN_OK = 0
ATTN_ERR_NULL = -1
ATTN_ERR_SHAPE = -2
ATTN_ERR_WINDOW = -3
ATTN_ERR_UNSUPPORTED = -4
ATTN_ERR_ALIGN = -5
ATTN_ERR_CUDA = -6
ATTN_ERR_SCALE = -7
ATTN_ERR_WORKSPACE = -8
ATTN_ERR_DEVICE_TIMEOUT = -9
ATTN_ERR_PAGE = -10
ATTN_ERR_SEQLENS = -11


class AttnError(RuntimeError):
    def __init__(self, status: int, what: str = "attn_fwd"):
        self.status = status
        super().__init__(f"{what} failed: {attn_status_string(status)} (status {status})")


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load the CUDA library; raise loudly if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"CUDA library {_LIB_PATH} is missing; build it with "
                "`python -m exact_attention_142_b200.build` (there is no fallback)")
        lib = ctypes.CDLL(_LIB_PATH)
        P, I, F, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.attn_fwd.restype = I
        lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I, P]
        lib.attn_fwd_fp8.restype = I
        lib.attn_fwd_fp8.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I, P, S, P]
        lib.attn_fwd_fp8_workspace_bytes.restype = S
        lib.attn_fwd_fp8_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.attn_fwd_accumulate.restype = I
        lib.attn_fwd_accumulate.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I, P]
        lib.attn_acc_to_bf16.restype = I
        lib.attn_acc_to_bf16.argtypes = [P, P, ctypes.c_longlong, P]
        lib.attn_fwd_host.restype = I
        lib.attn_fwd_host.argtypes = [P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I, P, S, P]
        lib.attn_fwd_host_workspace_bytes.restype = S
        lib.attn_fwd_host_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.attn_bwd.restype = I
        lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, F, I, I, I, P, I, P, S, P]
        lib.attn_bwd_workspace_bytes.restype = S
        lib.attn_bwd_workspace_bytes.argtypes = [I, I, I, I, I, I]
        lib.attn_decode.restype = I
        lib.attn_decode.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I, I, I, P,
                                    S, P]
        lib.attn_decode_noalloc.restype = I
        lib.attn_decode_noalloc.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, I, F, I, I,
                                            I, I, P]
        lib.attn_decode_noalloc_scratch_bytes.restype = S
        lib.attn_decode_noalloc_scratch_bytes.argtypes = []
        lib.attn_decode_workspace_bytes.restype = S
        lib.attn_decode_workspace_bytes.argtypes = [I, I, I, I, I, I, I, I]
        lib.attn_decode_default_splits.restype = I
        lib.attn_decode_default_splits.argtypes = [I, I, I, I, I]
        lib.attn_status_string.restype = ctypes.c_char_p
        lib.attn_status_string.argtypes = [I]
        lib.attn_device_status.restype = I
        lib.attn_device_status.argtypes = []
        lib.attn_selftest_bounded_wait.restype = I
        lib.attn_selftest_bounded_wait.argtypes = [ctypes.c_uint64, P]
        lib.attn_selftest_exp2_poly.restype = I
        lib.attn_selftest_exp2_poly.argtypes = [P, P, ctypes.c_longlong, P]
        _lib = lib
        return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr() if x.numel() > 0 else None
    if hasattr(x, "ctypes"):  # numpy array
        return x.ctypes.data
    raise TypeError(f"cannot take a pointer of {type(x)}")


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def attn_fwd(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal=False, window_left=-1,
             window_right=-1, cu_seqlens=None, max_seqlen=0, stream=None, check=True) -> int:
    """Enqueue the fused forward on device buffers (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq), int(Hkv),
                      int(N), int(d), float(scale), int(bool(causal)), int(window_left),
                      int(window_right), _ptr(cu_seqlens), int(max_seqlen), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc)
    return rc


def attn_fwd_fp8(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal=False, window_left=-1,
                 window_right=-1, cu_seqlens=None, max_seqlen=0, workspace=None, workspace_bytes=0,
                 stream=None, check=True) -> int:
    """The fused forward on e4m3 inputs (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq), int(Hkv),
                          int(N), int(d), float(scale), int(bool(causal)), int(window_left),
                          int(window_right), _ptr(cu_seqlens), int(max_seqlen), _ptr(workspace),
                          int(workspace_bytes), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_fp8")
    return rc


def attn_fwd_fp8_workspace_bytes(B, Hq, Hkv, N, d, packed) -> int:
    return int(load_library().attn_fwd_fp8_workspace_bytes(int(B), int(Hq), int(Hkv), int(N), int(d),
                                                           int(bool(packed))))


def attn_fwd_accumulate(q, k, v, o_acc, lse_acc, B, Hq, Hkv, N, d, scale, causal=False,
                        window_left=-1, window_right=-1, cu_seqlens=None, max_seqlen=0,
                        stream=None, check=True) -> int:
    """Merge this call's attention into an fp32 accumulator (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_fwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc), int(B),
                                 int(Hq), int(Hkv), int(N), int(d), float(scale), int(bool(causal)),
                                 int(window_left), int(window_right), _ptr(cu_seqlens),
                                 int(max_seqlen), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_accumulate")
    return rc


def attn_acc_to_bf16(o_acc, o, n, stream=None, check=True) -> int:
    rc = load_library().attn_acc_to_bf16(_ptr(o_acc), _ptr(o), int(n), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_acc_to_bf16")
    return rc


def attn_fwd_host_workspace_bytes(B, Hq, Hkv, N, d, packed) -> int:
    return int(load_library().attn_fwd_host_workspace_bytes(int(B), int(Hq), int(Hkv), int(N),
                                                            int(d), int(bool(packed))))


def attn_fwd_host(q, k, v, o, lse, B, Hq, Hkv, N, d, scale, causal=False, window_left=-1,
                  window_right=-1, cu_seqlens=None, max_seqlen=0, workspace=None,
                  workspace_bytes=0, stream=None, check=True) -> int:
    """Same operation on host buffers; copies run on `stream` (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_fwd_host(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), int(B), int(Hq),
                           int(Hkv), int(N), int(d), float(scale), int(bool(causal)),
                           int(window_left), int(window_right), _ptr(cu_seqlens), int(max_seqlen),
                           _ptr(workspace), int(workspace_bytes), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_host")
    return rc


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, B, Hq, Hkv, N, d, scale, causal=False,
             window_left=-1, window_right=-1, cu_seqlens=None, max_seqlen=0, workspace=None,
             workspace_bytes=0, stream=None, check=True) -> int:
    """Enqueue the backward pass on device buffers (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                      _ptr(dv), int(B), int(Hq), int(Hkv), int(N), int(d), float(scale),
                      int(bool(causal)), int(window_left), int(window_right), _ptr(cu_seqlens),
                      int(max_seqlen), _ptr(workspace), int(workspace_bytes), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd")
    return rc


def attn_bwd_workspace_bytes(B, Hq, Hkv, N, d, packed) -> int:
    return int(load_library().attn_bwd_workspace_bytes(int(B), int(Hq), int(Hkv), int(N), int(d),
                                                       int(bool(packed))))


def attn_decode(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv, Nq, d,
                page_size, pages_per_seq, num_pages, scale, causal=True, window_left=-1,
                window_right=-1, num_splits=1, workspace=None, workspace_bytes=0, stream=None,
                check=True) -> int:
    """Enqueue the key/value-cache decode on device buffers (see include/attn.h)."""
    lib = load_library()
    rc = lib.attn_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                         _ptr(cache_seqlens), _ptr(block_table), int(B), int(Hq), int(Hkv),
                         int(Nq), int(d), int(page_size), int(pages_per_seq), int(num_pages),
                         float(scale),
                         int(bool(causal)), int(window_left), int(window_right), int(num_splits),
                         _ptr(workspace), int(workspace_bytes), _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_decode")
    return rc




def attn_decode_noalloc(q, k_cache, v_cache, o, lse, cache_seqlens, block_table, B, Hq, Hkv, Nq,
                        d, page_size, pages_per_seq, num_pages, scale, causal=True,
                        window_left=-1, window_right=-1, num_splits=1, stream=None,
                        check=True) -> int:
    """attn_decode with the library's fixed scratch instead of a workspace, for
    callers that must not allocate device memory while they run (see
    include/attn.h)."""
    lib = load_library()
    rc = lib.attn_decode_noalloc(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(o), _ptr(lse),
                                 _ptr(cache_seqlens), _ptr(block_table), int(B), int(Hq),
                                 int(Hkv), int(Nq), int(d), int(page_size), int(pages_per_seq),
                                 int(num_pages), float(scale), int(bool(causal)),
                                 int(window_left), int(window_right), int(num_splits),
                                 _stream(stream))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_decode_noalloc")
    return rc


def attn_decode_noalloc_scratch_bytes() -> int:
    """Size of the library's fixed decode scratch array, read from the library."""
    return int(load_library().attn_decode_noalloc_scratch_bytes())


def attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, page_size, pages_per_seq, num_splits) -> int:
    return int(load_library().attn_decode_workspace_bytes(
        int(B), int(Hq), int(Hkv), int(Nq), int(d), int(page_size), int(pages_per_seq),
        int(num_splits)))


def attn_decode_default_splits(B, Hq, Hkv, Nq, max_cache_len) -> int:
    return int(load_library().attn_decode_default_splits(int(B), int(Hq), int(Hkv), int(Nq),
                                                         int(max_cache_len)))


def attn_status_string(status: int) -> str:
    return load_library().attn_status_string(int(status)).decode()


def attn_device_status() -> int:
    return int(load_library().attn_device_status())


def attn_selftest_bounded_wait(limit_ns: int, stream=None) -> int:
    return int(load_library().attn_selftest_bounded_wait(int(limit_ns), _stream(stream)))


def attn_selftest_exp2_poly(x, y, n, stream=None, check=True) -> int:
    """y = 2^x through the kernels' FMA-pipe exponential (see include/attn.h)."""
    rc = int(load_library().attn_selftest_exp2_poly(_ptr(x), _ptr(y), int(n), _stream(stream)))
    if check and rc != ATTN_OK:
        raise AttnError(rc, "attn_selftest_exp2_poly")
    return rc
