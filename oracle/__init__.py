"""CPU fp64 oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The product
(``exact_attention_142_b200``) never imports it and shares no code with it.

The arithmetic lives in ``attn_oracle.c`` (plain C, fp64, OpenMP over rows); it
follows the textbook definition of attention given on the "FlashAttention"
explainer page (ozercemkelahmet.com/tools/flashattention), sections "What it is"
and "Checking correctness".  This module only builds and loads that library and
marshals numpy arrays.

Pins (tests/test_oracle_pins.py) tie it to the pages' worked example, closed
forms, invariants and an independent library routine.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_SO = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False, src: str = _SRC, out: str = _SO) -> str:
    """Compile the oracle with gcc (-O2, no fast-math: rounding order is kept)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def load(path: Optional[str] = None):
    """Load (building if needed) the oracle shared library."""
    global _lib
    if path is None and _lib is not None:
        return _lib
    so = path or build()
    lib = ctypes.CDLL(so)
    lib.oracle_attn_fwd.restype = ctypes.c_int
    lib.oracle_attn_fwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q k v
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # o lse nvis
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,  # B Hq Hkv N d
        ctypes.c_double,  # scale
        ctypes.c_int, ctypes.c_int, ctypes.c_int,  # causal left right
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int,  # cu rows nrows threads
    ]
    lib.oracle_attn_kvcache.restype = ctypes.c_int
    lib.oracle_attn_kvcache.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q kc vc
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # o lse nvis
        ctypes.c_void_p, ctypes.c_void_p,  # cache_seqlens block_table
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,  # B Hq Hkv Nq d
        ctypes.c_int, ctypes.c_int, ctypes.c_double,  # page_size pages_per_seq scale
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,  # causal left right threads
    ]
    lib.oracle_attn_bwd.restype = ctypes.c_int
    lib.oracle_attn_bwd.argtypes = [
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # q k v dout
        ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,  # dq dk dv
        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,  # B Hq Hkv N d
        ctypes.c_double,  # scale
        ctypes.c_int, ctypes.c_int, ctypes.c_int,  # causal left right
        ctypes.c_void_p, ctypes.c_int,  # cu_seqlens threads
    ]
    lib.oracle_num_threads.restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def num_threads() -> int:
    return int(load().oracle_num_threads())


def _bits(a) -> np.ndarray:
    """Accept bf16 bit patterns as a uint16/int16 numpy array."""
    a = np.ascontiguousarray(a)
    if a.dtype == np.int16:
        a = a.view(np.uint16)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def attn_fwd(q, k, v, *, B: int, Hq: int, Hkv: int, N: int, d: int, scale: float,
             causal: bool = False, window_left: int = -1, window_right: int = -1,
             cu_seqlens: Optional[Sequence[int]] = None,
             rows: Optional[np.ndarray] = None, nthreads: int = 0, lib=None):
    """Run the oracle.

    q: [tokens, Hq, d] (or [B, N, Hq, d]) bf16 bits; k, v: [tokens, Hkv, d].
    Without ``rows`` returns full-layout (o [tokens,Hq,d], lse, nvis) where lse
    and nvis are [B,Hq,N] (dense) or [Hq,tokens] (packed).  With ``rows`` (an
    int64 array of (sequence, head, row) triples) returns compact
    (o [n,d], lse [n], nvis [n]).
    """
    lib = lib or load()
    q, k, v = _bits(q), _bits(k), _bits(v)
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        tokens = int(cu[-1])
    else:
        tokens = B * N
    if rows is None:
        o = np.empty((tokens, Hq, d), dtype=np.float64)
        lse_shape = (Hq, tokens) if cu is not None else (B, Hq, N)
        lse = np.empty(lse_shape, dtype=np.float64)
        nvis = np.empty(lse_shape, dtype=np.int64)
        rows_p, nrows = None, 0
    else:
        rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1, 3))
        nrows = rows.shape[0]
        o = np.empty((nrows, d), dtype=np.float64)
        lse = np.empty((nrows,), dtype=np.float64)
        nvis = np.empty((nrows,), dtype=np.int64)
        rows_p = rows.ctypes.data
    rc = lib.oracle_attn_fwd(
        q.ctypes.data, k.ctypes.data, v.ctypes.data,
        o.ctypes.data, lse.ctypes.data, nvis.ctypes.data,
        B, Hq, Hkv, N, d, float(scale), int(bool(causal)), int(window_left), int(window_right),
        None if cu is None else cu.ctypes.data, rows_p, nrows, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd failed with code {rc}")
    return o, lse, nvis


def attn_kvcache(q, k_cache, v_cache, cache_seqlens, *, B: int, Hq: int, Hkv: int, Nq: int,
                 d: int, page_size: int, pages_per_seq: int, scale: float,
                 causal: bool = True, window_left: int = -1, window_right: int = -1,
                 block_table=None, nthreads: int = 0, lib=None):
    """Newest-token attention against a (paged) key/value cache.

    q [B, Nq, Hq, d] bf16 bits; caches [num_pages, page_size, Hkv, d] bf16 bits;
    cache_seqlens int32 [B]; block_table int32 [B, pages_per_seq] or None
    (contiguous cache).  Returns o [B, Nq, Hq, d] fp64, lse [B, Hq, Nq], nvis.
    """
    lib = lib or load()
    q, k_cache, v_cache = _bits(q), _bits(k_cache), _bits(v_cache)
    cs = np.ascontiguousarray(np.asarray(cache_seqlens, dtype=np.int32))
    bt = None if block_table is None else np.ascontiguousarray(np.asarray(block_table, dtype=np.int32))
    o = np.empty((B, Nq, Hq, d), dtype=np.float64)
    lse = np.empty((B, Hq, Nq), dtype=np.float64)
    nvis = np.empty((B, Hq, Nq), dtype=np.int64)
    rc = lib.oracle_attn_kvcache(q.ctypes.data, k_cache.ctypes.data, v_cache.ctypes.data,
                                 o.ctypes.data, lse.ctypes.data, nvis.ctypes.data, cs.ctypes.data,
                                 None if bt is None else bt.ctypes.data, B, Hq, Hkv, Nq, d,
                                 page_size, pages_per_seq, float(scale), int(bool(causal)),
                                 int(window_left), int(window_right), int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_kvcache failed with code {rc}")
    return o, lse, nvis


def attn_bwd(q, k, v, dout, *, B: int, Hq: int, Hkv: int, N: int, d: int, scale: float,
             causal: bool = False, window_left: int = -1, window_right: int = -1,
             cu_seqlens: Optional[Sequence[int]] = None, nthreads: int = 0, lib=None):
    """Gradients of sum(dout * O) with respect to q, k, v.

    q, dout [tokens, Hq, d] (or [B, N, Hq, d]) bf16 bits; k, v [tokens, Hkv, d].
    Returns fp64 (dq [tokens, Hq, d], dk [tokens, Hkv, d], dv [tokens, Hkv, d]).
    """
    lib = lib or load()
    q, k, v, dout = _bits(q), _bits(k), _bits(v), _bits(dout)
    cu = None
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
        tokens = int(cu[-1])
    else:
        tokens = B * N
    dq = np.empty((tokens, Hq, d), dtype=np.float64)
    dk = np.empty((tokens, Hkv, d), dtype=np.float64)
    dv = np.empty((tokens, Hkv, d), dtype=np.float64)
    rc = lib.oracle_attn_bwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, dout.ctypes.data,
                             dq.ctypes.data, dk.ctypes.data, dv.ctypes.data, B, Hq, Hkv, N, d,
                             float(scale), int(bool(causal)), int(window_left), int(window_right),
                             None if cu is None else cu.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd failed with code {rc}")
    return dq, dk, dv
