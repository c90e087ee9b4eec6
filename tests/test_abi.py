"""The C ABI library loads, exports every symbol include/attn.h declares, and
its host-side validation returns the documented codes (no GPU needed: these
calls return before any CUDA call)."""
import ctypes
import os
import re

import pytest

import exact_attention_142_b200 as ea
from exact_attention_142_b200 import build as ea_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ea_build.build()
    return ea.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("attn_fwd", "attn_status_string", "attn_device_status"):
        assert required in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"{name} missing from {ea.library_path()}"


def test_status_strings(lib):
    for code in range(0, -10, -1):
        s = ea.attn_status_string(code)
        assert s and s != "unknown status", code
    assert ea.attn_status_string(-1234) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned fake address; validation rejects before use


def call(**over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, N=16, d=128,
                scale=0.1, causal=1, window_left=-1, window_right=-1, cu_seqlens=None,
                max_seqlen=0, stream=0)
    args.update(over)
    return ea.attn_fwd(check=False, **args)


@pytest.mark.parametrize("over,code", [
    (dict(B=0), ea.ATTN_ERR_SHAPE),
    (dict(Hq=0), ea.ATTN_ERR_SHAPE),
    (dict(Hkv=0), ea.ATTN_ERR_SHAPE),
    (dict(N=-1), ea.ATTN_ERR_SHAPE),
    (dict(Hq=6, Hkv=4), ea.ATTN_ERR_SHAPE),
    (dict(window_left=-2), ea.ATTN_ERR_WINDOW),
    (dict(window_right=-7), ea.ATTN_ERR_WINDOW),
    (dict(d=96), ea.ATTN_ERR_UNSUPPORTED),
    (dict(d=256), ea.ATTN_ERR_UNSUPPORTED),
    (dict(scale=0.0), ea.ATTN_ERR_SCALE),
    (dict(scale=-1.0), ea.ATTN_ERR_SCALE),
    (dict(scale=float("nan")), ea.ATTN_ERR_SCALE),
    (dict(scale=float("inf")), ea.ATTN_ERR_SCALE),
    (dict(q=None), ea.ATTN_ERR_NULL),
    (dict(lse=None), ea.ATTN_ERR_NULL),
    (dict(q=FAKE + 8), ea.ATTN_ERR_ALIGN),
    (dict(o=FAKE + 2), ea.ATTN_ERR_ALIGN),
    (dict(lse=FAKE + 2), ea.ATTN_ERR_ALIGN),
    (dict(B=70000, N=40000), ea.ATTN_ERR_SHAPE),  # tokens overflow 32-bit coordinates
    (dict(cu_seqlens=FAKE, N=10, max_seqlen=0), ea.ATTN_ERR_SHAPE),
    (dict(N=0), ea.ATTN_OK),                      # nothing to do, nothing enqueued
    (dict(N=0, q=None, k=None, v=None, o=None, lse=None), ea.ATTN_OK),
])
def test_validation_codes(lib, over, code):
    assert call(**over) == code


def test_host_workspace_size(lib):
    B, Hq, Hkv, N, d = 2, 8, 2, 100, 64
    got = ea.attn_fwd_host_workspace_bytes(B, Hq, Hkv, N, d, False)
    r = lambda x: (x + 255) // 256 * 256
    tokens = B * N
    want = r(tokens * Hq * d * 2) * 2 + 2 * r(tokens * Hkv * d * 2) + r(tokens * Hq * 4)
    assert got == want
    assert ea.attn_fwd_host_workspace_bytes(3, Hq, Hkv, 300, d, True) == \
        2 * r(300 * Hq * d * 2) + 2 * r(300 * Hkv * d * 2) + r(300 * Hq * 4) + r(4 * 4)
    assert ea.attn_fwd_host_workspace_bytes(0, Hq, Hkv, N, d, False) == 0


def test_host_entry_rejects_missing_workspace(lib):
    rc = ea.attn_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 2, 2, 16, 64, 0.1, True, -1, -1,
                          None, 0, None, 0, stream=0, check=False)
    assert rc == ea.ATTN_ERR_WORKSPACE


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from exact_attention_142_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        _binding.load_library()
