"""The C ABI library loads, exports every symbol include/attn.h declares, and
its host-side validation returns the documented codes.

Every call that passes made-up device addresses runs in a child process that
sees no GPU (CUDA_VISIBLE_DEVICES is empty): the checks under test return before
any CUDA call, and if one of them ever regressed the call could only fail to
find a device -- it can never launch a kernel on those addresses."""
import ctypes
import json
import os
import re
import subprocess
import sys

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
    for code in range(0, -12, -1):
        s = ea.attn_status_string(code)
        assert s and s != "unknown status", code
    assert ea.attn_status_string(-1234) == "unknown status"


FAKE = 1 << 20  # a 16-byte aligned made-up address, only ever passed with no GPU visible

_CHILD = r"""
import json, sys
sys.path.insert(0, sys.argv[1])
from exact_attention_142_b200 import _binding as b
calls = json.loads(sys.stdin.read())
print(json.dumps([getattr(b, fn)(check=False, **kw) for fn, kw in calls]))
"""


def run_without_gpu(calls):
    """[(binding function, kwargs)] -> return codes, from a child process in
    which no GPU is visible."""
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    res = subprocess.run([sys.executable, "-c", _CHILD, ROOT], input=json.dumps(calls),
                         capture_output=True, text=True, env=env, timeout=120)
    assert res.returncode == 0, res.stderr
    return json.loads(res.stdout.strip().splitlines()[-1])


def fwd_args(**over):
    args = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=4, Hkv=2, N=16, d=128,
                scale=0.1, causal=1, window_left=-1, window_right=-1, cu_seqlens=None,
                max_seqlen=0, stream=0)
    args.update(over)
    return args


FWD_CASES = [
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
]


def call_decode_args(**over):
    args = dict(q=FAKE, k_cache=FAKE, v_cache=FAKE, o=FAKE, lse=FAKE, cache_seqlens=FAKE,
                block_table=None, B=2, Hq=8, Hkv=2, Nq=1, d=128, page_size=16, pages_per_seq=8,
                num_pages=16, scale=0.1, causal=1, window_left=-1, window_right=-1, num_splits=1,
                workspace=None, workspace_bytes=0, stream=0)
    args.update(over)
    return args


DECODE_CASES = [
    (dict(B=0), ea.ATTN_ERR_SHAPE),
    (dict(Nq=0), ea.ATTN_ERR_SHAPE),
    (dict(Hq=6, Hkv=4), ea.ATTN_ERR_SHAPE),
    (dict(page_size=0), ea.ATTN_ERR_SHAPE),
    (dict(pages_per_seq=0), ea.ATTN_ERR_SHAPE),
    (dict(num_splits=0), ea.ATTN_ERR_SHAPE),
    (dict(page_size=1 << 20, pages_per_seq=1 << 12), ea.ATTN_ERR_SHAPE),  # > 2^31 keys
    (dict(num_pages=0), ea.ATTN_ERR_SHAPE),
    (dict(num_pages=15), ea.ATTN_ERR_SHAPE),              # contiguous cache needs B * pps pages
    (dict(num_pages=1 << 28, block_table=FAKE), ea.ATTN_ERR_SHAPE),  # rows overflow int32
    (dict(window_left=-3), ea.ATTN_ERR_WINDOW),
    (dict(d=80), ea.ATTN_ERR_UNSUPPORTED),
    (dict(Nq=17), ea.ATTN_ERR_UNSUPPORTED),
    (dict(scale=float("nan")), ea.ATTN_ERR_SCALE),
    (dict(cache_seqlens=None), ea.ATTN_ERR_NULL),
    (dict(v_cache=None), ea.ATTN_ERR_NULL),
    (dict(k_cache=FAKE + 4), ea.ATTN_ERR_ALIGN),
    (dict(lse=FAKE + 1), ea.ATTN_ERR_ALIGN),
    (dict(num_splits=4), ea.ATTN_ERR_WORKSPACE),          # 128 keys -> 2 slices, no workspace
    (dict(num_splits=4, workspace=FAKE, workspace_bytes=16), ea.ATTN_ERR_WORKSPACE),
    (dict(num_splits=4, workspace=FAKE + 16, workspace_bytes=1 << 20), ea.ATTN_ERR_WORKSPACE),
]


def _noalloc_args(**over):
    args = call_decode_args(**over)
    del args["workspace"], args["workspace_bytes"]
    return args


# attn_decode_noalloc: attn_decode's checks, then the size of its fixed array
# (256 sequences x 32 heads x 128 columns x 16 slices of fp32 partials: 64 MiB).
BIG = dict(B=256, Hq=32, Hkv=8, Nq=1, d=128, page_size=64, pages_per_seq=128, num_pages=256 * 128,
           num_splits=16)
NOALLOC_CASES = [
    (dict(BIG), ea.ATTN_ERR_WORKSPACE),
    (dict(BIG, q=None), ea.ATTN_ERR_NULL),
    (dict(BIG, d=80), ea.ATTN_ERR_UNSUPPORTED),
    (dict(num_splits=0), ea.ATTN_ERR_SHAPE),
]

HOST_CASES = [
    (dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, Hq=2, Hkv=2, N=16, d=64, scale=0.1,
          causal=True, window_left=-1, window_right=-1, cu_seqlens=None, max_seqlen=0,
          workspace=None, workspace_bytes=0, stream=0), ea.ATTN_ERR_WORKSPACE),
]

_ALL = ([("attn_fwd", fwd_args(**o), c) for o, c in FWD_CASES] +
        [("attn_decode", call_decode_args(**o), c) for o, c in DECODE_CASES] +
        [("attn_decode_noalloc", _noalloc_args(**o), c) for o, c in NOALLOC_CASES] +
        [("attn_fwd_host", kw, c) for kw, c in HOST_CASES])


@pytest.fixture(scope="module")
def no_gpu_codes(lib):
    return run_without_gpu([(fn, kw) for fn, kw, _ in _ALL])


@pytest.mark.parametrize("idx", range(len(_ALL)),
                         ids=[f"{fn}-{i}" for i, (fn, _, _) in enumerate(_ALL)])
def test_validation_codes(no_gpu_codes, idx):
    fn, kw, code = _ALL[idx]
    assert no_gpu_codes[idx] == code, (fn, kw)


def test_noalloc_scratch_size_matches_header(lib):
    text = open(os.path.join(ROOT, "include", "attn.h")).read()
    m = re.search(r"#define\s+ATTN_DECODE_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*\*\s*1024u\s*\*\s*1024u\)",
                  text)
    assert m, "ATTN_DECODE_NOALLOC_SCRATCH_BYTES not found in the header"
    assert ea.attn_decode_noalloc_scratch_bytes() == int(m.group(1)) * 1024 * 1024


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


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    from exact_attention_142_b200 import _binding
    monkeypatch.setattr(_binding, "_lib", None)
    monkeypatch.setattr(_binding, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="no fallback"):
        _binding.load_library()


def test_decode_workspace_size(lib):
    r = lambda x: (x + 255) // 256 * 256
    B, Hq, Hkv, Nq, d = 3, 16, 4, 2, 128
    # 1000 keys in 4 slices -> 256 keys per slice (a multiple of the 64-key tile) -> 4 slices
    got = ea.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, 100, 10, 4)
    rows = B * Nq * Hq
    assert got == r(4 * rows * d * 4) + r(4 * rows * 4)
    # 7 slices of 1000 keys -> ceil(143 / 64) * 64 = 192 keys -> 6 slices
    assert ea.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, 100, 10, 7) == \
        r(6 * rows * d * 4) + r(6 * rows * 4)
    assert ea.attn_decode_workspace_bytes(B, Hq, Hkv, Nq, d, 100, 10, 1) == 0
    assert ea.attn_decode_workspace_bytes(0, Hq, Hkv, Nq, d, 100, 10, 4) == 0


def test_decode_default_splits(lib):
    # no device here: 148 SMs x 2 CTAs = 296 slots
    # 64 sequences x 8 kv heads = 512 CTAs: 1.73 waves, last wave 216 >= 148 -> 1 slice
    assert ea.attn_decode_default_splits(64, 32, 8, 1, 8192) == 1
    # one sequence, 8 kv heads: 19 slices = 152 CTAs >= 148 slots
    assert ea.attn_decode_default_splits(1, 32, 8, 1, 8192) == 19
    # a short cache caps the slices (>= 256 keys each)
    assert ea.attn_decode_default_splits(1, 32, 8, 1, 300) == 1
    assert ea.attn_decode_default_splits(1, 32, 8, 1, 2048) == 8
    # 300 CTAs: last waves of 4, 8, 12 CTAs are too small; 4 slices = 4.05 waves
    assert ea.attn_decode_default_splits(75, 32, 4, 1, 8192) == 4
    assert ea.attn_decode_default_splits(0, 32, 8, 1, 8192) == 1
