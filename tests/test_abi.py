"""The C-ABI library loads on a machine without a GPU, exports every function
that include/*.h declares, and rejects bad arguments on the host before any
launch (no compute calls here)."""
import ctypes
import re
import subprocess
from pathlib import Path

import pytest

ROOT = Path(__file__).resolve().parent.parent
HEADERS = sorted((ROOT / "include").glob("*.h"))


@pytest.fixture(scope="module")
def libpa():
    from paged_kv_cache_331_b200 import build as B
    B.build()
    from paged_kv_cache_331_b200 import _binding
    return _binding.lib()


def declared_functions():
    names = set()
    for h in HEADERS:
        text = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names |= set(re.findall(r"\b(pa_[a-z_0-9]+)\s*\(", text))
    return sorted(names)


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("pa_store_kvcache", "pa_decode", "pa_decode_workspace_size", "pa_prefill_varlen",
                     "pa_rotary_store_kvcache", "pa_bm_allocate", "pa_bm_may_append", "pa_bm_prepare_prefill"):
        assert required in names


def test_library_exports_every_declared_symbol(libpa):
    so = ROOT / "paged_kv_cache_331_b200" / "libpagedattn.so"
    out = subprocess.run(["nm", "-D", "--defined-only", str(so)], capture_output=True, text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    for n in declared_functions():
        assert hasattr(libpa, n)
    # nothing else of ours leaks out of the library
    ours = sorted(n for n in exported if n.startswith("pa_") or "pa::" in n)
    assert set(ours) <= set(declared_functions())


def test_status_strings(libpa):
    assert libpa.pa_status_string(0) == b"PA_OK"
    assert libpa.pa_status_string(1) == b"PA_ERR_INVALID_ARG"
    assert libpa.pa_status_string(4) == b"PA_ERR_WORKSPACE"
    assert libpa.pa_version() >> 16 == 1


def test_host_side_argument_checks(libpa):
    L = libpa
    null = None
    # store: negative token count, short row stride
    assert L.pa_store_kvcache(null, null, 64, 64, null, null, null, -1, 1, 64, 16, 4, null) == 1
    assert L.pa_store_kvcache(null, null, 10, 64, null, null, null, 1, 1, 64, 16, 4, null) == 1
    assert L.pa_store_kvcache(null, null, 64, 64, null, null, null, 0, 1, 64, 16, 4, null) == 0   # nothing to do
    # decode: group size, head_dim, block size, chunk size
    args = lambda hq, hkv, d, bs, chunk: (null, null, null, null, null, 4, null, 100, 2, hq, hkv, d, bs, 8, 0.125,
                                          chunk, null, 0, null)
    assert L.pa_decode(*args(6, 4, 64, 16, 0)) == 1          # 6 % 4 != 0
    assert L.pa_decode(*args(4, 2, 96, 16, 0)) == 2          # head_dim 96 unsupported
    assert L.pa_decode(*args(4, 2, 64, 48, 0)) == 2          # block_size not a power of two
    assert L.pa_decode(*args(4, 2, 64, 16, 100)) == 1        # chunk not a multiple of 64
    assert L.pa_decode(*args(4, 2, 64, 16, 64)) == 1         # null pointers
    assert b"null" in L.pa_last_error()
    # prefill: unsupported group size, inconsistent max lengths
    pargs = lambda hq, hkv, mq, mk: (null, null, null, null, null, null, 10, mq, mk, null, 4, 2, hq, hkv, 64, 16, 8,
                                     0.125, 1, null)
    assert L.pa_prefill_varlen(*pargs(6, 2, 8, 8)) == 2      # G = 3
    assert L.pa_prefill_varlen(*pargs(4, 2, 9, 8)) == 1      # max_seqlen_q > max_seqlen_k


def test_workspace_size_arithmetic(libpa):
    """Explicit chunk size: partial (acc, m, l) rows for every (seq, head, chunk)."""
    B, H, Hkv, D = 3, 8, 2, 128
    n = libpa.pa_decode_workspace_size(B, H, Hkv, D, 1000, 16, 256)
    chunks = 4
    rows = B * H * chunks
    assert n == (rows * D * 4 + 255) // 256 * 256 + rows * 2 * 4
    assert libpa.pa_decode_workspace_size(B, H, Hkv, D, 256, 16, 256) == 0     # one chunk: no workspace
    assert libpa.pa_decode_workspace_size(B, H, Hkv, D, 1000, 16, 100) == 0    # invalid chunk -> 0


def test_more_rejections_before_any_launch(libpa):
    """Each call breaks one rule of its entry point and is refused with that rule's status, before any launch:
    1 = PA_ERR_INVALID_ARG, 2 = PA_ERR_UNSUPPORTED."""
    L, null = libpa, None
    mis = 0x1003                                             # a misaligned (never dereferenced) address
    # store_kvcache: a non-positive size, a row too long for the kernel
    assert L.pa_store_kvcache(null, null, 64, 64, null, null, null, 1, 0, 64, 16, 4, null) == 1
    assert L.pa_store_kvcache(null, null, 1 << 21, 1 << 21, null, null, null, 1, 2048, 1024, 16, 4, null) == 2
    # rotary table: null table, odd head_dim, base <= 1
    assert L.pa_rotary_cos_sin_cache(null, 16, 64, 1e4, null) == 1
    assert L.pa_rotary_cos_sin_cache(mis, 16, 63, 1e4, null) == 1
    assert L.pa_rotary_cos_sin_cache(mis, 16, 64, 1.0, null) == 1

    # rotary store: head_dim, head count, short q stride, null pointers, misaligned pointers
    def rot(d=64, hq=4, hkv=2, q_stride=None, ptr=null, n=3):
        qs = q_stride if q_stride is not None else hq * d
        return L.pa_rotary_store_kvcache(ptr, ptr, qs, ptr, ptr, hkv * d, hkv * d, ptr, ptr, 16, ptr, ptr, ptr, n,
                                         hq, hkv, d, 16, 4, null)
    assert rot(d=96) == 2
    assert rot(hq=8192) == 2
    assert rot(q_stride=10) == 1
    assert rot() == 1                                        # null pointers
    assert rot(ptr=mis) == 2                                 # 16-byte alignment
    assert rot(n=0) == 0                                     # nothing to do

    # decode: scale, negative context bound, table width
    dargs = lambda scale=0.125, maxL=100, mb=4: (null, null, null, null, null, mb, null, maxL, 2, 4, 2, 64, 16, 8,
                                                 scale, 0, null, 0, null)
    assert L.pa_decode(*dargs(scale=0.0)) == 1
    assert L.pa_decode(*dargs(scale=float("nan"))) == 1
    assert L.pa_decode(*dargs(maxL=-1)) == 1
    assert L.pa_decode(*dargs(mb=0)) == 1

    # prefill: negative counts, scale, table width
    pargs = lambda ns=4, tq=10, scale=0.125, mb=4: (null, null, null, null, null, null, tq, 8, 8, null, mb, ns, 4, 2,
                                                    64, 16, 8, scale, 1, null)
    assert L.pa_prefill_varlen(*pargs(ns=-1)) == 1
    assert L.pa_prefill_varlen(*pargs(tq=-1)) == 1
    assert L.pa_prefill_varlen(*pargs(scale=-1.0)) == 1
    assert L.pa_prefill_varlen(*pargs(mb=0)) == 1
    assert L.pa_prefill_varlen(*pargs(tq=0)) == 0            # no query rows: nothing to do

    # merge_partials: no partials, head_dim, null and misaligned pointers
    assert L.pa_merge_partials(null, null, null, 0, 4, 64, null) == 1
    assert L.pa_merge_partials(null, null, null, 2, 4, 96, null) == 2
    assert L.pa_merge_partials(null, null, null, 2, 4, 64, null) == 1
    assert L.pa_merge_partials(mis, mis, mis, 2, 4, 64, null) == 1
    assert L.pa_merge_partials(null, null, null, 2, 0, 64, null) == 0

    assert L.pa_status_string(99) == b"PA_ERR_UNKNOWN"
