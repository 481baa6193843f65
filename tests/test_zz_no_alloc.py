"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Such callers (a plugin in a process that owns all device memory, a C caller
without access to the allocator behind its buffers) cannot supply the
split-KV workspace pa_decode asks for; pa_decode_noalloc uses a fixed array
inside the library instead.  These tests call it through the C ABI and check
it against pa_decode with a caller-provided workspace and against the oracle,
on calls in a row of different sizes (a later call must not depend on what an
earlier one left in the shared array): explicit chunk sizes, the automatic
chunk choice on a long-context shape, and a shape that needs no scratch at
all (the library then passes no scratch pointer).  The file sorts last so
that a run stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from paged_kv_cache_331_b200._binding import lib
from gpu_helpers import DeviceDecode, MAX_ABS, MEAN_ABS, assert_attention_close, host_f32

pytestmark = pytest.mark.gpu

SCRATCH_LIMIT = 8 << 20   # PA_DECODE_NOALLOC_SCRATCH_BYTES in include/pa.h


def raw_noalloc(dw, out, chunk):
    """Direct C-ABI call (ctypes), the way a C caller would make it."""
    w = dw.w
    return lib().pa_decode_noalloc(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(dw.q.data_ptr()), ctypes.c_void_p(dw.k_cache.data_ptr()),
        ctypes.c_void_p(dw.v_cache.data_ptr()), ctypes.c_void_p(dw.block_tables.data_ptr()),
        w.max_blocks_per_seq, ctypes.c_void_p(dw.context_lens.data_ptr()), w.max_context_len, w.num_seqs,
        w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks, ctypes.c_float(w.scale), chunk,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def check_close(a, b):
    x, y = host_f32(a).astype(np.float64), host_f32(b).astype(np.float64)
    assert np.isfinite(x).all()
    err = np.abs(x - y)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (err.max(), err.mean())


def check_oracle(oracle, out, w):
    """The new rows are stored in both caches first (as the device workload was), then the oracle decodes."""
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    oracle.store_kvcache(w.new_k, w.new_v, kc, vc, w.slot_mapping)
    _, ref = oracle.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what=f"decode_noalloc {w.context_lens.tolist()}")


def workload(seed, lens, hq, hkv, d, bs):
    w = W.decode_workload(np.array(lens, np.int32), hq, hkv, d, bs, rng=np.random.default_rng(seed))
    dw = DeviceDecode(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    return dw


def run_cases(oracle, cases):
    for dw, chunk, expect_scratch in cases:
        w = dw.w
        need = pa.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, w.max_context_len,
                                        w.block_size, chunk)
        assert need <= SCRATCH_LIMIT and (need > 0) == expect_scratch
        ref = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, w.max_context_len, w.scale,
                        kv_chunk_size=chunk)
        out = torch.full_like(dw.q, float("nan"))
        assert raw_noalloc(dw, out, chunk) == 0, lib().pa_last_error()
        torch.cuda.synchronize()
        check_close(out, ref)
        check_oracle(oracle, out, w)
    assert pa.device_error() == 0


def test_noalloc_matches_workspace_decode_on_two_calls_in_a_row(oracle):
    # first call: long sequences split into many chunks; second: a different, smaller shape
    run_cases(oracle, [(workload(71, [3000, 1, 1700, 2048, 640], 16, 4, 128, 256), 256, True),
                       (workload(72, [90, 700, 33], 8, 2, 64, 16), 64, True)])


def test_noalloc_automatic_chunk_then_no_scratch(oracle):
    # kv_chunk_size 0 on a long-context shape (few sequences, so the automatic choice splits them: the library
    # sizes the scratch and the launch with the same choice), then a short batch that needs no split, where no
    # scratch pointer is passed at all
    run_cases(oracle, [(workload(74, [16384, 1, 16384], 32, 8, 128, 256), 0, True),
                       (workload(75, [300, 17, 512, 64], 16, 8, 128, 256), 0, False)])


def test_noalloc_rejects_shapes_beyond_its_scratch():
    dw = workload(73, [40, 17], 4, 2, 64, 16)
    w = dw.w
    # a claimed max context of 1M tokens with 64-token chunks needs far more than the fixed scratch
    need = pa.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, 1 << 20, w.block_size, 64)
    assert need > SCRATCH_LIMIT
    out = torch.zeros_like(dw.q)
    st = lib().pa_decode_noalloc(
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(dw.q.data_ptr()), ctypes.c_void_p(dw.k_cache.data_ptr()),
        ctypes.c_void_p(dw.v_cache.data_ptr()), ctypes.c_void_p(dw.block_tables.data_ptr()), w.max_blocks_per_seq,
        ctypes.c_void_p(dw.context_lens.data_ptr()), 1 << 20, w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim,
        w.block_size, w.num_blocks, ctypes.c_float(w.scale), 64, ctypes.c_void_p(0))
    assert st == 4   # PA_ERR_WORKSPACE
    assert b"static array" in lib().pa_last_error()
    torch.cuda.synchronize()
    assert not out.any()   # nothing was launched
