"""pa_store_decode (store of the new token + decode in one launch) and the
split-KV merge done by the last chunk's CTA, against the separate calls and the
oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DeviceDecode, assert_attention_close, dev_i32, host_bits

pytestmark = pytest.mark.gpu

CASES = [  # lens, hq, hkv, d, bs, kv_chunk_size
    ([1, 17, 256, 300], 4, 2, 64, 256, 0),
    ([5, 33, 64, 1, 100, 0, 129], 8, 2, 128, 16, 64),
    ([3000, 2500, 1], 16, 8, 128, 256, 512),
    ([700, 1], 5, 1, 64, 64, 128),
]


@pytest.mark.parametrize("lens,hq,hkv,d,bs,chunk", CASES)
def test_store_decode_equals_store_then_decode(oracle, lens, hq, hkv, d, bs, chunk):
    rng = np.random.default_rng(sum(lens) + hq)
    w = W.decode_workload(np.array(lens, np.int32), hq, hkv, d, bs, rng=rng)
    a, b = DeviceDecode(w), DeviceDecode(w)
    L = int(max(lens))
    out_f = pa.store_decode(a.q, a.new_k, a.new_v, a.slot_mapping, a.k_cache, a.v_cache, a.block_tables,
                            a.context_lens, L, w.scale, kv_chunk_size=chunk)
    pa.store_kvcache(b.new_k, b.new_v, b.k_cache, b.v_cache, b.slot_mapping)
    out_s = pa.decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, L, w.scale, kv_chunk_size=chunk)
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(a.v_cache.view(torch.int16), b.v_cache.view(torch.int16))
    assert torch.equal(out_f.view(torch.int16), out_s.view(torch.int16))
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out_f, ref, what="store_decode")


def test_store_decode_rejects_a_foreign_slot():
    rng = np.random.default_rng(3)
    w = W.decode_workload(np.array([40, 17], np.int32), 4, 2, 64, 16, rng=rng)
    dw = DeviceDecode(w)
    before = dw.k_cache.clone()
    bad = w.slot_mapping.copy()
    other = int(w.block_tables[1, 0]) * 16 + 3                # a slot of the other sequence
    bad[0] = other
    pa.device_error()
    pa.store_decode(dw.q, dw.new_k, dw.new_v, dev_i32(bad), dw.k_cache, dw.v_cache, dw.block_tables,
                    dw.context_lens, 40, w.scale)
    assert pa.device_error() == 5
    flat_before, flat_after = before.view(-1, 2, 64), dw.k_cache.view(-1, 2, 64)
    assert torch.equal(flat_after[other].view(torch.int16), flat_before[other].view(torch.int16))
    # sequence 1's own slot was stored
    assert torch.equal(flat_after[int(w.slot_mapping[1])].view(torch.int16), dw.new_k[1].view(torch.int16))


def test_in_kernel_merge_is_repeatable():
    """Back-to-back split launches (each uses a merge-counter slot that the last CTA resets) stay identical."""
    rng = np.random.default_rng(4)
    w = W.decode_workload(rng.integers(1, 4000, 24).astype(np.int32), 16, 8, 128, 256, rng=rng)
    dw = DeviceDecode(w)
    ref = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 4000, w.scale, kv_chunk_size=256)
    outs = [pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 4000, w.scale,
                      kv_chunk_size=256) for _ in range(40)]
    torch.cuda.synchronize()
    for o in outs:
        assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    assert pa.device_error() == 0


def test_merge_kernel_path_above_the_counter_capacity(oracle):
    """16 400 (sequence, kv head) pairs exceed the in-kernel merge's counters: the separate merge kernel runs."""
    rng = np.random.default_rng(5)
    B = 4100
    lens = rng.integers(1, 200, B).astype(np.int32)
    w = W.decode_workload(lens, 4, 4, 64, 16, rng=rng)
    dw = DeviceDecode(w)
    out = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 200, w.scale, kv_chunk_size=64)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    torch.cuda.synchronize()
    assert_attention_close(out, ref, what="merge-kernel path")
    assert pa.device_error() == 0
