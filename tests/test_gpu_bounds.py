"""Contract violations found on the device: each access that would leave the
caller's buffers is skipped (or clamped) and a code is recorded in the
library's device error word.

Every case runs on valid memory only.  The cache (or output) the call is given
is a view into a larger allocation whose extra blocks (rows) hold a sentinel,
placed where an unchecked access would land; the test checks that the
sentinel survives, that the code is the documented one and that the rest of
the call's results are still right.  A last test makes one bounded pipeline
wait run out (nothing arrives on its barrier) and checks that it returns with
code 1 and that later launches are unaffected.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DeviceDecode, DevicePrefill, assert_attention_close, dev_bf16, dev_i32

pytestmark = pytest.mark.gpu

SENTINEL = 0x7F7F   # a bf16 bit pattern no store in these tests writes


def padded_cache(host_cache, lead, tail):
    """The cache on the device inside an allocation with `lead` spare blocks before it and `tail` after it, all
    holding SENTINEL; returns (full allocation, view of the real cache)."""
    nb = host_cache.shape[0]
    full = torch.full((lead + nb + tail,) + host_cache.shape[1:], SENTINEL, dtype=torch.int16, device="cuda")
    full[lead:lead + nb] = torch.from_numpy(host_cache.view(np.int16)).cuda()
    full = full.view(torch.bfloat16)
    return full, full[lead:lead + nb]


def sentinel_intact(full, lead, nb):
    bits = full.view(torch.int16)
    return bool((bits[:lead] == SENTINEL).all()) and bool((bits[lead + nb:] == SENTINEL).all())


def test_store_kvcache_reports_slots_outside_the_cache():
    rng = np.random.default_rng(501)
    w = W.decode_workload(np.array([40, 17, 9], np.int32), 4, 2, 64, 16, rng=rng)
    nb, bs = w.num_blocks, w.block_size
    fk, kc = padded_cache(w.k_cache, 1, 2)
    fv, vc = padded_cache(w.v_cache, 1, 2)
    slots = w.slot_mapping.copy()
    slots[1] = nb * bs + 7        # would land in the first spare block after the cache
    slots[2] = -5                 # would land in the spare block before it
    pa.device_error()
    pa.store_kvcache(dev_bf16(w.new_k), dev_bf16(w.new_v), kc, vc, dev_i32(slots))
    torch.cuda.synchronize()
    assert pa.device_error() == 6
    assert sentinel_intact(fk, 1, nb) and sentinel_intact(fv, 1, nb)
    s0 = int(slots[0])            # the valid row was stored
    assert torch.equal(kc.view(-1, 2, 64)[s0].view(torch.int16), dev_bf16(w.new_k)[0].view(torch.int16))
    # -1 stays a silent skip
    slots[1:] = -1
    pa.store_kvcache(dev_bf16(w.new_k), dev_bf16(w.new_v), kc, vc, dev_i32(slots))
    assert pa.device_error() == 0


def test_rotary_store_reports_slots_outside_the_cache(oracle):
    rng = np.random.default_rng(502)
    w = W.decode_workload(np.array([40, 17], np.int32), 8, 2, 128, 16, rng=rng)
    nb, bs = w.num_blocks, w.block_size
    fk, kc = padded_cache(w.k_cache, 1, 1)
    fv, vc = padded_cache(w.v_cache, 1, 1)
    slots = w.slot_mapping.copy()
    slots[0] = nb * bs + 3
    table = pa.rotary_cos_sin_cache(64, 128, 1e4)
    pos = dev_i32(w.context_lens - 1)
    pa.device_error()
    q_rot = pa.rotary_store_kvcache(dev_bf16(w.q), dev_bf16(w.new_k), dev_bf16(w.new_v), pos, table, kc, vc,
                                    dev_i32(slots))
    torch.cuda.synchronize()
    assert pa.device_error() == 6
    assert sentinel_intact(fk, 1, nb) and sentinel_intact(fv, 1, nb)
    assert torch.isfinite(q_rot.float()).all()   # the query rows of both tokens were still rotated


def test_store_decode_reports_a_table_entry_outside_the_cache(oracle):
    rng = np.random.default_rng(503)
    w = W.decode_workload(np.array([40, 17], np.int32), 4, 2, 64, 16, rng=rng)
    nb, bs = w.num_blocks, w.block_size
    fk, kc = padded_cache(w.k_cache, 0, 2)
    fv, vc = padded_cache(w.v_cache, 0, 2)
    tables = w.block_tables.copy()
    slots = w.slot_mapping.copy()
    tables[0, (40 - 1) // bs] = nb              # sequence 0's newest position now points past the cache ...
    slots[0] = nb * bs + (40 - 1) % bs          # ... and its slot agrees with the table
    dw = DeviceDecode(w)
    pa.device_error()
    out = pa.store_decode(dw.q, dw.new_k, dw.new_v, dev_i32(slots), kc, vc, dev_i32(tables), dw.context_lens, 40,
                          w.scale)
    torch.cuda.synchronize()
    assert pa.device_error() == 6
    assert sentinel_intact(fk, 0, nb) and sentinel_intact(fv, 0, nb)
    # sequence 1 is untouched by the violation: its row stored, its output right
    s1 = int(slots[1])
    assert torch.equal(kc.view(-1, 2, 64)[s1].view(torch.int16), dw.new_k[1].view(torch.int16))
    oracle.store_kvcache(w.new_k[1:], w.new_v[1:], w.k_cache, w.v_cache, w.slot_mapping[1:])
    _, ref = oracle.decode(w.q[1:], w.k_cache, w.v_cache, w.block_tables[1:], w.context_lens[1:], w.scale,
                           want_f64=True)
    assert_attention_close(out[1:], ref, what="store_decode, the valid sequence")


@pytest.mark.parametrize("kind", ["above_max_context_len", "beyond_the_table"])
def test_decode_clamps_and_reports_context_lengths(oracle, kind):
    rng = np.random.default_rng(504)
    w = W.decode_workload(np.array([300, 17], np.int32), 8, 2, 128, 16, rng=rng)
    dw = DeviceDecode(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    lens = w.context_lens.copy()
    width = w.block_tables.shape[1] * w.block_size
    if kind == "above_max_context_len":
        max_len, clamped = 200, 200              # the context of 300 is above the max the call states
    else:
        lens[0] = width + 100                    # more keys than the table row holds blocks for
        max_len, clamped = int(lens[0]), width
    pa.device_error()
    out = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dev_i32(lens), max_len, w.scale,
                    kv_chunk_size=64)
    torch.cuda.synchronize()
    assert pa.device_error() == 7
    ref_lens = np.array([clamped, 17], np.int32)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, ref_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what=f"decode with a clamped context ({kind})")


def prefill_case(seed, prefix, sfx, hq=8, hkv=2, d=128, bs=16):
    w = W.prefill_workload(prefix, np.array(sfx, np.int32), hq, hkv, d, bs, rng=np.random.default_rng(seed))
    dw = DevicePrefill(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    oracle_store = (w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    return w, dw, oracle_store


def oracle_rows(oracle, w, store):
    oracle.store_kvcache(*store)
    _, ref = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                   w.scale, w.causal, want_f64=True)
    return ref


def rows_of(w, seqs):
    m = np.zeros(int(w.cu_seqlens_q[-1]), bool)
    for b in seqs:
        m[w.cu_seqlens_q[b]:w.cu_seqlens_q[b + 1]] = True
    return m


def test_prefill_skips_a_sequence_past_total_q(oracle):
    w, dw, store = prefill_case(505, 32, [20, 30, 25])
    T = int(w.cu_seqlens_q[-1])                # 75 rows; the call is told there are 60
    short = 60
    out_full = torch.full((T, w.num_heads, w.head_dim), SENTINEL, dtype=torch.int16, device="cuda")
    out_full = out_full.view(torch.bfloat16)
    pa.device_error()
    pa.prefill_varlen(dw.q[:short], dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                      w.max_seqlen_k, dw.block_tables, w.scale, True, out=out_full[:short])
    torch.cuda.synchronize()
    assert pa.device_error() == 8
    bits = out_full.view(torch.int16)
    assert bool((bits[int(w.cu_seqlens_q[2]):] == SENTINEL).all())   # sequence 2 was skipped whole
    ref = oracle_rows(oracle, w, store)
    keep = rows_of(w, [0, 1])
    assert_attention_close(out_full[:int(w.cu_seqlens_q[2])], ref[keep], what="prefill, the sequences inside total_q")


def test_prefill_skips_a_sequence_beyond_its_table_row(oracle):
    w, dw, store = prefill_case(506, 32, [60, 5, 10])
    width = w.block_tables.shape[1]
    assert -(-int(w.cu_seqlens_k[1]) // w.block_size) == width      # only sequence 0 needs the full width
    narrow = dev_i32(np.ascontiguousarray(w.block_tables[:, :width - 1]))
    out = torch.full_like(dw.q.view(torch.int16), SENTINEL).view(torch.bfloat16)
    pa.device_error()
    pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q, w.max_seqlen_k,
                      narrow, w.scale, True, out=out)
    torch.cuda.synchronize()
    assert pa.device_error() == 8
    assert bool((out[:int(w.cu_seqlens_q[1])].view(torch.int16) == SENTINEL).all())
    ref = oracle_rows(oracle, w, store)
    keep = rows_of(w, [1, 2])
    assert_attention_close(out[torch.from_numpy(keep).cuda()], ref[keep], what="prefill, sequences within the table")


def test_prefill_reports_a_table_entry_outside_the_cache(oracle):
    w, dw, store = prefill_case(507, 32, [20, 30, 25])
    tables = w.block_tables.copy()
    tables[1, 1] = w.num_blocks + 3             # sequence 1's second prefix block (the others keep the real one)
    pa.device_error()
    out = pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                            w.max_seqlen_k, dev_i32(tables), w.scale, True)
    torch.cuda.synchronize()
    assert pa.device_error() == 6
    ref = oracle_rows(oracle, w, store)
    keep = rows_of(w, [0, 2])
    assert_attention_close(out[torch.from_numpy(keep).cuda()], ref[keep], what="prefill, the other sequences")


def test_bounded_wait_runs_out_and_reports(oracle):
    """One CTA waits on an mbarrier nothing arrives on, with a 2 ms limit: the launch returns, code 1 is
    recorded (and cleared by the read), and the kernels launched after it run normally."""
    pa.device_error()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    pa.selftest_wait_timeout(2_000_000)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b)
    assert 2.0 <= ms < 1000.0, ms
    assert pa.device_error() == 1
    assert pa.device_error() == 0
    # the device is still usable: a prefill (which allocates all of an SM's tensor memory) and a decode
    w, dw, store = prefill_case(508, 32, [20, 30])
    out = pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                            w.max_seqlen_k, dw.block_tables, w.scale, True)
    torch.cuda.synchronize()
    assert_attention_close(out, oracle_rows(oracle, w, store), what="prefill after the timed-out wait")
    assert pa.device_error() == 0


def test_selftest_rejects_limits_out_of_range():
    for bad in (0, 999, 2_000_000_000):
        with pytest.raises(pa.PagedAttentionError):
            pa.selftest_wait_timeout(bad)
