"""Varlen causal prefill with prefix-cache blocks on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DevicePrefill, assert_attention_close, host_bits

pytestmark = pytest.mark.gpu


def store_and_prefill(dp):
    w = dp.w
    pa.store_kvcache(dp.new_k, dp.new_v, dp.k_cache, dp.v_cache, dp.slot_mapping)
    out = pa.prefill_varlen(dp.q, dp.k_cache, dp.v_cache, dp.cu_seqlens_q, dp.cu_seqlens_k, w.max_seqlen_q,
                            w.max_seqlen_k, dp.block_tables, w.scale, w.causal)
    torch.cuda.synchronize()
    return out


def oracle_prefill(oracle, w, row_select=None):
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, of = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables, w.scale,
                                  w.causal, row_select=row_select, want_f64=True)
    return of


CASES = [
    # prefix, suffixes, hq, hkv, d, bs, causal
    (0, [5, 17, 1], 4, 2, 64, 16, True),
    (0, [128, 129, 300], 2, 1, 128, 256, True),
    (256, [64, 1, 200], 16, 8, 128, 256, True),
    (32, [9, 20, 150], 4, 1, 128, 16, True),
    (64, [40, 3, 130], 8, 1, 64, 32, True),
    (128, [77, 255], 8, 8, 128, 128, True),
    (512, [300, 64], 16, 2, 128, 64, True),
    (32, [9, 20], 4, 4, 64, 16, False),
    (256, [100, 257], 8, 2, 128, 256, False),
    (512, [100, 40], 8, 2, 128, 512, True),
    (0, [700, 3], 4, 4, 64, 1024, True),
]


@pytest.mark.parametrize("prefix,sfx,hq,hkv,d,bs,causal", CASES)
def test_prefill_small_shapes(oracle, prefix, sfx, hq, hkv, d, bs, causal):
    rng = np.random.default_rng(prefix + sum(sfx) + hq + d + bs)
    w = W.prefill_workload(prefix, np.array(sfx, np.int32), hq, hkv, d, bs, rng=rng, causal=causal)
    out = store_and_prefill(DevicePrefill(w))
    ref = oracle_prefill(oracle, w)
    assert_attention_close(out, ref, what=f"prefill prefix={prefix} sfx={sfx} G={hq // hkv} D={d} bs={bs}")


def lone_tiles(w, causal=True):
    """Lone query tiles that see two key tiles or more, as (sequence, key tiles,
    rows that see no key past the first key tile).  The kernel pairs a
    sequence's 128-row query tiles (G heads x 128/G positions) into work items;
    with an odd count the sequence's last tile runs alone."""
    G = w.num_heads // w.num_kv_heads
    qp = 128 // G
    out = []
    for b in range(w.num_seqs):
        lq = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        lk = int(w.cu_seqlens_k[b + 1] - w.cu_seqlens_k[b])
        ntq = -(-lq // qp)
        if ntq % 2 == 0:
            continue
        qt = ntq - 1
        pos = [lk - lq + i for i in range(qt * qp, lq)]
        nkeys = min(lk, pos[-1] + 1) if causal else lk
        nt = -(-nkeys // 128)
        if nt >= 2:
            out.append((b, nt, sum(1 for p_ in pos if causal and p_ < 128)))
    return out


LONE_CASES = [
    # prefix, suffixes, hq, hkv, d, bs, causal: every case has a lone query tile over two key tiles or more
    (96, [50], 4, 2, 128, 32, True),                # 2 key tiles; rows at positions < 128 see none of tile 1
    (96, [50, 30, 64], 8, 4, 64, 16, True),         # D 64; one lone tile over a single key tile
    (0, [150, 130, 190], 2, 1, 128, 256, True),     # no prefix, lone third query tile
    (512, [200, 150, 64], 16, 8, 128, 256, True),   # an even and an odd number of key tiles
    (112, [100], 8, 8, 128, 16, True),              # G 1: 128 positions per tile
    (112, [30, 90], 16, 4, 128, 16, True),          # G 4
    (112, [40], 16, 2, 64, 16, True),               # G 8
    (32, [150], 4, 2, 128, 16, False),              # non-causal
    (1024, [64, 192, 320], 16, 8, 128, 256, True),  # 9 to 11 key tiles
]


@pytest.mark.parametrize("prefix,sfx,hq,hkv,d,bs,causal", LONE_CASES)
def test_prefill_lone_query_tiles(oracle, prefix, sfx, hq, hkv, d, bs, causal):
    rng = np.random.default_rng(7 * prefix + sum(sfx) + hq + d + bs)
    w = W.prefill_workload(prefix, np.array(sfx, np.int32), hq, hkv, d, bs, rng=rng, causal=causal)
    lone = lone_tiles(w, causal)
    assert lone, "the case must contain a lone query tile over two key tiles or more"
    out = store_and_prefill(DevicePrefill(w))
    ref = oracle_prefill(oracle, w)
    assert_attention_close(out, ref, what=f"lone-tile prefill prefix={prefix} sfx={sfx} G={hq // hkv} D={d} "
                                          f"causal={causal} lone={lone}")


def test_prefill_lone_cases_cover_the_edges():
    """The lone-tile cases include rows that see no key past the first key tile, even and odd key-tile counts,
    and every GQA group size the kernel instantiates."""
    unseen, even, odd, groups = 0, 0, 0, set()
    for prefix, sfx, hq, hkv, d, bs, causal in LONE_CASES:
        w = W.prefill_workload(prefix, np.array(sfx, np.int32), hq, hkv, d, bs, rng=np.random.default_rng(0),
                               causal=causal)
        for _, nt, rows in lone_tiles(w, causal):
            unseen += rows
            even += nt % 2 == 0
            odd += nt % 2 == 1
        groups.add(hq // hkv)
    assert unseen > 0 and even > 0 and odd > 0
    assert groups == {1, 2, 4, 8}


def test_prefill_prefix_workload_full_size(oracle):
    """The 32-sequence prefix-cached workload at full size (10 804 query tokens x 16 heads), every output element
    against the oracle, in the launch configuration the benchmark times."""
    w = W.prefix_prefill()
    out = store_and_prefill(DevicePrefill(w))
    ref = oracle_prefill(oracle, w)
    T = int(w.cu_seqlens_q[-1])
    assert out.shape == (T, w.num_heads, w.head_dim) and ref.shape == out.shape
    mx, mean = assert_attention_close(out, ref, what="prefix_prefill (all tokens)")
    print(f"prefix prefill: all {T} tokens x {w.num_heads} heads checked, max_abs={mx:.2e} mean_abs={mean:.2e}")


def test_prefill_shared_vs_duplicated_prefix_identical():
    """Prefix blocks shared by every block table give bitwise the same output as private copies."""
    a = W.prefill_workload(512, np.array([100, 37, 300], np.int32), 16, 8, 128, 256,
                           rng=np.random.default_rng(41), shared_prefix=True)
    b = W.prefill_workload(512, np.array([100, 37, 300], np.int32), 16, 8, 128, 256,
                           rng=np.random.default_rng(41), shared_prefix=False)
    for s in range(3):
        Lk = int(a.cu_seqlens_k[s + 1] - a.cu_seqlens_k[s])
        for p in range(0, Lk, 256):
            b.k_cache[b.block_tables[s, p // 256]] = a.k_cache[a.block_tables[s, p // 256]]
            b.v_cache[b.block_tables[s, p // 256]] = a.v_cache[a.block_tables[s, p // 256]]
    b.q[:] = a.q; b.new_k[:] = a.new_k; b.new_v[:] = a.new_v
    oa = store_and_prefill(DevicePrefill(a))
    ob = store_and_prefill(DevicePrefill(b))
    assert torch.equal(oa.view(torch.int16), ob.view(torch.int16))


def test_prefill_poisoned_cache(oracle):
    rng = np.random.default_rng(42)
    w = W.prefill_workload(64, np.array([50, 130, 7], np.int32), 8, 2, 128, 64, rng=rng, poison_unused=True)
    out = store_and_prefill(DevicePrefill(w))
    assert_attention_close(out, oracle_prefill(oracle, w), what="poisoned prefill")


def test_prefill_no_device_error():
    assert pa.device_error() == 0


def test_prefill_fully_cached_sequences_and_empty_batch(oracle):
    """A sequence whose prompt is entirely cached has no query rows (Lq = 0); the others are unaffected, and a
    batch with no query rows at all launches nothing."""
    rng = np.random.default_rng(31)
    w = W.prefill_workload(32, [0, 5, 0, 70], 8, 2, 128, 16, rng=rng)
    dw = DevicePrefill(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    out = pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                            w.max_seqlen_k, dw.block_tables, w.scale, True)
    torch.cuda.synchronize()
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                   w.scale, True, want_f64=True)
    assert_attention_close(out, ref, what="prefill with fully cached sequences")
    w0 = W.prefill_workload(32, [0, 0], 8, 2, 128, 16, rng=rng)
    d0 = DevicePrefill(w0)
    out0 = pa.prefill_varlen(d0.q, d0.k_cache, d0.v_cache, d0.cu_seqlens_q, d0.cu_seqlens_k, w0.max_seqlen_q,
                             w0.max_seqlen_k, d0.block_tables, w0.scale, True)
    torch.cuda.synchronize()
    assert out0.shape[0] == 0
    assert pa.device_error() == 0


def test_prefill_output_16_byte_aligned(oracle):
    """An output buffer that is 16- but not 32-byte aligned takes the 16-byte store path of the epilogue."""
    rng = np.random.default_rng(41)
    w = W.prefill_workload(256, [100, 37], 8, 2, 128, 256, rng=rng)
    dw = DevicePrefill(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    T = dw.q.shape[0]
    buf = torch.zeros(T * 8 * 128 + 8, dtype=torch.bfloat16, device="cuda")
    out = buf[8:].view(T, 8, 128)                        # 16-byte offset from a 256-byte aligned allocation
    assert out.data_ptr() % 32 == 16
    pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                      w.max_seqlen_k, dw.block_tables, w.scale, True, out=out)
    ref_out = pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                                w.max_seqlen_k, dw.block_tables, w.scale, True)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    assert not buf[:8].view(torch.int16).any()          # nothing written before the view
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                   w.scale, True, want_f64=True)
    assert_attention_close(out, ref, what="prefill, 16-byte aligned out")
    assert pa.device_error() == 0
