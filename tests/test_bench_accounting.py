"""The roofline numerators of bench.py (CPU only): algorithmic FLOPs of the
prefill and algorithmic bytes of the decode step, against counts made one
(query, key) pair or one cache row at a time."""
import numpy as np
import pytest

import bench
from paged_kv_cache_331_b200 import workloads as W


def brute_force_pairs(w):
    """Unmasked (query, key) pairs, one at a time: query i of sequence b sits at position Lk - Lq + i and sees keys
    0..position (causal) or all Lk keys."""
    n = 0
    for b in range(w.num_seqs):
        lq = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b])
        lk = int(w.cu_seqlens_k[b + 1] - w.cu_seqlens_k[b])
        for i in range(lq):
            pos = lk - lq + i
            for j in range(lk):
                if not w.causal or j <= pos:
                    n += 1
    return n


@pytest.mark.parametrize("prefix,sfx,causal", [(0, [5, 17, 1], True), (32, [9, 20, 0, 150], True),
                                                (256, [64, 1, 200], True), (32, [9, 20], False), (0, [0, 0], True)])
def test_prefill_flops_count_every_unmasked_pair(prefix, sfx, causal):
    w = W.prefill_workload(prefix, np.array(sfx, np.int32), 4, 2, 64, 16, rng=np.random.default_rng(1),
                           causal=causal)
    assert bench.prefill_flops(w) == 4 * w.head_dim * w.num_heads * brute_force_pairs(w)


def test_prefill_flops_of_the_prefix_workload():
    """32 sequences behind a 1024-token prefix: 4 D Hq sum_s [s * 1024 + s (s + 1) / 2]."""
    w = W.prefix_prefill()
    s = np.diff(w.cu_seqlens_q).astype(np.int64)
    closed = 4 * w.head_dim * w.num_heads * int((s * 1024 + s * (s + 1) // 2).sum())
    assert bench.prefill_flops(w) == closed == 107908702208


def brute_force_decode_bytes(w):
    """Every in-context K and V row of every kv head read once, q read and out written once, each table entry
    covering the context read once, each context length read once."""
    row = w.head_dim * 2
    kv = 0
    tables = 0
    for b in range(w.num_seqs):
        L = int(w.context_lens[b])
        seen = set()
        for j in range(L):
            blk = int(w.block_tables[b, j // w.block_size])
            seen.add(blk)
            kv += 2 * w.num_kv_heads * row                   # K and V of every kv head
        tables += len(seen) * 4
    qo = 2 * w.num_seqs * w.num_heads * row
    return kv, kv + qo + tables + 4 * w.num_seqs


@pytest.mark.parametrize("lens,bs", [([1, 17, 256, 300], 16), ([100, 1000, 4097], 256), ([0, 5], 64)])
def test_decode_bytes_count_every_row(lens, bs):
    w = W.decode_workload(np.array(lens, np.int32), 8, 2, 64, bs, rng=np.random.default_rng(2))
    assert bench.decode_algorithmic_bytes(w) == brute_force_decode_bytes(w)


def test_decode_store_bytes_count_live_rows():
    w = W.decode_workload(np.array([3, 40, 7], np.int32), 4, 2, 64, 16, rng=np.random.default_rng(3))
    w.slot_mapping[1] = -1                                      # a skipped row moves nothing
    row = w.num_kv_heads * w.head_dim * 2
    assert bench.decode_store_bytes(w) == 2 * (2 * row) * 2 + 4 * w.num_seqs


def test_decode_step_bytes_of_the_measured_layer():
    """The Qwen3-0.6B-shaped layer the headline is quoted on: 586 436 608 KV bytes per step, 587 488 068
    algorithmic bytes for the fused store + decode launch."""
    w = W.qwen3_decode(seed=2)
    kv, alg = bench.decode_algorithmic_bytes(w)
    assert kv == 586436608
    assert alg + bench.decode_store_bytes(w) == 587488068
