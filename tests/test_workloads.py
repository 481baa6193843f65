"""The five synthetic workloads against the configurations they stand for
(CPU only): sizes, length ranges, head layout, block pools and the layout of
their block tables, the new tokens' slots, the value distribution, and
determinism under the seed."""
import math

import numpy as np
import pytest

from paged_kv_cache_331_b200 import workloads as W


def check_tables(w, lens, shared=0):
    """Each sequence's first ceil(L / bs) entries are block ids in the pool, padded with -1; sequences share only
    their first ``shared`` entries (prefix-cache blocks), otherwise every block belongs to one sequence."""
    seen = {}
    for b, L in enumerate(lens):
        n = math.ceil(int(L) / w.block_size)
        row = w.block_tables[b]
        assert (row[:n] >= 0).all() and (row[:n] < w.k_cache.shape[0]).all()
        assert (row[n:] == -1).all()
        for i, blk in enumerate(row[:n]):
            if i < shared:
                continue
            assert int(blk) not in seen, (b, i, int(blk))
            seen[int(blk)] = b
    if shared:
        assert (w.block_tables[:, :shared] == w.block_tables[0, :shared]).all()
        assert not set(w.block_tables[0, :shared].tolist()) & set(seen)


def pool_for(lens, bs, shared_blocks=0):
    """The blocks the contexts need (shared prefix blocks counted once); a pool holds about 1.25 times that."""
    return sum(math.ceil(int(L) / bs) for L in lens) - shared_blocks * (len(lens) - 1)


def bf16_values(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32)


def test_tiny_decode():
    w = W.tiny_decode()
    assert w.context_lens.tolist() == [1, 17, 256, 300]
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size) == (4, 2, 64, 256)
    assert w.k_cache.shape == (16, 256, 2, 64) and w.v_cache.shape == w.k_cache.shape
    check_tables(w, w.context_lens)
    assert w.scale == 0.125


def test_qwen3_decode_layer():
    w = W.qwen3_decode()
    L = w.context_lens
    assert w.num_seqs == 64 and L.min() >= 128 and L.max() <= 4096
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size) == (16, 8, 128, 256)
    need = pool_for(L, 256)
    assert need <= w.k_cache.shape[0] <= math.ceil(1.25 * need) + 1
    check_tables(w, L)
    assert w.scale == pytest.approx(1 / math.sqrt(128))


def test_large_batch_decode():
    w = W.large_batch_decode()
    L = w.context_lens
    assert w.num_seqs == 256 and L.min() >= 101 and L.max() <= 2048
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size) == (32, 8, 128, 256)
    check_tables(w, L)


def test_long_context_decode():
    w = W.long_context_decode()
    assert w.context_lens.tolist() == [32768] * 8 + [1]
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size) == (32, 8, 128, 256)
    assert w.k_cache.shape[0] == 1200
    check_tables(w, w.context_lens)


def test_prefix_prefill():
    w = W.prefix_prefill()
    lq = np.diff(w.cu_seqlens_q)
    lk = np.diff(w.cu_seqlens_k)
    assert w.num_seqs == 32 and lq.min() >= 64 and lq.max() <= 512
    assert (lk - lq == 1024).all()
    assert (w.num_heads, w.num_kv_heads, w.head_dim, w.block_size, w.causal) == (16, 8, 128, 256, True)
    check_tables(w, lk, shared=4)
    assert w.max_seqlen_q == lq.max() and w.max_seqlen_k == lk.max()


def test_decode_slots_are_the_newest_positions():
    for w in (W.tiny_decode(), W.qwen3_decode()):
        for b, L in enumerate(w.context_lens):
            pos = int(L) - 1
            assert w.slot_mapping[b] == int(w.block_tables[b, pos // w.block_size]) * w.block_size + pos % w.block_size


def test_prefill_slots_are_the_suffix_positions():
    w = W.prefill_workload(32, np.array([9, 20, 0, 150], np.int32), 4, 2, 64, 16, rng=np.random.default_rng(3))
    lq, lk = np.diff(w.cu_seqlens_q), np.diff(w.cu_seqlens_k)
    t = 0
    for b in range(w.num_seqs):
        for i in range(int(lq[b])):
            pos = int(lk[b] - lq[b]) + i
            assert w.slot_mapping[t] == int(w.block_tables[b, pos // 16]) * 16 + pos % 16
            t += 1
    assert t == w.slot_mapping.shape[0]


def test_values_are_bf16_standard_normal():
    """Mean 0 and standard deviation 1 within six standard errors of each sample's size."""
    w = W.qwen3_decode()
    for a in (w.q, w.k_cache[:64], w.new_k):
        x = bf16_values(a).astype(np.float64).ravel()
        n = x.size
        assert a.dtype == np.uint16
        assert abs(x.mean()) < 6 / math.sqrt(n) and abs(x.std() - 1) < 6 / math.sqrt(2 * n)
        assert np.isfinite(x).all()


def test_same_seed_same_workload():
    a, b = W.tiny_decode(), W.tiny_decode()
    for f in ("context_lens", "block_tables", "q", "k_cache", "v_cache", "new_k", "new_v", "slot_mapping"):
        assert np.array_equal(getattr(a, f), getattr(b, f)), f
    c = W.tiny_decode(seed=11)
    assert not np.array_equal(a.q, c.q)
