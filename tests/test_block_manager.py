"""The library's C++ block manager against the block-manager oracle (CPU only).

Integer work, so the bar is bit-exact: after every operation of random traces
(shared system prompts, growth through may_append, releases, revivals of freed
prefix blocks) the block tables, cached-token counts, reference counts, block
hashes, free-block counts and the prefill / decode metadata must be identical.
The library's XXH64 is checked against the xxhash package.
"""
import numpy as np
import pytest
import xxhash

from oracle.block_manager import OracleBlockManager, block_hash as oracle_block_hash
from paged_kv_cache_331_b200 import _binding
from paged_kv_cache_331_b200 import block_manager as BM


@pytest.fixture(scope="module", autouse=True)
def built():
    from paged_kv_cache_331_b200 import build as B
    B.build()


def test_xxh64_matches_the_xxhash_package():
    rng = np.random.default_rng(0)
    for n in list(range(0, 130)) + [255, 256, 257, 1000, 4096 + 7]:
        data = rng.integers(0, 256, n, dtype=np.uint8).tobytes()
        for seed in (0, 1, 0x9E3779B97F4A7C15, int(rng.integers(0, 2 ** 63))):
            assert BM.xxh64(data, seed) == xxhash.xxh64_intdigest(data, seed=seed), (n, seed)


def test_block_hash_matches_the_oracle():
    rng = np.random.default_rng(1)
    for bs in (2, 16, 256):
        toks = rng.integers(-5, 2 ** 31 - 1, bs).astype(np.int32)
        prefix = int(rng.integers(0, 2 ** 63)) * 2 + 1
        assert BM.block_hash(toks) == oracle_block_hash(toks)
        assert BM.block_hash(toks, prefix) == oracle_block_hash(toks, prefix)


def _compare(lib, orc, live, max_blocks):
    assert lib.num_free_blocks() == orc.num_free_blocks()
    for sid, seq in orc.seqs.items():
        n, cached, nb = lib.sequence_info(sid)
        assert (n, cached, nb) == (len(seq), seq.num_cached_tokens, len(seq.block_table)), sid
        assert lib.block_table(sid) == seq.block_table, sid
    for b, blk in enumerate(orc.blocks):
        rc, has, h = lib.block_info(b)
        assert rc == blk.ref_count, b
        assert has == (blk.hash != -1), b
        if has:
            assert h == blk.hash, b
    if live:
        ids = sorted(live)
        a, o = lib.prepare_prefill(ids, max_blocks), orc.prepare_prefill(ids, max_blocks)
        for k in o:
            assert np.array_equal(a[k], o[k]), k
        full = [s for s in ids if len(orc.seqs[s].block_table) == orc.num_blocks_of(orc.seqs[s])]
        if full:
            a, o = lib.prepare_decode(full, max_blocks), orc.prepare_decode(full, max_blocks)
            for k in o:
                assert np.array_equal(a[k], o[k]), k


@pytest.mark.parametrize("seed,num_blocks,bs", [(0, 40, 4), (1, 24, 2), (2, 200, 16), (3, 12, 8)])
def test_random_traces_match_the_oracle(seed, num_blocks, bs):
    rng = np.random.default_rng(seed)
    lib, orc = BM.BlockManager(num_blocks, bs), OracleBlockManager(num_blocks, bs)
    vocab = 6
    systems = [list(rng.integers(0, vocab, int(rng.integers(1, 4 * bs)))) for _ in range(3)]
    live, sid = [], 0
    max_blocks = num_blocks
    for step in range(400):
        op = rng.integers(0, 4)
        if op == 0:                                   # a new request, often behind a shared system prompt
            toks = (systems[rng.integers(0, 3)] if rng.random() < 0.7 else []) + \
                list(rng.integers(0, vocab, int(rng.integers(1, 3 * bs))))
            lib.add_sequence(sid, toks)
            orc.add_sequence(sid, toks)
            assert lib.can_allocate(sid) == orc.can_allocate(sid)
            if orc.can_allocate(sid):
                lib.allocate(sid)
                orc.allocate(sid)
                live.append(sid)
            else:
                lib.remove_sequence(sid)
                orc.remove_sequence(sid)
            sid += 1
        elif op in (1, 2) and live:                   # decode growth
            s = live[rng.integers(0, len(live))]
            t = int(rng.integers(0, vocab))
            lib.append_token(s, t)
            orc.append_token(s, t)
            assert lib.can_append(s) == orc.can_append(s)
            if orc.can_append(s):
                lib.may_append(s)
                orc.may_append(s)
            else:                                     # preempted: its blocks go back
                lib.remove_sequence(s)
                orc.remove_sequence(s)
                live.remove(s)
        elif op == 3 and live:                        # a request finishes
            s = live.pop(rng.integers(0, len(live)))
            lib.remove_sequence(s)
            orc.remove_sequence(s)
        _compare(lib, orc, live, max_blocks)


def test_failures_change_nothing():
    bm = BM.BlockManager(3, 4)
    bm.add_sequence(1, list(range(10)))             # needs 3 blocks
    bm.add_sequence(2, [7, 7])
    bm.allocate(2)
    assert not bm.can_allocate(1)
    with pytest.raises(_binding.PagedAttentionError, match="NO_FREE_BLOCK"):
        bm.allocate(1)
    assert bm.sequence_info(1) == (10, 0, 0) and bm.num_free_blocks() == 2
    with pytest.raises(_binding.PagedAttentionError, match="INVALID_ARG"):
        bm.allocate(2)                                # already holds blocks
    with pytest.raises(_binding.PagedAttentionError, match="INVALID_ARG"):
        bm.add_sequence(2, [1])                       # duplicate id
    with pytest.raises(_binding.PagedAttentionError, match="INVALID_ARG"):
        bm.deallocate(99)
    with pytest.raises(_binding.PagedAttentionError, match="INVALID_ARG"):
        bm.prepare_prefill([2], 1, token_capacity=1)  # room for 1 of 2 tokens
    with pytest.raises(KeyError):
        bm.can_append(99)
