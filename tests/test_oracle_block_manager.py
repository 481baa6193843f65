"""Pins of the block-manager oracle (CPU only).

"Architektur im Überblick", Block Manager und KV-Cache-Verwaltung: reference
counted blocks, chained full-block hashes with a token comparison against
collisions, the three cases of may_append, and the slot ranges that prefill and
decode write.  Every pin below is written against what the pages and the page
table arithmetic fix; the planted mistakes at the end each fail one of them.
"""
import numpy as np
import pytest

from oracle import block_manager as OB
from oracle.block_manager import OracleBlockManager, block_hash

BS = 4


def _toks(*vals):
    return [int(v) for v in vals]


def pin_may_append_three_cases(BM):
    bm = BM(8, BS)
    bm.add_sequence(0, _toks(1, 2, 3, 4))
    bm.allocate(0)
    seq = bm.seqs[0]
    assert len(seq.block_table) == 1 and bm.blocks[seq.block_table[0]].hash == block_hash([1, 2, 3, 4])
    bm.append_token(0, 5)                   # len % 4 == 1: a new block
    bm.may_append(0)
    assert len(seq.block_table) == 2 and bm.blocks[seq.block_table[1]].hash == -1
    for t in (6, 7):                        # nothing to do
        bm.append_token(0, t)
        bm.may_append(0)
    assert len(seq.block_table) == 2 and bm.blocks[seq.block_table[1]].hash == -1
    bm.append_token(0, 8)                   # len % 4 == 0: the block is full, hash it chained
    bm.may_append(0)
    assert bm.blocks[seq.block_table[1]].hash == block_hash([5, 6, 7, 8], block_hash([1, 2, 3, 4]))
    assert bm.num_free_blocks() == 6


def pin_prefix_blocks_are_shared(BM):
    bm = BM(16, BS)
    a = _toks(1, 2, 3, 4, 5, 6, 7, 8, 9, 10)
    b = _toks(1, 2, 3, 4, 5, 6, 7, 8, 11)
    bm.add_sequence(0, a)
    bm.add_sequence(1, b)
    bm.allocate(0)
    bm.allocate(1)
    ta, tb = bm.seqs[0].block_table, bm.seqs[1].block_table
    assert ta[:2] == tb[:2] and ta[2] != tb[2]
    assert [bm.blocks[i].ref_count for i in ta[:2]] == [2, 2]
    assert bm.seqs[0].num_cached_tokens == 0 and bm.seqs[1].num_cached_tokens == 8
    assert bm.num_free_blocks() == 16 - 4


def pin_same_tokens_behind_another_prefix_are_not_shared(BM):
    bm = BM(16, BS)
    bm.add_sequence(0, _toks(1, 2, 3, 4, 9, 9, 9, 9))
    bm.add_sequence(1, _toks(5, 6, 7, 8, 9, 9, 9, 9))
    bm.allocate(0)
    bm.allocate(1)
    assert set(bm.seqs[0].block_table).isdisjoint(bm.seqs[1].block_table)
    assert bm.seqs[1].num_cached_tokens == 0
    # a third sequence with the first one's prefix must reach the first one's second block,
    # not the equal-token block that sits behind the other prefix
    bm.add_sequence(2, _toks(1, 2, 3, 4, 9, 9, 9, 9, 1))
    bm.allocate(2)
    assert bm.seqs[2].block_table[:2] == bm.seqs[0].block_table
    assert bm.seqs[2].num_cached_tokens == 8


def pin_token_comparison_guards_collisions(BM, monkeypatch):
    monkeypatch.setattr(OB, "block_hash", lambda tokens, prefix=None: 12345)
    bm = BM(16, BS)
    bm.add_sequence(0, _toks(1, 2, 3, 4))
    bm.add_sequence(1, _toks(5, 6, 7, 8))
    bm.allocate(0)
    bm.allocate(1)
    assert bm.seqs[0].block_table != bm.seqs[1].block_table
    assert bm.seqs[1].num_cached_tokens == 0


def pin_cached_tokens_are_a_leading_run(BM):
    bm = BM(16, BS)
    bm.add_sequence(0, _toks(1, 2, 3, 4, 5, 6, 7, 8, 9))
    bm.allocate(0)
    # the first block's entry disappears while the second block's remains
    del bm.hash_to_block_id[block_hash([1, 2, 3, 4])]
    bm.add_sequence(1, _toks(1, 2, 3, 4, 5, 6, 7, 8, 10))
    bm.allocate(1)
    assert bm.seqs[1].num_cached_tokens == 0
    assert set(bm.seqs[1].block_table).isdisjoint(bm.seqs[0].block_table)


def pin_freed_blocks_are_revived_by_their_prefix(BM):
    bm = BM(8, BS)
    toks = _toks(*range(1, 11))
    bm.add_sequence(0, toks)
    bm.allocate(0)
    first = list(bm.seqs[0].block_table)
    bm.remove_sequence(0)
    assert bm.num_free_blocks() == 8 and all(b.ref_count == 0 for b in bm.blocks)
    bm.add_sequence(1, toks)
    bm.allocate(1)
    assert bm.seqs[1].block_table[:2] == first[:2]
    assert bm.seqs[1].num_cached_tokens == 8


def pin_release_order_and_reuse(BM):
    bm = BM(4, BS)
    bm.add_sequence(0, _toks(*range(12)))                # takes blocks 0, 1, 2
    bm.allocate(0)
    assert bm.seqs[0].block_table == [0, 1, 2]
    bm.deallocate(0)                                      # released last-first: free = 3, 2, 1, 0
    bm.add_sequence(1, _toks(100, 101))
    bm.allocate(1)
    assert bm.seqs[1].block_table == [3]
    bm.add_sequence(2, _toks(200, 201))
    bm.allocate(2)
    assert bm.seqs[2].block_table == [2]


def pin_slots_follow_the_page_table(BM, oracle):
    rng = np.random.default_rng(3)
    bs = 16
    bm = BM(64, bs)
    system = list(rng.integers(0, 1000, 40))
    ids = []
    for s in range(6):
        toks = system + list(rng.integers(0, 1000, int(rng.integers(1, 50))))
        bm.add_sequence(s, toks)
        bm.allocate(s)
        ids.append(s)
    meta = bm.prepare_prefill(ids, 8)
    bt = meta["block_tables"]
    cu_q, cu_k = meta["cu_seqlens_q"], meta["cu_seqlens_k"]
    for r, s in enumerate(ids):
        seq = bm.seqs[s]
        assert cu_k[r + 1] - cu_k[r] == len(seq)
        assert cu_q[r + 1] - cu_q[r] == len(seq) - seq.num_cached_tokens
        for t in range(cu_q[r], cu_q[r + 1]):
            p = int(meta["positions"][t])
            blk, off = oracle.kv_location(bt, r, p, bs, 64)       # the attention oracle's page walk
            assert meta["slot_mapping"][t] == blk * bs + off
    # later sequences reuse the 2 full system blocks
    assert [bm.seqs[s].num_cached_tokens for s in ids] == [0] + [32] * 5
    for s in ids:
        bm.append_token(s, 7)
        bm.may_append(s)
    d = bm.prepare_decode(ids, 8)
    for r, s in enumerate(ids):
        n = len(bm.seqs[s])
        assert d["context_lens"][r] == n and d["positions"][r] == n - 1
        blk, off = oracle.kv_location(d["block_tables"], r, n - 1, bs, 64)
        assert d["slot_mapping"][r] == blk * bs + off


def pin_reference_counts_match_the_tables(BM):
    rng = np.random.default_rng(9)
    bm = BM(40, BS)
    prompts = [[1, 2, 3, 4, 5, 6, 7, 8], [1, 2, 3, 4, 9, 9, 9, 9], [3, 3, 3]]
    live = []
    for step in range(300):
        op = rng.integers(0, 3)
        if op == 0:
            sid = step
            bm.add_sequence(sid, list(prompts[rng.integers(0, 3)]) + list(rng.integers(0, 5, rng.integers(0, 9))))
            if bm.can_allocate(sid):
                bm.allocate(sid)
                live.append(sid)
            else:
                bm.remove_sequence(sid)
        elif op == 1 and live:
            sid = live[rng.integers(0, len(live))]
            bm.append_token(sid, int(rng.integers(0, 5)))
            if bm.can_append(sid):
                bm.may_append(sid)
            else:
                bm.remove_sequence(sid)
                live.remove(sid)
        elif op == 2 and live:
            sid = live.pop(rng.integers(0, len(live)))
            bm.remove_sequence(sid)
        counts = np.zeros(40, int)
        for sid in live:
            seq = bm.seqs[sid]
            assert len(seq.block_table) == bm.num_blocks_of(seq)
            for b in seq.block_table:
                counts[b] += 1
        assert [b.ref_count for b in bm.blocks] == counts.tolist()
        assert bm.num_free_blocks() == int((counts == 0).sum())
        assert set(bm.free_block_ids) == set(np.nonzero(counts == 0)[0].tolist())


PINS = [pin_may_append_three_cases, pin_prefix_blocks_are_shared, pin_same_tokens_behind_another_prefix_are_not_shared,
        pin_token_comparison_guards_collisions, pin_cached_tokens_are_a_leading_run,
        pin_freed_blocks_are_revived_by_their_prefix, pin_release_order_and_reuse, pin_slots_follow_the_page_table,
        pin_reference_counts_match_the_tables]


def _run(pin, BM, monkeypatch, oracle):
    args = {"monkeypatch": monkeypatch, "oracle": oracle}
    import inspect
    names = list(inspect.signature(pin).parameters)[1:]
    pin(BM, **{n: args[n] for n in names})


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_block_manager_oracle(pin, monkeypatch, oracle):
    _run(pin, OracleBlockManager, monkeypatch, oracle)


# ---- planted mistakes: each must fail at least one pin ---------------------------------------------

class NoStickyMiss(OracleBlockManager):
    def allocate(self, seq_id):
        seq = self.seqs[seq_id]
        h = None
        for i in range(self.num_blocks_of(seq)):
            tokens = self.block_tokens(seq, i)
            h = OB.block_hash(tokens, h) if len(tokens) == self.block_size else None
            block_id = self.hash_to_block_id.get(h, -1) if h is not None else -1
            if block_id == -1 or self.blocks[block_id].token_ids != tokens:
                block_id = self.free_block_ids[0]
                block = self._take(block_id)
            else:
                seq.num_cached_tokens += self.block_size
                block = self.blocks[block_id]
                if block_id in self.used_block_ids:
                    block.ref_count += 1
                else:
                    block = self._take(block_id)
            if h is not None:
                block.hash, block.token_ids = h, list(tokens)
                self.hash_to_block_id[h] = block_id
            seq.block_table.append(block_id)


class NoTokenCheck(OracleBlockManager):
    def allocate(self, seq_id):
        seq = self.seqs[seq_id]
        h, miss = None, False
        for i in range(self.num_blocks_of(seq)):
            tokens = self.block_tokens(seq, i)
            h = OB.block_hash(tokens, h) if len(tokens) == self.block_size else None
            block_id = self.hash_to_block_id.get(h, -1) if h is not None else -1
            miss = miss or block_id == -1
            if miss:
                block_id = self.free_block_ids[0]
                block = self._take(block_id)
            else:
                seq.num_cached_tokens += self.block_size
                block = self.blocks[block_id]
                if block_id in self.used_block_ids:
                    block.ref_count += 1
                else:
                    block = self._take(block_id)
            if h is not None:
                block.hash, block.token_ids = h, list(tokens)
                self.hash_to_block_id[h] = block_id
            seq.block_table.append(block_id)


class UnchainedHash(OracleBlockManager):
    def allocate(self, seq_id):
        real = OB.block_hash
        OB.block_hash = lambda tokens, prefix=None: real(tokens)
        try:
            super().allocate(seq_id)
        finally:
            OB.block_hash = real


class AppendOffByOne(OracleBlockManager):
    def may_append(self, seq_id):
        seq = self.seqs[seq_id]
        if len(seq) % self.block_size == 0:          # allocates one token too early
            block_id = self.free_block_ids[0]
            self._take(block_id)
            seq.block_table.append(block_id)


class ReleaseInTableOrder(OracleBlockManager):
    def deallocate(self, seq_id):
        seq = self.seqs[seq_id]
        for block_id in seq.block_table:
            b = self.blocks[block_id]
            b.ref_count -= 1
            if b.ref_count == 0:
                self._release(block_id)
        seq.num_cached_tokens = 0
        seq.block_table = []


class HitNotCounted(OracleBlockManager):
    def allocate(self, seq_id):
        super().allocate(seq_id)
        self.seqs[seq_id].num_cached_tokens = 0


class DecodeSlotOffByOne(OracleBlockManager):
    def prepare_decode(self, seq_ids, max_blocks_per_seq):
        d = super().prepare_decode(seq_ids, max_blocks_per_seq)
        d["slot_mapping"] = d["slot_mapping"] + 1
        return d


MUTANTS = [NoStickyMiss, NoTokenCheck, UnchainedHash, AppendOffByOne, ReleaseInTableOrder, HitNotCounted,
           DecodeSlotOffByOne]


@pytest.mark.parametrize("BM", MUTANTS, ids=lambda c: c.__name__)
def test_planted_block_manager_mistake_is_caught(BM, monkeypatch, oracle):
    caught = []
    for pin in PINS:
        with monkeypatch.context() as mp:
            try:
                _run(pin, BM, mp, oracle)
            except (AssertionError, IndexError, KeyError, ValueError):
                caught.append(pin.__name__)
    assert caught, f"{BM.__name__} passed every pin"
