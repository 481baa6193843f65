"""Oracle of the KV-cache block manager -- TEST INFRASTRUCTURE ONLY.

Plain Python restatement of the block manager the pages describe, for the
tests that check the library's C++ block manager against it.  Only ``tests/``
may import it; the product never does.  It shares no code with the library.

Sources (web pages about nano-vllm):
 - "Architektur im Überblick", "Block Manager und KV-Cache-Verwaltung":
   a block holds block_id, ref_count, hash (-1 = none) and token_ids; blocks
   are shared between sequences by reference count and freed when it drops
   to zero.
 - same page, "Hash-basiertes Prefix Caching": allocate() walks the
   sequence's blocks, hashes every full block chained with the previous
   block's hash, and reuses a block whose hash maps to it and whose token ids
   are equal (the comparison guards against collisions); otherwise it takes
   the first free block.  A hit adds block_size to num_cached_tokens.
 - same page, "Dynamische Block-Erweiterung": may_append() distinguishes
   len(seq) % block_size == 1 (a new block is needed), == 0 (the last block
   just filled: hash it) and anything else (nothing to do).
 - same page, "Kern-Designentscheidungen" 2: blocks are hashed with xxHash
   and looked up in a hash_to_block_id dictionary.
 - same page, "Block-Berechnung und Token-Appending": num_blocks =
   ceil(num_tokens / block_size), last_block_num_tokens = num_tokens -
   (num_blocks - 1) * block_size.
 - same page, "Prefill- und Decode-Vorbereitung": prefill computes tokens
   from num_cached_tokens on, at positions range(num_cached_tokens, seqlen),
   and writes the slots range(block*bs, block*bs + n) of every non-cached
   block; decode computes the last token.

Readings where the pages are silent (each also stated in the design notes):
 - the hash is XXH64 (seed 0) of the previous block's hash as 8 little-endian
   bytes (absent for the first block) followed by the block's token ids as
   4-byte little-endian integers; the xxhash library computes it here;
 - once a block misses, every later block of the sequence is a miss too:
   prefill skips only a leading run of cached tokens, so a later hit could not
   be used;
 - when a block that still carries a hash is taken for new content, its
   dictionary entry is dropped, so a hit always means the same prefix chain;
 - a block freed with a hash keeps it (and its tokens) until it is reused, so
   a later sequence with the same prefix can revive it.
"""
from __future__ import annotations

from collections import deque

import numpy as np
import xxhash


def block_hash(token_ids, prefix=None) -> int:
    """XXH64 of [prefix hash, 8 bytes LE] + token ids (int32 LE), seed 0."""
    h = xxhash.xxh64(seed=0)
    if prefix is not None:
        h.update(int(prefix).to_bytes(8, "little"))
    h.update(np.asarray(token_ids, dtype="<i4").tobytes())
    return h.intdigest()


class Block:
    def __init__(self, block_id):
        self.block_id = block_id
        self.ref_count = 0
        self.hash = -1
        self.token_ids = []


class Sequence:
    def __init__(self, token_ids):
        self.token_ids = list(token_ids)
        self.num_cached_tokens = 0
        self.block_table = []

    def __len__(self):
        return len(self.token_ids)


class OracleBlockManager:
    def __init__(self, num_blocks, block_size):
        assert num_blocks > 0 and block_size >= 2
        self.block_size = block_size
        self.blocks = [Block(i) for i in range(num_blocks)]
        self.hash_to_block_id = {}
        self.free_block_ids = deque(range(num_blocks))
        self.used_block_ids = set()
        self.seqs = {}

    # -- sequences ------------------------------------------------------------
    def add_sequence(self, seq_id, token_ids):
        assert seq_id not in self.seqs
        self.seqs[seq_id] = Sequence(token_ids)

    def append_token(self, seq_id, token_id):
        self.seqs[seq_id].token_ids.append(int(token_id))

    def remove_sequence(self, seq_id):
        if self.seqs[seq_id].block_table:
            self.deallocate(seq_id)
        del self.seqs[seq_id]

    def num_blocks_of(self, seq):
        return (len(seq) + self.block_size - 1) // self.block_size

    def block_tokens(self, seq, i):
        return seq.token_ids[i * self.block_size:(i + 1) * self.block_size]

    # -- blocks ---------------------------------------------------------------
    def _take(self, block_id):
        """Give a free block a new owner: reset it, dropping its stale hash entry."""
        b = self.blocks[block_id]
        assert b.ref_count == 0
        if b.hash != -1 and self.hash_to_block_id.get(b.hash) == block_id:
            del self.hash_to_block_id[b.hash]
        b.ref_count = 1
        b.hash = -1
        b.token_ids = []
        self.free_block_ids.remove(block_id)
        self.used_block_ids.add(block_id)
        return b

    def _release(self, block_id):
        assert self.blocks[block_id].ref_count == 0
        self.used_block_ids.remove(block_id)
        self.free_block_ids.append(block_id)

    def num_free_blocks(self):
        return len(self.free_block_ids)

    # -- the three operations of the pages ----------------------------------
    def can_allocate(self, seq_id):
        return len(self.free_block_ids) >= self.num_blocks_of(self.seqs[seq_id])

    def allocate(self, seq_id):
        seq = self.seqs[seq_id]
        assert not seq.block_table
        h = None
        miss = False
        for i in range(self.num_blocks_of(seq)):
            tokens = self.block_tokens(seq, i)
            h = block_hash(tokens, h) if len(tokens) == self.block_size else None
            block_id = self.hash_to_block_id.get(h, -1) if h is not None else -1
            if block_id == -1 or self.blocks[block_id].token_ids != tokens:
                miss = True
            if miss:
                block_id = self.free_block_ids[0]
                block = self._take(block_id)
            else:
                seq.num_cached_tokens += self.block_size
                block = self.blocks[block_id]
                if block_id in self.used_block_ids:
                    block.ref_count += 1
                else:   # freed but still holding this content: revive it
                    block = self._take(block_id)
            if h is not None:
                block.hash = h
                block.token_ids = list(tokens)
                self.hash_to_block_id[h] = block_id
            seq.block_table.append(block_id)

    def deallocate(self, seq_id):
        seq = self.seqs[seq_id]
        for block_id in reversed(seq.block_table):
            b = self.blocks[block_id]
            b.ref_count -= 1
            if b.ref_count == 0:
                self._release(block_id)
        seq.num_cached_tokens = 0
        seq.block_table = []

    def can_append(self, seq_id):
        seq = self.seqs[seq_id]
        return len(self.free_block_ids) >= (1 if len(seq) % self.block_size == 1 else 0)

    def may_append(self, seq_id):
        """Called after a token was appended: make room for it, or seal the block it filled."""
        seq = self.seqs[seq_id]
        table = seq.block_table
        last = self.blocks[table[-1]]
        n = len(seq)
        if n % self.block_size == 1:
            assert last.hash != -1
            block_id = self.free_block_ids[0]
            self._take(block_id)
            table.append(block_id)
        elif n % self.block_size == 0:
            assert last.hash == -1
            tokens = self.block_tokens(seq, len(table) - 1)
            prefix = self.blocks[table[-2]].hash if len(table) > 1 else None
            h = block_hash(tokens, prefix)
            last.hash = h
            last.token_ids = list(tokens)
            self.hash_to_block_id[h] = last.block_id
        else:
            assert last.hash == -1

    # -- batch metadata ------------------------------------------------------
    def prepare_prefill(self, seq_ids, max_blocks_per_seq):
        bs = self.block_size
        cu_q, cu_k, slots, positions = [0], [0], [], []
        tables = np.full((len(seq_ids), max_blocks_per_seq), -1, np.int32)
        for r, sid in enumerate(seq_ids):
            seq = self.seqs[sid]
            n = len(seq)
            positions.extend(range(seq.num_cached_tokens, n))
            cu_q.append(cu_q[-1] + n - seq.num_cached_tokens)
            cu_k.append(cu_k[-1] + n)
            nb = self.num_blocks_of(seq)
            for i in range(seq.num_cached_tokens // bs, nb):
                start = seq.block_table[i] * bs
                count = bs if i != nb - 1 else n - (nb - 1) * bs
                slots.extend(range(start, start + count))
            assert len(seq.block_table) <= max_blocks_per_seq
            tables[r, :len(seq.block_table)] = seq.block_table
        return dict(block_tables=tables, cu_seqlens_q=np.array(cu_q, np.int32), cu_seqlens_k=np.array(cu_k, np.int32),
                    slot_mapping=np.array(slots, np.int32), positions=np.array(positions, np.int32))

    def prepare_decode(self, seq_ids, max_blocks_per_seq):
        bs = self.block_size
        B = len(seq_ids)
        tables = np.full((B, max_blocks_per_seq), -1, np.int32)
        ctx, slots, pos = (np.zeros(B, np.int32) for _ in range(3))
        for r, sid in enumerate(seq_ids):
            seq = self.seqs[sid]
            n = len(seq)
            nb = self.num_blocks_of(seq)
            ctx[r] = n
            pos[r] = n - 1
            slots[r] = seq.block_table[-1] * bs + (n - (nb - 1) * bs) - 1
            assert len(seq.block_table) <= max_blocks_per_seq
            tables[r, :len(seq.block_table)] = seq.block_table
        return dict(block_tables=tables, context_lens=ctx, slot_mapping=slots, positions=pos)
