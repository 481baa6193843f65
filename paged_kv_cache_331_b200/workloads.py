"""Seeded synthetic inputs for the paged-KV attention path.

This module only draws random numbers and lays them out the way a
nano-vLLM-style engine hands them to the attention layer; it holds none of
the attention arithmetic.  Both the CPU oracle and the CUDA library consume
what it produces, so neither can hide a mistake behind a shared helper.

Layouts follow "Architektur im Überblick" (nano-vllm architecture page),
section "Dynamische KV-Cache-Allokation": one cache per layer,
``k_cache``/``v_cache`` of shape ``[num_blocks, block_size, num_kv_heads,
head_dim]``.  The per-token ``slot_mapping`` is the engine-side metadata
built in "Prefill- und Decode-Vorbereitung": the slot of a token at logical
position ``pos`` is ``block_table[pos // block_size] * block_size +
pos % block_size`` (the page/offset split of the lshu.cn essay, §3.2).  It
is input construction, not part of the path; the oracle's store/gather
round-trip test pins it.

All floating tensors are bf16 held as ``uint16`` bit patterns: a float32
N(0,1) draw rounded to the nearest bf16 (ties to even).  Draw order per
workload: context lengths -> block permutation -> Q -> cache contents ->
new K/V rows.
"""
from __future__ import annotations

import math
import os
from dataclasses import dataclass, field

import numpy as np

BF16_NAN = np.uint16(0x7FC0)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bits."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    nan = (u & 0x7FFFFFFF) > 0x7F800000
    lsb = (u >> 16) & 1
    r = ((u + np.uint32(0x7FFF) + lsb) >> 16).astype(np.uint16)
    if nan.any():
        r[nan] = BF16_NAN
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def randn_bf16(rng: np.random.Generator, shape, chunk: int = 1 << 22) -> np.ndarray:
    """N(0,1) draws rounded to bf16.

    One 63-bit seed is drawn from ``rng``; chunk i of the flattened tensor is
    then drawn from ``default_rng([seed, i])``.  The chunks are independent, so
    they are generated on several host threads; the result depends only on
    ``rng``'s state and the shape.
    """
    n = int(np.prod(shape))
    seed = int(rng.integers(0, 2**63 - 1))
    out = np.empty(n, dtype=np.uint16)
    starts = list(range(0, n, chunk))

    def fill(i):
        s = starts[i]
        e = min(n, s + chunk)
        out[s:e] = f32_to_bf16_bits(np.random.default_rng([seed, i]).standard_normal(e - s, dtype=np.float32))

    if len(starts) <= 2:
        for i in range(len(starts)):
            fill(i)
    else:
        from concurrent.futures import ThreadPoolExecutor
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 4, 32)) as ex:
            list(ex.map(fill, range(len(starts))))
    return out.reshape(shape)


def slots_for_positions(block_table: np.ndarray, positions, block_size: int) -> np.ndarray:
    """Engine-side slot metadata for the given logical positions of one sequence."""
    pos = np.asarray(positions, dtype=np.int64)
    return (block_table[pos // block_size].astype(np.int64) * block_size + pos % block_size).astype(np.int32)


@dataclass
class DecodeWorkload:
    """One decode step: store each sequence's new token, then attend over the cache."""
    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    context_lens: np.ndarray          # [B] int32, includes the new token
    block_tables: np.ndarray          # [B, max_blocks] int32, -1 padded
    q: np.ndarray                     # [B, Hq, D] bf16 bits
    k_cache: np.ndarray               # [num_blocks, bs, Hkv, D] bf16 bits
    v_cache: np.ndarray
    new_k: np.ndarray                 # [B, Hkv, D] bf16 bits (token at position L-1)
    new_v: np.ndarray
    slot_mapping: np.ndarray          # [B] int32
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0


@dataclass
class PrefillWorkload:
    """One varlen prefill step over sequences whose leading blocks may be cached."""
    name: str
    num_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    scale: float
    causal: bool
    cu_seqlens_q: np.ndarray          # [B+1] int32
    cu_seqlens_k: np.ndarray          # [B+1] int32
    block_tables: np.ndarray          # [B, max_blocks] int32, -1 padded
    q: np.ndarray                     # [sum Lq, Hq, D] bf16 bits
    k_cache: np.ndarray
    v_cache: np.ndarray
    new_k: np.ndarray                 # [sum Lq, Hkv, D] bf16 bits (uncached tokens)
    new_v: np.ndarray
    slot_mapping: np.ndarray          # [sum Lq] int32
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.cu_seqlens_q.shape[0] - 1)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_seqlen_q(self) -> int:
        return int(np.diff(self.cu_seqlens_q).max()) if self.num_seqs else 0

    @property
    def max_seqlen_k(self) -> int:
        return int(np.diff(self.cu_seqlens_k).max()) if self.num_seqs else 0


def _assign_blocks(rng, nblocks_per_seq, block_size, pool_blocks, pool_factor, shared_prefix_blocks=0):
    demand = int(sum(nblocks_per_seq)) + shared_prefix_blocks
    pool = int(pool_blocks) if pool_blocks is not None else max(1, int(math.ceil(pool_factor * demand)))
    if pool < demand:
        raise ValueError(f"pool of {pool} blocks is smaller than the demand of {demand}")
    perm = rng.permutation(pool).astype(np.int32)
    width = max(1, max((n + shared_prefix_blocks for n in nblocks_per_seq), default=1))
    tables = np.full((len(nblocks_per_seq), width), -1, dtype=np.int32)
    shared = perm[:shared_prefix_blocks]
    cur = shared_prefix_blocks
    for b, n in enumerate(nblocks_per_seq):
        tables[b, :shared_prefix_blocks] = shared
        tables[b, shared_prefix_blocks:shared_prefix_blocks + n] = perm[cur:cur + n]
        cur += n
    return tables, pool, perm


def decode_workload(context_lens, num_heads, num_kv_heads, head_dim, block_size, *, rng,
                    pool_blocks=None, pool_factor=1.25, scale=None, name="decode",
                    poison_unused=False) -> DecodeWorkload:
    """Build a decode step from already-drawn context lengths (the first draw)."""
    lens = np.asarray(context_lens, dtype=np.int32)
    nb = [int(math.ceil(int(L) / block_size)) for L in lens]
    tables, pool, _ = _assign_blocks(rng, nb, block_size, pool_blocks, pool_factor)
    B = len(lens)
    q = randn_bf16(rng, (B, num_heads, head_dim))
    k_cache = randn_bf16(rng, (pool, block_size, num_kv_heads, head_dim))
    v_cache = randn_bf16(rng, (pool, block_size, num_kv_heads, head_dim))
    new_k = randn_bf16(rng, (B, num_kv_heads, head_dim))
    new_v = randn_bf16(rng, (B, num_kv_heads, head_dim))
    slots = np.full(B, -1, dtype=np.int32)
    for b, L in enumerate(lens):
        if L > 0:
            slots[b] = slots_for_positions(tables[b], [int(L) - 1], block_size)[0]
    if poison_unused:
        _poison_outside_context(k_cache, v_cache, tables, lens, block_size)
    return DecodeWorkload(name=name, num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                          block_size=block_size, num_blocks=pool,
                          scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)),
                          context_lens=lens, block_tables=tables, q=q, k_cache=k_cache, v_cache=v_cache,
                          new_k=new_k, new_v=new_v, slot_mapping=slots)


def prefill_workload(prefix_len, suffix_lens, num_heads, num_kv_heads, head_dim, block_size, *, rng,
                     pool_blocks=None, pool_factor=1.25, scale=None, causal=True, shared_prefix=True,
                     name="prefill", poison_unused=False) -> PrefillWorkload:
    """Build a prefill step: every sequence has ``prefix_len`` cached tokens and a new suffix.

    With ``shared_prefix`` the cached prefix occupies the same physical blocks in
    every block table (prefix-cache hits share whole blocks, "Hash-basiertes
    Prefix Caching"); otherwise each sequence gets its own copy of the same
    prefix contents in distinct blocks.  ``prefix_len`` must be a multiple of
    ``block_size`` because only full blocks are shared.
    """
    if prefix_len % block_size:
        raise ValueError("a cached prefix covers whole blocks only")
    sfx = np.asarray(suffix_lens, dtype=np.int32)
    B = len(sfx)
    pblk = prefix_len // block_size
    nb_sfx = [int(math.ceil(int(s) / block_size)) for s in sfx]
    if shared_prefix:
        tables, pool, _ = _assign_blocks(rng, nb_sfx, block_size, pool_blocks, pool_factor, shared_prefix_blocks=pblk)
    else:
        tables, pool, _ = _assign_blocks(rng, [n + pblk for n in nb_sfx], block_size, pool_blocks, pool_factor)
    total_q = int(sfx.sum())
    q = randn_bf16(rng, (total_q, num_heads, head_dim))
    k_cache = randn_bf16(rng, (pool, block_size, num_kv_heads, head_dim))
    v_cache = randn_bf16(rng, (pool, block_size, num_kv_heads, head_dim))
    new_k = randn_bf16(rng, (total_q, num_kv_heads, head_dim))
    new_v = randn_bf16(rng, (total_q, num_kv_heads, head_dim))
    if not shared_prefix and pblk:
        # duplicated prefix: copy sequence 0's prefix contents into every other sequence's own blocks
        for b in range(1, B):
            for i in range(pblk):
                k_cache[tables[b, i]] = k_cache[tables[0, i]]
                v_cache[tables[b, i]] = v_cache[tables[0, i]]
    cu_q = np.zeros(B + 1, dtype=np.int32)
    cu_q[1:] = np.cumsum(sfx)
    cu_k = np.zeros(B + 1, dtype=np.int32)
    cu_k[1:] = np.cumsum(sfx + prefix_len)
    slots = np.empty(total_q, dtype=np.int32)
    for b in range(B):
        slots[cu_q[b]:cu_q[b + 1]] = slots_for_positions(tables[b], np.arange(prefix_len, prefix_len + sfx[b]), block_size)
    if poison_unused:
        _poison_outside_context(k_cache, v_cache, tables, sfx + prefix_len, block_size)
    return PrefillWorkload(name=name, num_heads=num_heads, num_kv_heads=num_kv_heads, head_dim=head_dim,
                           block_size=block_size, num_blocks=pool,
                           scale=float(scale if scale is not None else 1.0 / math.sqrt(head_dim)), causal=causal,
                           cu_seqlens_q=cu_q, cu_seqlens_k=cu_k, block_tables=tables, q=q, k_cache=k_cache,
                           v_cache=v_cache, new_k=new_k, new_v=new_v, slot_mapping=slots,
                           meta={"prefix_len": prefix_len, "shared_prefix": shared_prefix})


def _poison_outside_context(k_cache, v_cache, tables, lens, block_size):
    """Fill every cache row that no sequence may read with NaN."""
    used = np.zeros(k_cache.shape[:2], dtype=bool)
    for b, L in enumerate(lens):
        for pos_blk in range(int(math.ceil(int(L) / block_size))):
            blk = tables[b, pos_blk]
            n = min(block_size, int(L) - pos_blk * block_size)
            used[blk, :n] = True
    k_cache[~used] = BF16_NAN
    v_cache[~used] = BF16_NAN


# ----------------------------------------------------------------------------------------------
# The five named workloads.  ``seed`` defaults to the workload number.

def tiny_decode(seed: int = 1, **kw) -> DecodeWorkload:
    """4 sequences, context {1,17,256,300}, block_size 256, 4 q / 2 kv heads, head_dim 64, 16-block pool."""
    rng = np.random.default_rng(seed)
    return decode_workload([1, 17, 256, 300], 4, 2, 64, 256, rng=rng, pool_blocks=16, name="tiny_decode", **kw)


def qwen3_decode(seed: int = 2, num_seqs: int = 64, **kw) -> DecodeWorkload:
    """Qwen3-0.6B-shaped decode layer: context U[128,4096], 16 q / 8 kv heads, head_dim 128."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(128, 4096, size=num_seqs, endpoint=True).astype(np.int32)
    return decode_workload(lens, 16, 8, 128, 256, rng=rng, name="qwen3_0.6b_decode_b64", **kw)


def large_batch_decode(seed: int = 3, num_seqs: int = 256, **kw) -> DecodeWorkload:
    """256 sequences, context U[100,1024] prompt + U[1,1024] generated, 32 q / 8 kv heads."""
    rng = np.random.default_rng(seed)
    prompt = rng.integers(100, 1024, size=num_seqs, endpoint=True)
    gen = rng.integers(1, 1024, size=num_seqs, endpoint=True)
    return decode_workload((prompt + gen).astype(np.int32), 32, 8, 128, 256, rng=rng,
                           name="large_batch_decode_b256", **kw)


def prefix_prefill(seed: int = 4, num_seqs: int = 32, shared_prefix: bool = True, **kw) -> PrefillWorkload:
    """32 sequences sharing a 1024-token prefix (4 blocks), suffix U[64,512], 16 q / 8 kv heads, causal."""
    rng = np.random.default_rng(seed)
    sfx = rng.integers(64, 512, size=num_seqs, endpoint=True).astype(np.int32)
    return prefill_workload(1024, sfx, 16, 8, 128, 256, rng=rng, shared_prefix=shared_prefix,
                            name="prefix_cached_prefill_b32", **kw)


def long_context_decode(seed: int = 5, **kw) -> DecodeWorkload:
    """8 sequences at context 32768 plus one at context 1; 32 q / 8 kv heads; 1200-block pool."""
    rng = np.random.default_rng(seed)
    lens = np.array([32768] * 8 + [1], dtype=np.int32)
    return decode_workload(lens, 32, 8, 128, 256, rng=rng, pool_blocks=1200, name="long_context_decode", **kw)


WORKLOADS = {
    "tiny_decode": tiny_decode,
    "qwen3_decode": qwen3_decode,
    "large_batch_decode": large_batch_decode,
    "prefix_prefill": prefix_prefill,
    "long_context_decode": long_context_decode,
}
