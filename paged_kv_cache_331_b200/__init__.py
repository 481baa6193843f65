"""Attention over a paged KV cache on B200 (sm_100a).

The computation lives in ``libpagedattn.so`` (C ABI in ``include/pa.h``);
this package is its Python face:

    store_kvcache(key, value, k_cache, v_cache, slot_mapping)
    rotary_cos_sin_cache(max_position, head_dim, base)
    rotary_store_kvcache(q, key, value, positions, cos_sin_cache, k_cache, v_cache, slot_mapping)
    decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale)
    prefill_varlen(q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                   block_tables, scale, causal=True)

The shared library is loaded on first use; importing the package does not
touch CUDA.  ``workloads`` builds seeded synthetic inputs.
"""
from ._binding import (PagedAttentionError, decode, decode_chunk_size, decode_chunk_size_for, decode_noalloc,
                       decode_partial, decode_workspace_size, device_error, lib, merge_partials, prefill_varlen, rotary_cos_sin_cache,
                       rotary_store_kvcache, selftest_wait_timeout, store_decode, store_kvcache)

__all__ = ["store_kvcache", "rotary_cos_sin_cache", "rotary_store_kvcache", "decode", "decode_noalloc",
           "decode_partial", "merge_partials", "store_decode",
           "prefill_varlen", "decode_workspace_size", "decode_chunk_size", "decode_chunk_size_for", "device_error", "selftest_wait_timeout", "PagedAttentionError",
           "lib"]
