/*
 * pa_block_manager.h -- host-side KV-cache block manager of libpagedattn.so.
 *
 * The step before the attention path: it decides which physical cache blocks
 * a sequence's tokens live in, shares whole prefix blocks between sequences,
 * and writes the metadata arrays (block_tables, slot_mapping, positions,
 * cu_seqlens, context_lens) that pa_store_kvcache, pa_rotary_store_kvcache,
 * pa_decode and pa_prefill_varlen consume.
 *
 * ("Architektur im Überblick", "Block Manager und KV-Cache-Verwaltung":
 * blocks carry block_id, ref_count, hash and token_ids and are freed when the
 * reference count drops to zero; "Hash-basiertes Prefix Caching": allocate
 * hashes every full block chained with the previous block's hash, and reuses
 * a block whose hash maps to it and whose tokens are equal; "Dynamische
 * Block-Erweiterung": may_append's three cases; "Kern-Designentscheidungen"
 * 2: xxHash and a hash_to_block_id dictionary; "Prefill- und
 * Decode-Vorbereitung": the slots and positions prefill and decode write.)
 *
 * Semantics where the pages are silent:
 * - A block's hash is XXH64 (seed 0) of the previous block's hash as 8
 *   little-endian bytes (absent for a sequence's first block) followed by the
 *   block's token ids as 4-byte little-endian integers.
 * - Cached tokens are a leading run: once one block misses, every later block
 *   of the sequence is allocated fresh.
 * - A block taken for new content drops its old dictionary entry; a freed
 *   block keeps its hash and tokens and can be revived by a later hit.
 * - Free blocks are handed out first-in first-out; deallocate releases a
 *   sequence's blocks last block first.
 *
 * Everything here runs on the host: all pointers are HOST pointers owned by
 * the caller, nothing touches a GPU.  A manager is not thread-safe; use one
 * per scheduler thread.  Sequences are named by caller-chosen int64 ids.
 * Functions returning pa_status report contract violations (unknown or
 * duplicate sequence, wrong state, buffer too small) as PA_ERR_INVALID_ARG
 * and an exhausted free list as PA_ERR_NO_FREE_BLOCK, before changing any
 * state; pa_last_error() holds the message.
 */
#ifndef PAGED_ATTN_PA_BLOCK_MANAGER_H
#define PAGED_ATTN_PA_BLOCK_MANAGER_H

#include <stddef.h>
#include <stdint.h>

#include "pa.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct pa_block_manager pa_block_manager;

/* XXH64 of len bytes (the published xxHash specification, 64-bit variant). */
PA_API uint64_t pa_xxh64(const void* data, size_t len, uint64_t seed);

/* The hash of one full block: XXH64 (seed 0) of [prefix as 8 LE bytes if
 * has_prefix] followed by token_ids[0 .. n) as 4-byte LE integers. */
PA_API uint64_t pa_bm_block_hash(const int32_t* token_ids, int32_t n, int32_t has_prefix, uint64_t prefix);

/* A manager of num_blocks blocks of block_size tokens (block_size >= 2), all
 * free (free order 0, 1, ...).  NULL on invalid arguments or out of memory. */
PA_API pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size);
PA_API void pa_bm_destroy(pa_block_manager* bm);
PA_API int32_t pa_bm_num_free_blocks(const pa_block_manager* bm);

/* Sequences: register with their prompt tokens, append generated tokens,
 * remove (which deallocates first if needed). */
PA_API pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* token_ids,
                                    int32_t num_tokens);
PA_API pa_status pa_bm_append_token(pa_block_manager* bm, int64_t seq_id, int32_t token_id);
PA_API pa_status pa_bm_remove_sequence(pa_block_manager* bm, int64_t seq_id);

/* can_allocate: enough free blocks for all of the sequence's blocks (1/0;
 * -1 for an unknown sequence).  allocate: give the sequence its block table,
 * reusing cached prefix blocks; the sequence must hold no blocks. */
PA_API int32_t pa_bm_can_allocate(const pa_block_manager* bm, int64_t seq_id);
PA_API pa_status pa_bm_allocate(pa_block_manager* bm, int64_t seq_id);
/* Drop the sequence's references (last block first); num_cached_tokens = 0. */
PA_API pa_status pa_bm_deallocate(pa_block_manager* bm, int64_t seq_id);

/* After a token was appended to an allocated sequence of n tokens:
 * n % block_size == 1 takes a new block, n % block_size == 0 hashes the block
 * that just filled, anything else changes nothing.  can_append says whether a
 * free block is available when one is needed (1/0; -1 unknown sequence). */
PA_API int32_t pa_bm_can_append(const pa_block_manager* bm, int64_t seq_id);
PA_API pa_status pa_bm_may_append(pa_block_manager* bm, int64_t seq_id);

/* Introspection. */
PA_API pa_status pa_bm_sequence_info(const pa_block_manager* bm, int64_t seq_id, int32_t* num_tokens,
                                     int32_t* num_cached_tokens, int32_t* num_table_blocks);
PA_API pa_status pa_bm_block_table(const pa_block_manager* bm, int64_t seq_id, int32_t* out, int32_t capacity);
PA_API pa_status pa_bm_block_info(const pa_block_manager* bm, int32_t block_id, int32_t* ref_count,
                                  int32_t* has_hash, uint64_t* hash);

/*
 * pa_bm_prepare_prefill -- metadata of a prefill batch of allocated sequences:
 *   block_tables  [num_seqs, max_blocks_per_seq], padded with -1;
 *   cu_seqlens_q  [num_seqs+1]: prefix sums of the uncached token counts;
 *   cu_seqlens_k  [num_seqs+1]: prefix sums of the sequence lengths;
 *   slot_mapping, positions [total_q]: for every uncached token, its cache
 *                 slot block_table[p / bs] * bs + p % bs and its position p
 *                 (p runs from num_cached_tokens to len - 1);
 *   *total_q      the number of uncached tokens (<= token_capacity, the
 *                 length of slot_mapping and positions).
 */
PA_API pa_status pa_bm_prepare_prefill(const pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                                       int32_t max_blocks_per_seq, int32_t token_capacity, int32_t* block_tables,
                                       int32_t* cu_seqlens_q, int32_t* cu_seqlens_k, int32_t* slot_mapping,
                                       int32_t* positions, int32_t* total_q);

/*
 * pa_bm_prepare_decode -- metadata of a decode step (the last token of each
 * sequence):  block_tables [num_seqs, max_blocks_per_seq] (-1 padded),
 * context_lens[b] = len, positions[b] = len - 1, slot_mapping[b] = that
 * token's slot.
 */
PA_API pa_status pa_bm_prepare_decode(const pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                                      int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* context_lens,
                                      int32_t* slot_mapping, int32_t* positions);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_PA_BLOCK_MANAGER_H */
