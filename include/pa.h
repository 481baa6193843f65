/*
 * pa.h -- C ABI of the paged-KV attention library (libpagedattn.so), sm_100a.
 *
 * The library implements the attention step of a nano-vLLM-style serving
 * engine over a paged KV cache:
 *
 *   pa_store_kvcache   scatter the new tokens' K/V rows into cache slots
 *   pa_rotary_store_kvcache
 *                      rotary embedding of q and k fused with that scatter
 *   pa_decode          one query token per sequence against its cached keys
 *                      (GQA; long contexts split across CTAs and merged by
 *                      the last CTA of each sequence and kv head)
 *   pa_decode_partial, pa_merge_partials
 *                      the same split across GPUs: per-device partials,
 *                      combined after an all-gather
 *   pa_prefill_varlen  causal varlen prefill whose leading blocks may be
 *                      shared prefix-cache blocks
 *
 * Conventions shared by every entry point
 * ----------------------------------------
 * - Pointers named *_cache, q, out, key, value, block_tables, context_lens,
 *   cu_seqlens_*, slot_mapping, positions, cos_sin_cache, table and workspace
 *   are DEVICE pointers owned by the
 *   caller.  The library never allocates, frees or retains them.
 * - bf16 tensors are passed as void*; their layouts are stated per argument.
 *   Every tensor is dense row-major unless a row stride is given.
 * - k_cache / v_cache are one layer's cache, [num_blocks, block_size,
 *   num_kv_heads, head_dim] bf16 ("Architektur im Überblick", section
 *   "Dynamische KV-Cache-Allokation": the per-layer views of the engine's
 *   [2, num_layers, num_blocks, block_size, kv_heads, head_dim] tensor).
 *   Base addresses must be 16-byte aligned.
 * - stream is a cudaStream_t (NULL = legacy default stream).  Every call is
 *   asynchronous on that stream; none synchronises the host.
 * - Argument and shape errors are reported synchronously, before anything is
 *   launched: PA_ERR_INVALID_ARG for values outside the contract,
 *   PA_ERR_UNSUPPORTED for legal shapes this build has no kernel for,
 *   PA_ERR_WORKSPACE for a workspace that is too small, PA_ERR_CUDA when a
 *   launch fails (pa_last_error() then holds the CUDA message).
 * - Device-side contract: block ids in the used part of block_tables lie in
 *   [0, num_blocks); slots are unique; context_lens[b] <= max_context_len and
 *   <= max_blocks_per_seq*block_size; cu_seqlens_q/k agree with total_q,
 *   max_seqlen_q/k and the table width.  The kernels check every one of
 *   these that could send an access outside the caller's buffers, skip or
 *   clamp that access and record a code (pa_device_error); uniqueness of
 *   slots is not checked.
 * - Supported: head_dim 64 or 128; num_heads a multiple of num_kv_heads
 *   with group size G = num_heads / num_kv_heads in 1..8 for decode and
 *   G in {1, 2, 4, 8} for prefill; block_size a power of two in [16, 1024];
 *   num_blocks * block_size < 2^31.
 */
#ifndef PAGED_ATTN_PA_H
#define PAGED_ATTN_PA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum pa_status {
    PA_OK = 0,
    PA_ERR_INVALID_ARG = 1,
    PA_ERR_UNSUPPORTED = 2,
    PA_ERR_CUDA = 3,
    PA_ERR_WORKSPACE = 4,
    PA_ERR_NO_FREE_BLOCK = 5   /* block manager (pa_block_manager.h): no free cache block left */
} pa_status;

/* Static string naming a status code. */
PA_API const char* pa_status_string(int status);

/* Message describing the last failed call on this host thread ("" if none). */
PA_API const char* pa_last_error(void);

/* Library ABI version: (major << 16) | minor. */
PA_API int32_t pa_version(void);

/*
 * pa_store_kvcache -- write the new tokens' K/V rows into the cache.
 * ("Nano-vLLM 源碼學習" §二.2: a store_kvcache kernel stores key and value
 * into the cache; "Architektur im Überblick", "Prefill- und
 * Decode-Vorbereitung": the engine builds one slot per new token.)
 *
 * For each t in [0, num_tokens) with s = slot_mapping[t] != -1:
 *   k_cache[s / block_size][s % block_size][:][:] = key[t][:][:]
 *   v_cache[s / block_size][s % block_size][:][:] = value[t][:][:]
 * A bit copy.  Slots equal to -1 are skipped; a slot outside
 * [0, num_blocks*block_size) other than -1 breaks the contract: it is also
 * skipped, never written out of bounds, and device error code 6 is recorded.
 *
 * key, value:    [num_tokens, num_kv_heads, head_dim] bf16, row t starting at
 *                element t*key_row_stride (t*value_row_stride); the strides
 *                are in elements and may exceed num_kv_heads*head_dim (views
 *                into a fused QKV buffer).
 * slot_mapping:  [num_tokens] int32.
 * num_tokens == 0 launches nothing and returns PA_OK.
 */
PA_API pa_status pa_store_kvcache(const void* key, const void* value, int64_t key_row_stride, int64_t value_row_stride,
                           void* k_cache, void* v_cache, const int32_t* slot_mapping, int32_t num_tokens,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           void* stream);

/*
 * pa_rotary_cos_sin_cache -- fill the rotary embedding's cos/sin table.
 * ("Nano-vLLM 源碼學習", layers, 7 rotary_embedding.py: the RotaryEmbedding
 * class encodes positions through sines and cosines, built once and cached.)
 *
 * For p in [0, max_position) and i in [0, head_dim/2), with
 * theta_i = base^(-2i/head_dim) and the angle p*theta_i taken in double:
 *   table[p*head_dim + i]              = (float) cos(p*theta_i)
 *   table[p*head_dim + head_dim/2 + i] = (float) sin(p*theta_i)
 * table: caller-owned device buffer of max_position*head_dim floats.
 * head_dim even in [2, 1024]; base > 1; max_position*head_dim < 2^31.
 */
PA_API pa_status pa_rotary_cos_sin_cache(float* table, int32_t max_position, int32_t head_dim, double base,
                                  void* stream);

/*
 * pa_rotary_store_kvcache -- rotary position embedding of q and k fused with
 * pa_store_kvcache.  ("Nano-vLLM 源碼學習", layers, 7 rotary_embedding.py and
 * §二.2; "Architektur im Überblick", Attention-Mechanismus: rotary_emb is
 * applied to q and k before attention stores k and v in the cache.)
 *
 * For every token t at position p = positions[t], each head row x (head_dim
 * values) of q[t] and key[t] is rotated pairwise, element i with element
 * i + head_dim/2, by the angle whose cos/sin sit in row p of cos_sin_cache:
 *   y_i = x_i cos - x_{i+D/2} sin,   y_{i+D/2} = x_{i+D/2} cos + x_i sin
 * in float, rounded to bf16 (nearest-even).  The rotated query rows go to
 * q_out; if s = slot_mapping[t] != -1 the rotated key rows and the unchanged
 * value rows are written to slot s exactly as pa_store_kvcache writes them.
 *
 * q:             [num_tokens, num_heads, head_dim] bf16, row t at element
 *                t*q_row_stride (views into a fused QKV buffer allowed).
 * q_out:         [num_tokens, num_heads, head_dim] bf16, dense.  May be q
 *                itself when q_row_stride == num_heads*head_dim; must not
 *                otherwise overlap q, key or value.
 * key, value:    as for pa_store_kvcache.
 * positions:     [num_tokens] int32 in [0, max_position).  A position
 *                outside that range leaves the token's q_out rows and K cache
 *                rows unwritten and sets device error code 4.  A slot outside
 *                the cache (other than -1) is skipped and sets code 6.
 * cos_sin_cache: [max_position, head_dim] float as pa_rotary_cos_sin_cache
 *                fills it.
 * Requires head_dim 64 or 128, every pointer 16-byte aligned and every row
 * stride a multiple of 8 elements (PA_ERR_UNSUPPORTED otherwise).
 * num_tokens == 0 launches nothing and returns PA_OK.
 */
PA_API pa_status pa_rotary_store_kvcache(void* q_out, const void* q, int64_t q_row_stride, const void* key,
                                  const void* value, int64_t key_row_stride, int64_t value_row_stride,
                                  const int32_t* positions, const float* cos_sin_cache, int32_t max_position,
                                  void* k_cache, void* v_cache, const int32_t* slot_mapping, int32_t num_tokens,
                                  int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, void* stream);

/*
 * pa_decode_chunk_size -- tokens per split-KV chunk that pa_decode uses when
 * its kv_chunk_size argument is 0, for this shape on the current device.
 * Returns a multiple of 64, or a value >= max_context_len meaning "no split";
 * returns -1 for invalid arguments.
 */
PA_API int32_t pa_decode_chunk_size(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int32_t block_size);

/*
 * pa_decode_chunk_size_for -- the same choice for a device with sm_count
 * streaming multiprocessors, without querying any device (usable on a host
 * with no GPU, e.g. to plan workspace sizes).  The choice aims at about four
 * waves of two CTAs per SM: no split while num_seqs * num_kv_heads already
 * reaches 8 * sm_count or max_context_len <= 512; otherwise the split count
 * within one of that target whose chunks (whole 64-token tiles) overhang the
 * longest context least (of equal overhangs, the fewest chunks), and at most
 * ceil(max_context_len / 512) chunks.
 * Returns -1 for invalid arguments.
 */
PA_API int32_t pa_decode_chunk_size_for(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len,
                                        int32_t sm_count);

/*
 * pa_decode_workspace_size -- bytes of workspace pa_decode needs for these
 * arguments (0 when no sequence is split).  kv_chunk_size as for pa_decode.
 * Returns 0 for invalid arguments as well; pa_decode then reports them.
 */
PA_API size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t block_size, int32_t kv_chunk_size);

/*
 * pa_decode -- paged GQA decode, one query token per sequence.
 * ("Nano-vLLM 源碼學習" §二.2, decode stage: attention against the KV cache;
 * lshu.cn essay on Nano-vLLM §3.2: K/V of logical position j of a sequence
 * are gathered from page j / block_size, offset j % block_size of its page
 * table.)
 *
 * For b in [0, num_seqs), h in [0, num_heads), L = context_lens[b],
 * g = h / (num_heads / num_kv_heads), K_j = k_cache[block_tables[b][j/bs]][j%bs][g]:
 *   out[b][h] = sum_{j<L} softmax_j(scale * <q[b][h], K_j>) * V_j
 * L == 0 gives out[b][h] = 0.  The newest token (position L-1) must already
 * be in the cache (call pa_store_kvcache first, or use pa_store_decode).
 *
 * q, out:         [num_seqs, num_heads, head_dim] bf16 (dense).
 * block_tables:   [num_seqs, max_blocks_per_seq] int32; entries past
 *                 ceil(L/block_size) are never read (may be -1).
 * context_lens:   [num_seqs] int32, each <= max_context_len and <=
 *                 max_blocks_per_seq*block_size; a larger (or negative) one
 *                 is clamped into that range and sets device error code 7.
 * kv_chunk_size:  0 = automatic; otherwise tokens per split-KV chunk, a
 *                 multiple of 64 (a value >= max_context_len disables the
 *                 split).  Sequences longer than one chunk are processed by
 *                 several CTAs whose partial (max, sum, weighted V) results
 *                 are merged by the last of them to finish (through device
 *                 counters the library keeps and resets itself); above
 *                 16384 sequences x kv heads a second kernel merges them.
 * workspace:      device buffer of at least pa_decode_workspace_size(...)
 *                 bytes (may be NULL when that size is 0); fully written
 *                 before it is read, so its contents need no initialisation.
 *                 Concurrent calls must not share a workspace.
 *                 Calls that overlap on the GPU (other streams) use distinct
 *                 merge counters while fewer than 16 are in flight; a CUDA
 *                 graph keeps the counters it was captured with, so its
 *                 replays must not overlap a launch that drew the same ones
 *                 (one captured 16 split launches later, or an eager one).
 * Dispatch order: a launch of 2..512 sequences (at most 8192 CTAs, split or
 * not) takes its longest sequences first.  The CTAs of the first wave start in
 * sequence order; CTA 0 sorts the others by context length and passes each
 * later CTA its sequence through a per-device entry array that every launch
 * leaves clean.  Slots of that array rotate like the merge counters, with the
 * same rule for overlapping launches and graph replays.  The result does not
 * depend on the order.
 */
PA_API pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t kv_chunk_size,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_noalloc -- pa_decode for callers that cannot allocate.
 * (The pages have no counterpart: this is a calling convenience of this
 * library, not part of the method.)
 *
 * Some callers cannot give the library a device buffer of their own: a
 * plugin inside a process that owns and pre-partitions all device memory, or
 * a C caller with no handle on the allocator behind its device memory.  This
 * entry point computes exactly what pa_decode computes, with the same
 * arguments minus the workspace: the split-KV partials go to a fixed array
 * of PA_DECODE_NOALLOC_SCRATCH_BYTES inside the library (reserved on every
 * GPU that loads it, until the library is unloaded).  It allocates nothing.
 *
 * - Shapes whose pa_decode_workspace_size exceeds that limit are rejected
 *   with PA_ERR_WORKSPACE before anything is launched (a larger
 *   kv_chunk_size needs less scratch).
 * - All calls on one device share the array: calls whose kernels may overlap
 *   on that device race and return garbage, so order them.  The array keeps
 *   the last call's contents; nothing needs it zeroed, since every partial a
 *   call reads is written earlier in that call.
 * - The array's device address is looked up on the first call made on each
 *   device; make that first call before any stream capture starts.  A
 *   successful lookup is kept until the library is unloaded (it is stale
 *   after a reset of the device's primary context, e.g. cudaDeviceReset); a
 *   failed one is retried on the next call.
 */
#define PA_DECODE_NOALLOC_SCRATCH_BYTES ((size_t)8 << 20)

PA_API pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                   const int32_t* block_tables, int32_t max_blocks_per_seq,
                                   const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs,
                                   int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                   int32_t num_blocks, float scale, int32_t kv_chunk_size, void* stream);

/*
 * pa_store_decode -- pa_store_kvcache of one new token per sequence followed
 * by pa_decode, in one launch.  ("Nano-vLLM 源碼學習" §二.2: in decode the
 * attention layer stores the new token's k and v, then attends over the cache;
 * "Architektur im Überblick", CUDA Graph Optimierung: fewer launches per
 * decode step.)
 *
 * key, value: [num_seqs, num_kv_heads, head_dim] bf16 with row strides in
 * elements, as for pa_store_kvcache; slot_mapping: [num_seqs] int32.  Token b
 * is the newest token of sequence b: slot_mapping[b] must be -1 (nothing is
 * stored) or the slot of position context_lens[b]-1 in block_tables[b].  The
 * CTA that reads that position writes the row to the slot and attends over
 * the new row (not what the slot held before), so the result equals the two
 * separate calls.  Any other slot is not written and sets device error code
 * 5; the right slot past the end of the cache sets code 6 and is not
 * written either.  key/value rows must be 16-byte aligned with strides that are
 * multiples of 8 elements (PA_ERR_UNSUPPORTED otherwise).  Every other
 * argument, the workspace rule and the errors are pa_decode's.
 * The row is written at the slot the block-table entry for position
 * context_lens[b]-1 names; if that entry lies outside the cache the row is
 * not written and device error code 6 is recorded.
 */
PA_API pa_status pa_store_decode(void* out, const void* q, const void* key, const void* value, int64_t key_row_stride,
                          int64_t value_row_stride, const int32_t* slot_mapping, void* k_cache, void* v_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t max_context_len, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                          int32_t kv_chunk_size, void* workspace, size_t workspace_bytes, void* stream);

/*
 * pa_decode_partial -- pa_decode over the keys this caller holds, returning
 * an fp32 partial instead of the bf16 output, so that partials computed on
 * different GPUs (each holding part of every sequence's context) can be
 * combined with pa_merge_partials after an all-gather.  (Split-KV across
 * devices: the pages' engine shards attention by heads only; the key split
 * and its log-sum-exp combination are the same as the in-GPU split of
 * pa_decode, exact up to rounding.)
 *
 * Over the context_lens[b] keys that block_tables[b] names here:
 *   o_part[b][h][:] = sum_j p_j V_j / sum_j p_j,   p_j = 2^(s_j - max s)
 *   lse_part[b][h]  = log2 sum_j 2^(s_j),           s_j = scale*log2(e)*<q[b,h], K_j>
 * A sequence with no keys here gets o_part = 0 and lse_part = -inf.
 * o_part:   [num_seqs, num_heads, head_dim] fp32 (16-byte aligned).
 * lse_part: [num_seqs, num_heads] fp32.
 * Every other argument, the workspace rule and the errors are pa_decode's.
 */
PA_API pa_status pa_decode_partial(float* o_part, float* lse_part, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, int32_t kv_chunk_size, void* workspace, size_t workspace_bytes,
                            void* stream);

/*
 * pa_merge_partials -- combine num_partials partials of every row (one row
 * per sequence and query head):
 *   M = max_r lse_r,  out = sum_r 2^(lse_r - M) o_r / sum_r 2^(lse_r - M)
 * rounded to bf16; a row whose partials all have lse = -inf is 0.
 * o_parts:   [num_partials, num_rows, head_dim] fp32.
 * lse_parts: [num_partials, num_rows] fp32.
 * out:       [num_rows, head_dim] bf16.  head_dim 64 or 128.
 */
PA_API pa_status pa_merge_partials(void* out, const float* o_parts, const float* lse_parts, int32_t num_partials,
                            int32_t num_rows, int32_t head_dim, void* stream);

/*
 * pa_prefill_varlen -- varlen causal prefill against the paged cache.
 * ("Nano-vLLM 源碼學習" §二.2, prefill stage: varlen attention with prefix
 * cache support; "Architektur im Überblick", "Prefill- und
 * Decode-Vorbereitung": only the uncached tokens are computed and their
 * positions start at num_cached_tokens; "Hash-basiertes Prefix Caching":
 * cached prefix blocks are whole blocks shared by reference.)
 *
 * Sequence b has Lq = cu_seqlens_q[b+1]-cu_seqlens_q[b] query tokens (its
 * uncached tokens, whose K/V were stored with pa_store_kvcache beforehand)
 * and Lk = cu_seqlens_k[b+1]-cu_seqlens_k[b] >= Lq keys, all read from the
 * cache through block_tables[b].  Query i sits at position Lk - Lq + i; with
 * causal != 0 it attends keys 0 .. Lk-Lq+i, otherwise keys 0 .. Lk-1.
 *
 * q, out:         [total_q, num_heads, head_dim] bf16 (dense), total_q =
 *                 cu_seqlens_q[num_seqs] - cu_seqlens_q[0]; row t of q/out
 *                 belongs to the sequence b with cu_seqlens_q[b] <= t +
 *                 cu_seqlens_q[0] < cu_seqlens_q[b+1].
 * cu_seqlens_q/k: [num_seqs+1] int32, non-decreasing.
 * max_seqlen_q/k: upper bounds of Lq and Lk over the batch.
 * block_tables:   as for pa_decode, entries past ceil(Lk/block_size) unread.
 *
 * Checked on the device: a sequence whose cu_seqlens_q/k disagree with
 * total_q, max_seqlen_q/k or the table width (Lk > max_blocks_per_seq *
 * block_size) is skipped, its output rows left unwritten, and device error
 * code 8 is recorded; a used block-table entry outside the cache records
 * code 6 and reads zeros.  Nothing is read or written outside the caller's
 * buffers.
 */
PA_API pa_status pa_prefill_varlen(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t total_q,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, const int32_t* block_tables,
                            int32_t max_blocks_per_seq, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t causal,
                            void* stream);

/*
 * pa_device_error -- read and clear the library's device-side error word on
 * the current device (synchronises the given stream).  Kernels set it instead
 * of hanging when a pipeline wait exceeds its time limit (about one second),
 * and pa_rotary_store_kvcache sets it for a position outside its table.
 * Codes: 0 none, 1 a pipeline wait (or a decode CTA's wait for its place in
 * the dispatch order) timed out, 2 the wait for in-flight copies
 * at exit timed out, 3 dynamic shared memory misaligned, 4 rotary position
 * out of range, 5 a pa_store_decode slot that is not the new token's,
 * 6 a slot (other than -1) or a used block-table entry outside the cache
 * (the store is skipped; decode and prefill read zeros for that block),
 * 7 a decode context length above max_context_len or the table width (it is
 * clamped), 8 a prefill sequence whose cu_seqlens_q/k disagree with
 * total_q, max_seqlen_q/k or the table width (that sequence is skipped: its
 * output rows are not written).  The first code recorded since the last
 * read wins.  Diagnostic only.
 */
PA_API pa_status pa_device_error(int32_t* code_out, void* stream);

/*
 * pa_selftest_wait_timeout -- launch one CTA whose pipeline wait has nothing
 * to arrive on, to check the time-limited waits the kernels rely on.  The
 * wait gives up after limit_ns nanoseconds (1e3 .. 1e9) and records code 1
 * in the device error word (pa_device_error); the CTA then frees the tensor
 * memory it allocated and returns, as the kernels do on that path.  Nothing
 * hangs and nothing faults; later launches are unaffected.  Diagnostic only.
 */
PA_API pa_status pa_selftest_wait_timeout(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_ATTN_PA_H */
