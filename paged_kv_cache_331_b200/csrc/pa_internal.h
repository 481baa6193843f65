// Host-side declarations shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "pa.h"

namespace pa {

struct DeviceInfo {
  int device;
  int sm_count;
  int max_smem_optin;
  unsigned int* error_word;   // device address of the library's error word on this device
};

// Properties of the current device (cached per device).
const DeviceInfo* current_device_info();

// Record a failure message for pa_last_error() on this host thread.
void set_last_error(const char* fmt, ...);

// 3-D tiled tensor map over bf16 data: dims (d0 innermost, d1, d2), byte
// strides of dims 1 and 2, box (b0, b1, b2).  Returns false on failure
// (message recorded).
bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                    CUtensorMapSwizzle swizzle);

// ------------------------------------------------------------------ store --
cudaError_t launch_store_kvcache(const void* key, const void* value, int64_t key_row_stride,
                                 int64_t value_row_stride, void* k_cache, void* v_cache,
                                 const int32_t* slot_mapping, int32_t num_tokens, int32_t row_elems,
                                 int64_t num_slots, cudaStream_t stream);

// ----------------------------------------------------------------- rotary --
struct RotaryArgs {
  void* q_out;                 // [num_tokens, num_heads, head_dim], dense
  const void* q;               // row stride q_row_stride (elements)
  const void* key;             // row stride key_row_stride
  const void* value;           // row stride value_row_stride
  const int32_t* positions;    // [num_tokens]
  const float* cos_sin;        // [max_position, head_dim]: cos | sin
  void* k_cache;
  void* v_cache;
  const int32_t* slot_mapping;
  int64_t q_row_stride;
  int64_t key_row_stride;
  int64_t value_row_stride;
  int64_t num_slots;
  int32_t max_position;
  int32_t num_tokens;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
};
cudaError_t launch_rotary_store(const RotaryArgs& a, cudaStream_t stream);
cudaError_t launch_rotary_table(float* table, int32_t max_position, int32_t head_dim, double base,
                                cudaStream_t stream);

// ----------------------------------------------------------------- decode --
struct DecodeArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_acc;            // [B, Hq, max_chunks, D] (unused when max_chunks == 1)
  float* ws_ml;             // [B, Hq, max_chunks, 2]
  float* o_part;            // non-null: write fp32 partials (o, lse) instead of out
  float* lse_part;
  const void* new_k;        // fused store (slot_mapping non-null): new rows written before decoding
  const void* new_v;
  int64_t new_k_stride;
  int64_t new_v_stride;
  const int32_t* slot_mapping;
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  int32_t num_seqs;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t num_blocks;
  int32_t chunk_tokens;     // multiple of the decode tile
  int32_t max_chunks;
  float scale;
};

constexpr int kDecodeTile = 64;   // tokens per decode pipeline stage

int32_t decode_auto_chunk(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int sm_count);
pa_status launch_decode(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_merge_lse(void* out, const float* o_parts, const float* lse_parts, int32_t num_parts,
                             int32_t num_rows, int32_t head_dim, cudaStream_t stream);

// ---------------------------------------------------------------- prefill --
struct PrefillArgs {
  void* out;
  const void* q;
  const void* k_cache;
  const void* v_cache;
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  const int32_t* block_tables;
  int32_t total_q;
  int32_t max_seqlen_q;
  int32_t max_seqlen_k;
  int32_t max_blocks_per_seq;
  int32_t num_seqs;
  int32_t num_heads;
  int32_t num_kv_heads;
  int32_t head_dim;
  int32_t block_size;
  int32_t num_blocks;
  float scale;
  int32_t causal;
};

pa_status launch_prefill(const PrefillArgs& a, cudaStream_t stream);

}  // namespace pa
