// C ABI of the paged-KV attention library: argument validation, tensor-map
// encoding and dispatch to the kernels.  Nothing here allocates device
// memory; every buffer belongs to the caller.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <mutex>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {

// One error word per device that loads the library; kernels record a code
// here instead of hanging when a pipeline wait runs out of time.
__device__ unsigned int g_device_error = 0;

namespace {

thread_local char t_last_error[512] = "";

constexpr int kMaxDevices = 64;
DeviceInfo g_devinfo[kMaxDevices];
std::once_flag g_devinfo_once[kMaxDevices];

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

bool is_pow2(int32_t x) { return x > 0 && (x & (x - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pa_status fail(pa_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
  return st;
}

// Shape rules shared by decode and prefill.
pa_status check_cache_shape(const char* who, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                            int32_t block_size, int32_t num_blocks) {
  if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "%s: num_heads (%d) must be a positive multiple of num_kv_heads (%d)", who,
                num_heads, num_kv_heads);
  if (num_blocks <= 0) return fail(PA_ERR_INVALID_ARG, "%s: num_blocks must be positive", who);
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "%s: head_dim %d not supported (64 or 128)", who, head_dim);
  if (!is_pow2(block_size) || block_size < 16 || block_size > 1024)
    return fail(PA_ERR_UNSUPPORTED, "%s: block_size %d not supported (power of two in [16, 1024])", who,
                block_size);
  if (static_cast<int64_t>(num_blocks) * block_size >= (int64_t(1) << 31))
    return fail(PA_ERR_UNSUPPORTED, "%s: num_blocks * block_size must stay below 2^31", who);
  return PA_OK;
}

}  // namespace

void set_last_error(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_last_error, sizeof t_last_error, fmt, ap);
  va_end(ap);
}

const DeviceInfo* current_device_info() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = 0;
  std::call_once(g_devinfo_once[dev], [dev] {
    DeviceInfo& d = g_devinfo[dev];
    d.device = dev;
    d.sm_count = 148;
    d.max_smem_optin = 227 * 1024;
    cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.max_smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    d.error_word = nullptr;
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, g_device_error) == cudaSuccess) d.error_word = static_cast<unsigned int*>(addr);
  });
  return &g_devinfo[dev];
}

bool encode_bf16_3d(CUtensorMap* map, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                    uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t b0, uint32_t b1, uint32_t b2,
                    CUtensorMapSwizzle swizzle) {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  if (!g_encode) {
    set_last_error("cuTensorMapEncodeTiled is not available from the driver");
    return false;
  }
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_last_error("cuTensorMapEncodeTiled failed (%d): dims %llu x %llu x %llu, box %u x %u x %u", (int)r,
                   (unsigned long long)d0, (unsigned long long)d1, (unsigned long long)d2, b0, b1, b2);
    return false;
  }
  return true;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_status_string(int status) {
  switch (status) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID_ARG: return "PA_ERR_INVALID_ARG";
    case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
    case PA_ERR_WORKSPACE: return "PA_ERR_WORKSPACE";
    case PA_ERR_NO_FREE_BLOCK: return "PA_ERR_NO_FREE_BLOCK";
    default: return "PA_ERR_UNKNOWN";
  }
}

const char* pa_last_error(void) { return t_last_error; }

int32_t pa_version(void) { return (1 << 16) | 0; }

pa_status pa_store_kvcache(const void* key, const void* value, int64_t key_row_stride, int64_t value_row_stride,
                           void* k_cache, void* v_cache, const int32_t* slot_mapping, int32_t num_tokens,
                           int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                           void* stream) {
  t_last_error[0] = 0;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "store_kvcache: num_tokens < 0");
  if (num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0)
    return fail(PA_ERR_INVALID_ARG, "store_kvcache: num_kv_heads, head_dim, block_size, num_blocks must be > 0");
  const int64_t row = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (row > (int64_t(1) << 20)) return fail(PA_ERR_UNSUPPORTED, "store_kvcache: row of %lld elements too long",
                                            (long long)row);
  if (key_row_stride < row || value_row_stride < row)
    return fail(PA_ERR_INVALID_ARG, "store_kvcache: row strides must be >= num_kv_heads*head_dim");
  if (num_tokens == 0) return PA_OK;
  if (!key || !value || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "store_kvcache: null pointer");
  const int64_t num_slots = static_cast<int64_t>(num_blocks) * block_size;
  cudaError_t e = launch_store_kvcache(key, value, key_row_stride, value_row_stride, k_cache, v_cache, slot_mapping,
                                       num_tokens, static_cast<int32_t>(row), num_slots,
                                       static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "store_kvcache launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_rotary_cos_sin_cache(float* table, int32_t max_position, int32_t head_dim, double base, void* stream) {
  t_last_error[0] = 0;
  if (!table) return fail(PA_ERR_INVALID_ARG, "rotary_cos_sin_cache: null table");
  if (max_position <= 0 || head_dim < 2 || head_dim > 1024 || head_dim % 2)
    return fail(PA_ERR_INVALID_ARG, "rotary_cos_sin_cache: need max_position > 0 and an even head_dim in [2, 1024]");
  if (!(base > 1.0)) return fail(PA_ERR_INVALID_ARG, "rotary_cos_sin_cache: base must be > 1");
  if (static_cast<int64_t>(max_position) * head_dim >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID_ARG, "rotary_cos_sin_cache: max_position*head_dim must be < 2^31");
  cudaError_t e = launch_rotary_table(table, max_position, head_dim, base, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "rotary_cos_sin_cache launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

static bool ranges_overlap(const void* a, size_t a_bytes, const void* b, size_t b_bytes) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + b_bytes && y < x + a_bytes;
}

pa_status pa_rotary_store_kvcache(void* q_out, const void* q, int64_t q_row_stride, const void* key,
                                  const void* value, int64_t key_row_stride, int64_t value_row_stride,
                                  const int32_t* positions, const float* cos_sin_cache, int32_t max_position,
                                  void* k_cache, void* v_cache, const int32_t* slot_mapping, int32_t num_tokens,
                                  int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                  int32_t num_blocks, void* stream) {
  t_last_error[0] = 0;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "rotary_store_kvcache: num_tokens < 0");
  if (num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0 ||
      max_position <= 0)
    return fail(PA_ERR_INVALID_ARG,
                "rotary_store_kvcache: num_heads, num_kv_heads, head_dim, block_size, num_blocks, max_position "
                "must be > 0");
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "rotary_store_kvcache: head_dim %d (supported: 64, 128)", head_dim);
  if (num_heads > 4096 || num_kv_heads > 4096)
    return fail(PA_ERR_UNSUPPORTED, "rotary_store_kvcache: more than 4096 heads");
  const int64_t qrow = static_cast<int64_t>(num_heads) * head_dim;
  const int64_t kvrow = static_cast<int64_t>(num_kv_heads) * head_dim;
  if (q_row_stride < qrow || key_row_stride < kvrow || value_row_stride < kvrow)
    return fail(PA_ERR_INVALID_ARG, "rotary_store_kvcache: row strides shorter than the rows");
  if (static_cast<int64_t>(max_position) * head_dim >= (int64_t(1) << 31))
    return fail(PA_ERR_INVALID_ARG, "rotary_store_kvcache: max_position*head_dim must be < 2^31");
  if (num_tokens == 0) return PA_OK;
  if (!q_out || !q || !key || !value || !positions || !cos_sin_cache || !k_cache || !v_cache || !slot_mapping)
    return fail(PA_ERR_INVALID_ARG, "rotary_store_kvcache: null pointer");
  auto al16 = [](const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; };
  if (!al16(q_out) || !al16(q) || !al16(key) || !al16(value) || !al16(cos_sin_cache) || !al16(k_cache) ||
      !al16(v_cache) || q_row_stride % 8 || key_row_stride % 8 || value_row_stride % 8)
    return fail(PA_ERR_UNSUPPORTED,
                "rotary_store_kvcache: pointers must be 16-byte aligned and row strides multiples of 8 elements");
  const size_t out_bytes = static_cast<size_t>(num_tokens) * qrow * 2;
  const bool in_place = q_out == q && q_row_stride == qrow;
  auto span = [&](int64_t stride, int64_t row) {
    return (static_cast<size_t>(num_tokens - 1) * stride + row) * 2;
  };
  if ((!in_place && ranges_overlap(q_out, out_bytes, q, span(q_row_stride, qrow))) ||
      ranges_overlap(q_out, out_bytes, key, span(key_row_stride, kvrow)) ||
      ranges_overlap(q_out, out_bytes, value, span(value_row_stride, kvrow)))
    return fail(PA_ERR_INVALID_ARG, "rotary_store_kvcache: q_out overlaps q (other than in place), key or value");
  RotaryArgs a{};
  a.q_out = q_out;
  a.q = q;
  a.key = key;
  a.value = value;
  a.positions = positions;
  a.cos_sin = cos_sin_cache;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.slot_mapping = slot_mapping;
  a.q_row_stride = q_row_stride;
  a.key_row_stride = key_row_stride;
  a.value_row_stride = value_row_stride;
  a.num_slots = static_cast<int64_t>(num_blocks) * block_size;
  a.max_position = max_position;
  a.num_tokens = num_tokens;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  cudaError_t e = launch_rotary_store(a, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "rotary_store_kvcache launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

int32_t pa_decode_chunk_size(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int32_t block_size) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_context_len < 0 || block_size <= 0) return -1;
  return decode_auto_chunk(num_seqs, num_kv_heads, max_context_len, current_device_info()->sm_count);
}

int32_t pa_decode_chunk_size_for(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int32_t sm_count) {
  if (num_seqs < 0 || num_kv_heads <= 0 || max_context_len < 0 || sm_count <= 0) return -1;
  return decode_auto_chunk(num_seqs, num_kv_heads, max_context_len, sm_count);
}

static int32_t resolve_chunk(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int32_t kv_chunk_size) {
  if (kv_chunk_size == 0)
    return decode_auto_chunk(num_seqs, num_kv_heads, max_context_len, current_device_info()->sm_count);
  return kv_chunk_size;
}

static int32_t chunks_for(int32_t max_context_len, int32_t chunk) {
  if (max_context_len <= 0) return 1;
  const int64_t n = (static_cast<int64_t>(max_context_len) + chunk - 1) / chunk;
  return static_cast<int32_t>(n < 1 ? 1 : n);
}

static size_t workspace_bytes_for(int32_t num_seqs, int32_t num_heads, int32_t head_dim, int32_t nchunks) {
  if (nchunks <= 1) return 0;
  const size_t rows = static_cast<size_t>(num_seqs) * num_heads * nchunks;
  const size_t acc = (rows * head_dim * sizeof(float) + 255) / 256 * 256;
  return acc + rows * 2 * sizeof(float);
}

size_t pa_decode_workspace_size(int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_context_len, int32_t block_size, int32_t kv_chunk_size) {
  if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
      block_size <= 0 || kv_chunk_size < 0 || (kv_chunk_size % kDecodeTile))
    return 0;
  const int32_t chunk = resolve_chunk(num_seqs, num_kv_heads, max_context_len, kv_chunk_size);
  return workspace_bytes_for(num_seqs, num_heads, head_dim, chunks_for(max_context_len, chunk));
}

// The store a fused call makes before decoding (none when slot_mapping is null).
struct FusedStore {
  const void* key = nullptr;
  const void* value = nullptr;
  int64_t key_row_stride = 0;
  int64_t value_row_stride = 0;
  const int32_t* slot_mapping = nullptr;
};

// pa_decode, pa_decode_partial and pa_store_decode: out (bf16) or the fp32
// partials (o_part, lse_part), with an optional fused store.
static pa_status decode_common(const char* who, void* out, float* o_part, float* lse_part, const void* q,
                               const void* k_cache, const void* v_cache, const int32_t* block_tables,
                               int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t max_context_len,
                               int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int32_t num_blocks, float scale, int32_t kv_chunk_size,
                               void* workspace, size_t workspace_bytes, void* stream,
                               const FusedStore& fs = FusedStore()) {
  t_last_error[0] = 0;
  const bool partial = o_part != nullptr || lse_part != nullptr;
  if (num_seqs < 0) return fail(PA_ERR_INVALID_ARG, "decode: num_seqs < 0");
  pa_status st = check_cache_shape("decode", num_heads, num_kv_heads, head_dim, block_size, num_blocks);
  if (st != PA_OK) return st;
  if (max_context_len < 0 || max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "decode: max_context_len must be >= 0 and max_blocks_per_seq > 0");
  if (kv_chunk_size < 0 || kv_chunk_size % kDecodeTile)
    return fail(PA_ERR_INVALID_ARG, "decode: kv_chunk_size must be 0 or a positive multiple of %d", kDecodeTile);
  if (!(scale > 0.f) || !isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "decode: scale must be finite and > 0");
  if (num_seqs == 0) return PA_OK;
  if ((partial ? (!o_part || !lse_part) : !out) || !q || !k_cache || !v_cache || !block_tables || !context_lens)
    return fail(PA_ERR_INVALID_ARG, "%s: null pointer", who);
  if (!aligned16(q) || !aligned16(partial ? static_cast<const void*>(o_part) : out) || !aligned16(k_cache) ||
      !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "%s: q, the output and the caches must be 16-byte aligned", who);
  if (static_cast<int64_t>(num_seqs) > 65535) return fail(PA_ERR_UNSUPPORTED, "decode: more than 65535 sequences");
  const int32_t chunk = resolve_chunk(num_seqs, num_kv_heads, max_context_len, kv_chunk_size);
  const int32_t nchunks = chunks_for(max_context_len, chunk);
  const size_t need = workspace_bytes_for(num_seqs, num_heads, head_dim, nchunks);
  if (need && (!workspace || workspace_bytes < need || !aligned16(workspace)))
    return fail(PA_ERR_WORKSPACE, "decode: workspace of %zu bytes (16-byte aligned) required, got %zu", need,
                workspace ? workspace_bytes : (size_t)0);
  if (fs.slot_mapping) {
    const int64_t row = static_cast<int64_t>(num_kv_heads) * head_dim;
    if (!fs.key || !fs.value) return fail(PA_ERR_INVALID_ARG, "%s: null key or value", who);
    if (fs.key_row_stride < row || fs.value_row_stride < row)
      return fail(PA_ERR_INVALID_ARG, "%s: row strides must be >= num_kv_heads*head_dim", who);
    if (!aligned16(fs.key) || !aligned16(fs.value) || fs.key_row_stride % 8 || fs.value_row_stride % 8)
      return fail(PA_ERR_UNSUPPORTED, "%s: key/value rows must be 16-byte aligned (use pa_store_kvcache + pa_decode)",
                  who);
  }
  DecodeArgs a{};
  a.new_k = fs.key;
  a.new_v = fs.value;
  a.new_k_stride = fs.key_row_stride;
  a.new_v_stride = fs.value_row_stride;
  a.slot_mapping = fs.slot_mapping;
  a.out = out;
  a.o_part = o_part;
  a.lse_part = lse_part;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.block_tables = block_tables;
  a.context_lens = context_lens;
  const size_t rows = static_cast<size_t>(num_seqs) * num_heads * nchunks;
  a.ws_acc = static_cast<float*>(workspace);
  a.ws_ml = need ? reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                            (rows * head_dim * sizeof(float) + 255) / 256 * 256)
                 : nullptr;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.max_context_len = max_context_len;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.chunk_tokens = chunk;
  a.max_chunks = nchunks;
  a.scale = scale;
  return launch_decode(a, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                    int32_t max_context_len, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t kv_chunk_size,
                    void* workspace, size_t workspace_bytes, void* stream) {
  return decode_common("decode", out, nullptr, nullptr, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                       context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                       num_blocks, scale, kv_chunk_size, workspace, workspace_bytes, stream);
}

pa_status pa_decode_partial(float* o_part, float* lse_part, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                            const int32_t* context_lens, int32_t max_context_len, int32_t num_seqs, int32_t num_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            float scale, int32_t kv_chunk_size, void* workspace, size_t workspace_bytes,
                            void* stream) {
  if (!o_part || !lse_part) {
    t_last_error[0] = 0;
    if (num_seqs == 0) return PA_OK;
    return fail(PA_ERR_INVALID_ARG, "decode_partial: null o_part or lse_part");
  }
  return decode_common("decode_partial", nullptr, o_part, lse_part, q, k_cache, v_cache, block_tables,
                       max_blocks_per_seq, context_lens, max_context_len, num_seqs, num_heads, num_kv_heads,
                       head_dim, block_size, num_blocks, scale, kv_chunk_size, workspace, workspace_bytes, stream);
}

pa_status pa_store_decode(void* out, const void* q, const void* key, const void* value, int64_t key_row_stride,
                          int64_t value_row_stride, const int32_t* slot_mapping, void* k_cache, void* v_cache,
                          const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                          int32_t max_context_len, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                          int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                          int32_t kv_chunk_size, void* workspace, size_t workspace_bytes, void* stream) {
  if (!slot_mapping) {
    t_last_error[0] = 0;
    if (num_seqs == 0) return PA_OK;
    return fail(PA_ERR_INVALID_ARG, "store_decode: null slot_mapping");
  }
  FusedStore fs;
  fs.key = key;
  fs.value = value;
  fs.key_row_stride = key_row_stride;
  fs.value_row_stride = value_row_stride;
  fs.slot_mapping = slot_mapping;
  return decode_common("store_decode", out, nullptr, nullptr, q, k_cache, v_cache, block_tables, max_blocks_per_seq,
                       context_lens, max_context_len, num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                       num_blocks, scale, kv_chunk_size, workspace, workspace_bytes, stream, fs);
}

pa_status pa_merge_partials(void* out, const float* o_parts, const float* lse_parts, int32_t num_partials,
                            int32_t num_rows, int32_t head_dim, void* stream) {
  t_last_error[0] = 0;
  if (num_partials <= 0 || num_rows < 0) return fail(PA_ERR_INVALID_ARG, "merge_partials: need num_partials > 0");
  if (head_dim != 64 && head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "merge_partials: head_dim %d not supported (64 or 128)", head_dim);
  if (num_rows == 0) return PA_OK;
  if (!out || !o_parts || !lse_parts) return fail(PA_ERR_INVALID_ARG, "merge_partials: null pointer");
  if ((reinterpret_cast<uintptr_t>(out) & 3u) || (reinterpret_cast<uintptr_t>(o_parts) & 3u) ||
      (reinterpret_cast<uintptr_t>(lse_parts) & 3u))
    return fail(PA_ERR_INVALID_ARG, "merge_partials: pointers must be 4-byte aligned");
  cudaError_t e = launch_merge_lse(out, o_parts, lse_parts, num_partials, num_rows, head_dim,
                                   static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "merge_partials launch: %s", cudaGetErrorString(e));
  return PA_OK;
}

pa_status pa_prefill_varlen(void* out, const void* q, const void* k_cache, const void* v_cache,
                            const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k, int32_t total_q,
                            int32_t max_seqlen_q, int32_t max_seqlen_k, const int32_t* block_tables,
                            int32_t max_blocks_per_seq, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t causal,
                            void* stream) {
  t_last_error[0] = 0;
  if (num_seqs < 0 || total_q < 0) return fail(PA_ERR_INVALID_ARG, "prefill: num_seqs and total_q must be >= 0");
  pa_status st = check_cache_shape("prefill", num_heads, num_kv_heads, head_dim, block_size, num_blocks);
  if (st != PA_OK) return st;
  const int G = num_heads / num_kv_heads;
  if (G != 1 && G != 2 && G != 4 && G != 8)
    return fail(PA_ERR_UNSUPPORTED, "prefill: query heads per kv head = %d not supported (1, 2, 4, 8)", G);
  if (max_seqlen_q < 0 || max_seqlen_k < max_seqlen_q || max_blocks_per_seq <= 0)
    return fail(PA_ERR_INVALID_ARG, "prefill: need 0 <= max_seqlen_q <= max_seqlen_k and max_blocks_per_seq > 0");
  if (!(scale > 0.f) || !isfinite(scale)) return fail(PA_ERR_INVALID_ARG, "prefill: scale must be finite and > 0");
  if (num_seqs == 0 || total_q == 0 || max_seqlen_q == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !cu_seqlens_q || !cu_seqlens_k || !block_tables)
    return fail(PA_ERR_INVALID_ARG, "prefill: null pointer");
  if (!aligned16(q) || !aligned16(out) || !aligned16(k_cache) || !aligned16(v_cache))
    return fail(PA_ERR_INVALID_ARG, "prefill: q, out, k_cache and v_cache must be 16-byte aligned");
  if (num_seqs > 65535) return fail(PA_ERR_UNSUPPORTED, "prefill: more than 65535 sequences");
  PrefillArgs a;
  a.out = out;
  a.q = q;
  a.k_cache = k_cache;
  a.v_cache = v_cache;
  a.cu_seqlens_q = cu_seqlens_q;
  a.cu_seqlens_k = cu_seqlens_k;
  a.block_tables = block_tables;
  a.total_q = total_q;
  a.max_seqlen_q = max_seqlen_q;
  a.max_seqlen_k = max_seqlen_k;
  a.max_blocks_per_seq = max_blocks_per_seq;
  a.num_seqs = num_seqs;
  a.num_heads = num_heads;
  a.num_kv_heads = num_kv_heads;
  a.head_dim = head_dim;
  a.block_size = block_size;
  a.num_blocks = num_blocks;
  a.scale = scale;
  a.causal = causal;
  return launch_prefill(a, static_cast<cudaStream_t>(stream));
}

pa_status pa_device_error(int32_t* code_out, void* stream) {
  t_last_error[0] = 0;
  if (!code_out) return fail(PA_ERR_INVALID_ARG, "device_error: null code_out");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  unsigned int v = 0, zero = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof v, 0, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof zero, 0, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "device_error: %s", cudaGetErrorString(e));
  *code_out = static_cast<int32_t>(v);
  return PA_OK;
}

}  // extern "C"
