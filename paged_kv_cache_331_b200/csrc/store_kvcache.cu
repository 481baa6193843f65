// store_kvcache: scatter the new tokens' K/V rows into their cache slots.
//
// ("Nano-vLLM 源碼學習" §二.2: a store_kvcache kernel writes key and value
// into the cache; "Architektur im Überblick", "Prefill- und
// Decode-Vorbereitung": one slot per new token.)
//
// A pure copy bound by HBM bandwidth.  One warp moves one row (all kv heads
// of one token, K or V): every lane issues all of its 16-byte loads before
// its stores, so a warp keeps the whole row in flight, and consecutive lanes
// touch consecutive 16-byte chunks (512 contiguous bytes per warp access).
// A row whose base or stride is not 16-byte aligned falls back to 4-byte or
// 2-byte accesses with the same structure.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kStoreThreads = 256;
constexpr int kMaxChunksPerLane = 8;   // 16-byte chunks held per lane per pass

template <typename V>
__device__ __forceinline__ V load_row_chunk(const V* p);

template <>
__device__ __forceinline__ uint4 load_row_chunk<uint4>(const uint4* p) { return ld_nc_v4(p); }
template <>
__device__ __forceinline__ uint32_t load_row_chunk<uint32_t>(const uint32_t* p) { return __ldg(p); }
template <>
__device__ __forceinline__ uint16_t load_row_chunk<uint16_t>(const uint16_t* p) { return __ldg(p); }

// One warp per (token, K|V) row.  `row_units` = row length in units of V.
template <typename V>
__global__ void __launch_bounds__(kStoreThreads) store_kvcache_kernel(
    const V* __restrict__ key, const V* __restrict__ value, int64_t key_stride_units, int64_t value_stride_units,
    V* __restrict__ k_cache, V* __restrict__ v_cache, const int32_t* __restrict__ slot_mapping, int32_t num_tokens,
    int32_t row_units, int64_t num_slots, unsigned int* __restrict__ err) {
  const int64_t wid = (static_cast<int64_t>(blockIdx.x) * kStoreThreads + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (wid >= 2 * static_cast<int64_t>(num_tokens)) return;
  const int64_t t = wid >> 1;
  const bool is_v = wid & 1;
  const int32_t slot = __ldg(slot_mapping + t);
  if (slot < 0 || slot >= num_slots) {   // -1: skip; anything else out of range is reported, never written
    if (slot != -1 && lane == 0) record_error(err, kErrOutOfCache);
    return;
  }
  const V* src = is_v ? value + t * value_stride_units : key + t * key_stride_units;
  V* dst = (is_v ? v_cache : k_cache) + static_cast<int64_t>(slot) * row_units;
  for (int base = 0; base < row_units; base += 32 * kMaxChunksPerLane) {
    V r[kMaxChunksPerLane];
#pragma unroll
    for (int i = 0; i < kMaxChunksPerLane; ++i) {
      const int u = base + i * 32 + lane;
      if (u < row_units) r[i] = load_row_chunk<V>(src + u);
    }
#pragma unroll
    for (int i = 0; i < kMaxChunksPerLane; ++i) {
      const int u = base + i * 32 + lane;
      if (u < row_units) dst[u] = r[i];
    }
  }
}

template <typename V>
cudaError_t launch_typed(const void* key, const void* value, int64_t key_row_stride, int64_t value_row_stride,
                         void* k_cache, void* v_cache, const int32_t* slot_mapping, int32_t num_tokens,
                         int32_t row_elems, int64_t num_slots, cudaStream_t stream) {
  constexpr int kElemsPerUnit = sizeof(V) / 2;
  const int64_t warps = 2 * static_cast<int64_t>(num_tokens);
  const int64_t blocks = (warps * 32 + kStoreThreads - 1) / kStoreThreads;
  store_kvcache_kernel<V><<<static_cast<unsigned>(blocks), kStoreThreads, 0, stream>>>(
      static_cast<const V*>(key), static_cast<const V*>(value), key_row_stride / kElemsPerUnit,
      value_row_stride / kElemsPerUnit, static_cast<V*>(k_cache), static_cast<V*>(v_cache), slot_mapping,
      num_tokens, row_elems / kElemsPerUnit, num_slots, current_device_info()->error_word);
  return cudaGetLastError();
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

}  // namespace

cudaError_t launch_store_kvcache(const void* key, const void* value, int64_t key_row_stride,
                                 int64_t value_row_stride, void* k_cache, void* v_cache,
                                 const int32_t* slot_mapping, int32_t num_tokens, int32_t row_elems,
                                 int64_t num_slots, cudaStream_t stream) {
  auto fits = [&](size_t unit_bytes) {
    const size_t e = unit_bytes / 2;
    return aligned(key, unit_bytes) && aligned(value, unit_bytes) && aligned(k_cache, unit_bytes) &&
           aligned(v_cache, unit_bytes) && key_row_stride % e == 0 && value_row_stride % e == 0 && row_elems % e == 0;
  };
  if (fits(16))
    return launch_typed<uint4>(key, value, key_row_stride, value_row_stride, k_cache, v_cache, slot_mapping,
                               num_tokens, row_elems, num_slots, stream);
  if (fits(4))
    return launch_typed<uint32_t>(key, value, key_row_stride, value_row_stride, k_cache, v_cache, slot_mapping,
                                  num_tokens, row_elems, num_slots, stream);
  return launch_typed<uint16_t>(key, value, key_row_stride, value_row_stride, k_cache, v_cache, slot_mapping,
                                num_tokens, row_elems, num_slots, stream);
}

}  // namespace pa
