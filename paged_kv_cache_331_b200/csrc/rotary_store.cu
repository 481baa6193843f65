// Rotary position embedding fused with store_kvcache.
//
// ("Nano-vLLM 源碼學習", layers, 7 rotary_embedding.py: RotaryEmbedding adds
// the position to q and k through sines and cosines held in a cos/sin cache;
// "Architektur im Überblick", Attention-Mechanismus: the attention layer
// applies rotary_emb to q and k, then its attention stores k and v into the
// paged cache with store_kvcache.)
//
// The rotation pairs element i with element i + D/2 of a head (RoFormer's
// rotation in the half-split layout):
//   y_i       = x_i cos(p theta_i) - x_{i+D/2} sin(p theta_i)
//   y_{i+D/2} = x_{i+D/2} cos(p theta_i) + x_i sin(p theta_i)
// with cos/sin taken from row p of a float table [max_position, D] (cos in
// the first D/2 columns, sin in the last D/2).
//
// One pass over the new tokens, bound by HBM bandwidth: each token's query
// rows are rotated into q_out, its key rows rotated and written to their
// cache slot, its value rows copied there.  A group of D/16 threads owns one
// head row; thread j of the group moves elements [8j, 8j+8) of both halves
// with 16-byte accesses, so a warp covers 32/(D/16) whole consecutive rows.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kRotThreads = 256;

__device__ __forceinline__ float4 ld_nc_f4(const float* p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "l"(p));
  return v;
}

// Rotate 8 pairs (lo[i], hi[i]) by the angles whose cos/sin are c[i], s[i].
__device__ __forceinline__ void rotate8(uint4& lo, uint4& hi, const float* c, const float* s) {
  uint32_t* L = reinterpret_cast<uint32_t*>(&lo);
  uint32_t* H = reinterpret_cast<uint32_t*>(&hi);
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const float a0 = bf16lo(L[w]), a1 = bf16hi(L[w]);
    const float b0 = bf16lo(H[w]), b1 = bf16hi(H[w]);
    const float c0 = c[2 * w], c1 = c[2 * w + 1], s0 = s[2 * w], s1 = s[2 * w + 1];
    const float ylo0 = __fmaf_rn(a0, c0, -(b0 * s0)), ylo1 = __fmaf_rn(a1, c1, -(b1 * s1));
    const float yhi0 = __fmaf_rn(b0, c0, a0 * s0), yhi1 = __fmaf_rn(b1, c1, a1 * s1);
    L[w] = pack_bf16x2(ylo0, ylo1);
    H[w] = pack_bf16x2(yhi0, yhi1);
  }
}

template <int D>
__global__ void __launch_bounds__(kRotThreads) rotary_store_kernel(RotaryArgs a, unsigned int* err) {
  constexpr int TPR = D / 16;   // threads per head row
  constexpr int HALF = D / 2;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * kRotThreads + threadIdx.x;
  const int64_t row = gid / TPR;
  const int j = static_cast<int>(gid % TPR);
  const int rows_per_token = a.num_heads + 2 * a.num_kv_heads;
  if (row >= static_cast<int64_t>(a.num_tokens) * rows_per_token) return;
  const int64_t t = row / rows_per_token;
  const int r = static_cast<int>(row % rows_per_token);
  const int64_t kv_row = static_cast<int64_t>(a.num_kv_heads) * D;
  const int e0 = 8 * j;   // first element of this thread in each half

  if (r >= a.num_heads + a.num_kv_heads) {   // value row: a copy into the slot
    const int32_t slot = __ldg(a.slot_mapping + t);
    if (slot < 0 || slot >= a.num_slots) {   // -1: skip; anything else is reported, never written
      if (slot != -1 && j == 0) record_error(err, kErrOutOfCache);
      return;
    }
    const int h = r - a.num_heads - a.num_kv_heads;
    const uint16_t* src = static_cast<const uint16_t*>(a.value) + t * a.value_row_stride + static_cast<int64_t>(h) * D;
    uint16_t* dst = static_cast<uint16_t*>(a.v_cache) + slot * kv_row + static_cast<int64_t>(h) * D;
    const uint4 lo = ld_nc_v4(reinterpret_cast<const uint4*>(src + e0));
    const uint4 hi = ld_nc_v4(reinterpret_cast<const uint4*>(src + HALF + e0));
    *reinterpret_cast<uint4*>(dst + e0) = lo;
    *reinterpret_cast<uint4*>(dst + HALF + e0) = hi;
    return;
  }

  const bool is_q = r < a.num_heads;
  int32_t slot = 0;
  if (!is_q) {
    slot = __ldg(a.slot_mapping + t);
    if (slot < 0 || slot >= a.num_slots) {
      if (slot != -1 && j == 0) record_error(err, kErrOutOfCache);
      return;
    }
  }
  const int32_t pos = __ldg(a.positions + t);
  if (pos < 0 || pos >= a.max_position) {
    record_error(err, kErrBadPosition);
    return;
  }
  const uint16_t* src = is_q ? static_cast<const uint16_t*>(a.q) + t * a.q_row_stride + static_cast<int64_t>(r) * D
                           : static_cast<const uint16_t*>(a.key) + t * a.key_row_stride +
                                 static_cast<int64_t>(r - a.num_heads) * D;
  uint4 lo = ld_nc_v4(reinterpret_cast<const uint4*>(src + e0));
  uint4 hi = ld_nc_v4(reinterpret_cast<const uint4*>(src + HALF + e0));
  const float* cs = a.cos_sin + static_cast<int64_t>(pos) * D;
  float c[8], s[8];
  *reinterpret_cast<float4*>(c) = ld_nc_f4(cs + e0);
  *reinterpret_cast<float4*>(c + 4) = ld_nc_f4(cs + e0 + 4);
  *reinterpret_cast<float4*>(s) = ld_nc_f4(cs + HALF + e0);
  *reinterpret_cast<float4*>(s + 4) = ld_nc_f4(cs + HALF + e0 + 4);
  rotate8(lo, hi, c, s);
  uint16_t* dst = is_q ? static_cast<uint16_t*>(a.q_out) + (t * a.num_heads + r) * D
                     : static_cast<uint16_t*>(a.k_cache) + slot * kv_row + static_cast<int64_t>(r - a.num_heads) * D;
  *reinterpret_cast<uint4*>(dst + e0) = lo;
  *reinterpret_cast<uint4*>(dst + HALF + e0) = hi;
}

// One thread per (position, frequency): the angle p * base^(-2i/D) in double,
// its cosine and sine rounded once to float.
__global__ void rotary_table_kernel(float* table, int32_t max_position, int32_t head_dim, double base) {
  const int half = head_dim / 2;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (gid >= static_cast<int64_t>(max_position) * half) return;
  const int32_t p = static_cast<int32_t>(gid / half);
  const int i = static_cast<int>(gid % half);
  const double theta = pow(base, -2.0 * i / head_dim);
  double sn, cn;
  sincos(static_cast<double>(p) * theta, &sn, &cn);
  table[static_cast<int64_t>(p) * head_dim + i] = static_cast<float>(cn);
  table[static_cast<int64_t>(p) * head_dim + half + i] = static_cast<float>(sn);
}

}  // namespace

cudaError_t launch_rotary_store(const RotaryArgs& a, cudaStream_t stream) {
  const int64_t rows = static_cast<int64_t>(a.num_tokens) * (a.num_heads + 2 * a.num_kv_heads);
  const int64_t threads = rows * (a.head_dim / 16);
  const unsigned blocks = static_cast<unsigned>((threads + kRotThreads - 1) / kRotThreads);
  unsigned int* err = current_device_info()->error_word;
  if (a.head_dim == 128)
    rotary_store_kernel<128><<<blocks, kRotThreads, 0, stream>>>(a, err);
  else
    rotary_store_kernel<64><<<blocks, kRotThreads, 0, stream>>>(a, err);
  return cudaGetLastError();
}

cudaError_t launch_rotary_table(float* table, int32_t max_position, int32_t head_dim, double base,
                                cudaStream_t stream) {
  const int64_t n = static_cast<int64_t>(max_position) * (head_dim / 2);
  const unsigned blocks = static_cast<unsigned>((n + 255) / 256);
  rotary_table_kernel<<<blocks, 256, 0, stream>>>(table, max_position, head_dim, base);
  return cudaGetLastError();
}

}  // namespace pa
