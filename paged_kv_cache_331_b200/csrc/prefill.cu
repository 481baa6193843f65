// Varlen causal prefill over a paged KV cache with prefix-cache blocks,
// on the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM).
//
// ("Nano-vLLM 源碼學習" §二.2, prefill stage: varlen attention with prefix
// cache support; "Architektur im Überblick", "Prefill- und
// Decode-Vorbereitung": only uncached tokens are computed, their positions
// start at num_cached_tokens, so query i of a sequence with Lk keys and Lq
// new tokens sits at position Lk - Lq + i.)
//
// Work item = one CTA: (query tile, kv head g, sequence b).  The M = 128 rows
// of the tile pack the G query heads that share kv head g, QP = 128 / G query
// positions each (row r -> head g*G + r / QP, position qt*QP + r % QP), so a
// K/V tile loaded once serves all G heads.  Keys stream in tiles of 128
// tokens gathered through the block table (TMA boxes whose row coordinate is
// block_id * block_size + offset).
//
// Roles (192 threads):
//   warps 0-3  softmax: thread r owns row r (= TMEM lane r); reads S from
//              TMEM, masks, online softmax in the exp2 domain, writes P
//              (bf16, 128B-swizzled K-major) to shared memory, rescales the O
//              accumulator in TMEM when the running max grows, epilogue.
//   warp 4     TMA producer: Q tile once, then K/V tiles, 2 stages.
//   warp 5     TMEM allocator and single-thread MMA issuer:
//              S_j = Q K_j^T  (M128 N128, K = head_dim)  into one of 2 S buffers
//              O  += P_j V_j  (M128 N=head_dim, K = 128 tokens)
// S_{j+1} is issued before waiting for softmax_j, so the tensor core works
// on the next tile while the softmax runs.
//
// The running max moves lazily (only when a row's max grows by more than
// 2^8), and P is double-buffered, so softmax_{j+1} normally waits for neither
// PV_j nor an O correction.
//
// Every wait is time-limited (pa_device.cuh); on a timeout the kernel records
// an error code, drains its copies and MMAs, frees TMEM and returns.
#include <cuda_runtime.h>

#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kBM = 128;         // rows per tile (G heads x QP positions)
constexpr int kBN = 128;         // kv tokens per tile
constexpr int kStages = 2;       // K/V pipeline depth
constexpr int kThreads = 192;
constexpr int kSoftmaxThreads = 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kChunkBytes = kBM * 128;   // one 64-element-wide, 128-row swizzled chunk

struct PrefillParams {
  __nv_bfloat16* out;
  const int32_t* cu_seqlens_q;
  const int32_t* cu_seqlens_k;
  const int32_t* block_tables;
  int32_t max_blocks_per_seq;
  int32_t num_heads;
  int32_t block_size;
  int32_t box_rows;          // min(128, block_size)
  int32_t causal;
  float scale_log2;
  unsigned int* err;
};

template <int D>
struct PrefillSmem {
  static constexpr int kChunks = D / 64;
  static constexpr size_t q_off = 0;
  static constexpr size_t k_off = q_off + kChunks * kChunkBytes;
  static constexpr size_t v_off = k_off + kStages * kChunks * kChunkBytes;
  static constexpr size_t p_off = v_off + kStages * kChunks * kChunkBytes;   // two P buffers
  static constexpr size_t bar_off = p_off + 2 * 2 * kChunkBytes;
  // barriers: q_full, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done[2], mma_done
  static constexpr int kNumBars = 16;
  static constexpr size_t tmem_slot_off = bar_off + kNumBars * 8;
  static constexpr size_t bytes = tmem_slot_off + 16;
  static constexpr size_t alloc_bytes = bytes + 1024;   // slack for 1024-byte alignment
};

// Byte offset of 16-byte unit u (0..7) of row r inside a 128B-swizzled chunk.
__device__ __forceinline__ uint32_t sw128(int r, int u) { return r * 128 + ((u ^ (r & 7)) << 4); }

__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

__device__ __forceinline__ void fadd2(float& d0, float& d1, float a0, float a1) {
  asm("{\n\t.reg .b64 A, C;\n\t"
      "mov.b64 A, {%2, %3};\n\t"
      "mov.b64 C, {%0, %1};\n\t"
      "add.rn.f32x2 C, A, C;\n\t"
      "mov.b64 {%0, %1}, C;\n\t}"
      : "+f"(d0), "+f"(d1)
      : "f"(a0), "f"(a1));
}

// A row's running max only moves when the tile max exceeds it by more than
// 2^kRescaleLog2 (in exp2 units); until then the stale max keeps every
// probability <= 2^kRescaleLog2, exact after the final division, and the O
// accumulator in TMEM needs no correction.
constexpr float kRescaleLog2 = 8.0f;

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p) {
  using Smem = PrefillSmem<D>;
  constexpr int QP = kBM / G;                 // query positions per tile
  constexpr int kChunks = D / 64;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, 0, 0);
  constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, 0, 1);
  constexpr uint32_t kColO = 2 * kBN;        // TMEM columns: S0 [0,128), S1 [128,256), O [256, 256+D)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + Smem::q_off;
  uint8_t* sK = smem + Smem::k_off;
  uint8_t* sV = smem + Smem::v_off;
  uint8_t* sP = smem + Smem::p_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bar_off);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;
  uint64_t* k_empty = bars + 3;
  uint64_t* v_full = bars + 5;
  uint64_t* v_empty = bars + 7;
  uint64_t* s_full = bars + 9;
  uint64_t* p_full = bars + 11;
  uint64_t* o_done = bars + 13;
  uint64_t* mma_done = bars + 15;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::tmem_slot_off);

  const int b = blockIdx.z, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cq0 = __ldg(p.cu_seqlens_q), cq_b = __ldg(p.cu_seqlens_q + b), cq_b1 = __ldg(p.cu_seqlens_q + b + 1);
  const int Lq = cq_b1 - cq_b;
  const int Lk = __ldg(p.cu_seqlens_k + b + 1) - __ldg(p.cu_seqlens_k + b);
  const int ntq = (Lq + QP - 1) / QP;
  const int qt = ntq - 1 - static_cast<int>(blockIdx.x);   // longest tiles of a sequence first
  if (qt < 0 || Lk < Lq || Lk <= 0) return;
  const int q_row0 = cq_b - cq0;                           // first q/out row of this sequence
  const int pos_off = Lk - Lq;                             // position of query 0
  const int i_last = min(Lq, (qt + 1) * QP) - 1;
  const int n_keys = p.causal ? min(Lk, pos_off + i_last + 1) : Lk;   // keys any row of the tile may see
  const int nt = (n_keys + kBN - 1) / kBN;
  // keys every row of the tile sees: tiles entirely below this need no mask
  const int full_keys = p.causal ? min(Lk, pos_off + qt * QP + 1) : Lk;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], kSoftmaxThreads);
      mbar_init(&o_done[s], 1);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    // ---------------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      mbar_arrive_expect_tx(q_full, kChunks * kChunkBytes);
      for (int hh = 0; hh < G; ++hh)
        for (int c = 0; c < kChunks; ++c)
          tma_load_3d(sQ + c * kChunkBytes + hh * QP * 128, &tmQ, q_full, c * 64, g * G + hh, q_row0 + qt * QP);
      const int32_t* bt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq;
      const int bs_shift = __ffs(p.block_size) - 1;
      const int nblk_valid = (Lk + p.block_size - 1) >> bs_shift;
      // One K or V tile: boxes past the last block of the sequence are skipped
      // (their table entries may be -1).
      auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int j) {
        int nbox = kBN / p.box_rows;
        while (nbox > 0 && ((j * kBN + (nbox - 1) * p.box_rows) >> bs_shift) >= nblk_valid) --nbox;
        mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbox * p.box_rows * 128 * kChunks));
        for (int k = 0; k < nbox; ++k) {
          const int tok = j * kBN + k * p.box_rows;
          const int blk = __ldg(bt + (tok >> bs_shift));
          const int row = (blk << bs_shift) + (tok & (p.block_size - 1));
          for (int c = 0; c < kChunks; ++c) tma_load_3d(dst + c * kChunkBytes + k * p.box_rows * 128, map, bar, c * 64, g, row);
        }
      };
      // K runs one tile ahead of V: K_j's slot frees as soon as S_j is computed,
      // V_j's only after PV_j.
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      if (nt > 0 && (ok = mbar_wait(&k_empty[0], 1, p.err))) {
        load_tile(&tmK, sK, &k_full[0], 0);
        k_issued = 1;
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          const int s1 = (j + 1) % kStages;
          if (!(ok = mbar_wait(&k_empty[s1], (((j + 1) / kStages) & 1) ^ 1, p.err))) break;
          load_tile(&tmK, sK + s1 * kChunks * kChunkBytes, &k_full[s1], j + 1);
          k_issued = j + 2;
        }
        const int s = j % kStages;
        if (!(ok = mbar_wait(&v_empty[s], ((j / kStages) & 1) ^ 1, p.err))) break;
        load_tile(&tmV, sV + s * kChunks * kChunkBytes, &v_full[s], j);
        v_issued = j + 1;
      }
      mbar_wait(q_full, 0, p.err, kErrDrainTimeout);
      for (int j = max(0, k_issued - kStages); j < k_issued; ++j)
        mbar_wait(&k_full[j % kStages], (j / kStages) & 1, p.err, kErrDrainTimeout);
      for (int j = max(0, v_issued - kStages); j < v_issued; ++j)
        mbar_wait(&v_full[j % kStages], (j / kStages) & 1, p.err, kErrDrainTimeout);
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, p.err);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV), p_base = smem_u32(sP);
      auto issue_s = [&](int j) {   // S[j%2] = Q K_j^T
        const int s = j % kStages;
        const uint32_t d_tmem = tmem + (j & 1) * kBN;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(q_base + c * kChunkBytes + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(k_base + (s * kChunks + c) * kChunkBytes + kk * 32, 16, 1024, 2);
            tc_mma_ss(d_tmem, ad, bd, kIdescS, (c | kk) != 0);
          }
        tc_commit(&s_full[j & 1]);
        tc_commit(&k_empty[s]);
      };
      if (ok && nt > 0) {
        ok = mbar_wait(&k_full[0], 0, p.err);
        if (ok) {
          tc_fence_after();
          issue_s(0);
        }
      }
      for (int j = 0; ok && j < nt; ++j) {
        if (j + 1 < nt) {
          const int s1 = (j + 1) % kStages;
          if (!(ok = mbar_wait(&k_full[s1], ((j + 1) / kStages) & 1, p.err))) break;
          tc_fence_after();
          issue_s(j + 1);
        }
        const int s = j % kStages;
        if (!(ok = mbar_wait(&v_full[s], (j / kStages) & 1, p.err))) break;
        if (!(ok = mbar_wait(&p_full[j & 1], (j >> 1) & 1, p.err))) break;
        tc_fence_after();
        const uint32_t pb = p_base + (j & 1) * 2 * kChunkBytes;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {   // O += P_j V_j, 16 tokens per MMA
          const uint64_t ad = smem_desc(pb + (kk >> 2) * kChunkBytes + (kk & 3) * 32, 16, 1024, 2);
          const uint64_t bd = smem_desc(v_base + s * kChunks * kChunkBytes + kk * 2048, kChunkBytes, 1024, 2);
          tc_mma_ss(tmem + kColO, ad, bd, kIdescO, (j | kk) != 0);
        }
        tc_commit(&o_done[j & 1]);
        tc_commit(&v_empty[s]);
      }
      // wait for every MMA this thread issued before TMEM can be released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, p.err, kErrDrainTimeout);
    }
  } else {
    // ------------------------------------------------------------------ softmax --
    const int r = threadIdx.x;                 // row / TMEM lane
    const int hh = r / QP;
    const int i = qt * QP + (r % QP);          // query index within the sequence
    const bool row_valid = i < Lq;
    const int p_row = p.causal ? min(pos_off + i, Lk - 1) : Lk - 1;   // last visible key
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                   // running max in raw score units
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      if (!(ok = mbar_wait_warp(&s_full[j & 1], (j >> 1) & 1, p.err))) break;
      tc_fence_after();
      float x[kBN];
      {
        uint32_t v[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(lane_base + (j & 1) * kBN + c * 32, v[c]);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) x[c * 32 + e] = __uint_as_float(v[c][e]);
      }
      const int col0 = j * kBN;
      if (col0 + kBN > full_keys) {   // tile reaches past some row's last visible key
#pragma unroll
        for (int e = 0; e < kBN; ++e)
          if (col0 + e > p_row) x[e] = -INFINITY;
      }
      float mt = -INFINITY;
#pragma unroll
      for (int e = 0; e < kBN; e += 2) mt = max3(mt, x[e], x[e + 1]);
      // lazy rescale: move the max only when it grew by more than 2^kRescaleLog2
      const bool grow = (mt - m_run) * sl2 > kRescaleLog2;
      const float m_new = grow ? mt : m_run;
      const float alpha = grow ? fast_exp2((m_run - m_new) * sl2) : 1.f;
      const float nms = -m_new * sl2;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int e = 0; e < kBN; e += 2) {
        float a0 = nms, a1 = nms;
        ffma2(a0, a1, x[e], x[e + 1], sl2, sl2);
        const float p0 = fast_exp2(a0), p1 = fast_exp2(a1);
        fadd2(rs0, rs1, p0, p1);
        pk[e / 2] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * alpha + (rs0 + rs1);
      // P buffer j%2 was last read by PV_{j-2}
      if (j >= 2 && !(ok = mbar_wait_warp(&o_done[j & 1], ((j - 2) >> 1) & 1, p.err))) break;
      uint8_t* pbuf = sP + (j & 1) * 2 * kChunkBytes;
#pragma unroll
      for (int u = 0; u < kBN / 8; ++u) {
        uint8_t* dst = pbuf + (u >> 3) * kChunkBytes + sw128(r, u & 7);
        *reinterpret_cast<uint4*>(dst) = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
      }
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // rescale O rows whose max moved (alpha = 1 elsewhere) once PV_{j-1} has landed
        if (!(ok = mbar_wait_warp(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, p.err))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + kColO + c * 32, v);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(lane_base + kColO + c * 32, v);
        }
        tc_wait_st();
      }
      m_run = m_new;
      if (col0 + kBN > Lk) {
        // last tile reaches past the context: zero V rows >= Lk (they may hold
        // anything, and 0 * NaN would poison the PV product)
        const int s = j % kStages;
        if (!(ok = mbar_wait_warp(&v_full[s], (j / kStages) & 1, p.err))) break;
        if (col0 + r >= Lk) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(sV + (s * kChunks + c) * kChunkBytes + r * 128 + u * 16) =
                  make_uint4(0, 0, 0, 0);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(&p_full[j & 1]);
    }
    if (ok && nt > 0) ok = mbar_wait_warp(&o_done[(nt - 1) & 1], ((nt - 1) >> 1) & 1, p.err);
    tc_fence_after();
    if (ok) {   // warp-uniform: every lane takes part in the TMEM loads
      const float inv = 1.f / l_run;
      __nv_bfloat16* orow =
          p.out + (static_cast<int64_t>(q_row0 + i) * p.num_heads + g * G + hh) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_base + kColO + c * 32, v);
        tc_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * u + 0]) * inv, __uint_as_float(v[8 * u + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(v[8 * u + 2]) * inv, __uint_as_float(v[8 * u + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(v[8 * u + 4]) * inv, __uint_as_float(v[8 * u + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(v[8 * u + 6]) * inv, __uint_as_float(v[8 * u + 7]) * inv);
          if (row_valid) *reinterpret_cast<uint4*>(orow + c * 32 + u * 8) = w;
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 5) tmem_dealloc(tmem, kTmemCols);
}

template <int D, int G>
pa_status launch_typed(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                       const PrefillParams& p, dim3 grid, cudaStream_t stream) {
  using Smem = PrefillSmem<D>;
  static int configured_device = -1;
  const DeviceInfo* di = current_device_info();
  if (configured_device != di->device) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Smem::alloc_bytes));
    if (e != cudaSuccess) {
      set_last_error("cudaFuncSetAttribute(prefill): %s", cudaGetErrorString(e));
      return PA_ERR_CUDA;
    }
    configured_device = di->device;
  }
  prefill_kernel<D, G><<<grid, kThreads, Smem::alloc_bytes, stream>>>(tmQ, tmK, tmV, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("prefill launch: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <int D>
pa_status dispatch_group(int G, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const PrefillParams& p, dim3 grid, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_typed<D, 1>(tmQ, tmK, tmV, p, grid, stream);
    case 2: return launch_typed<D, 2>(tmQ, tmK, tmV, p, grid, stream);
    case 4: return launch_typed<D, 4>(tmQ, tmK, tmV, p, grid, stream);
    case 8: return launch_typed<D, 8>(tmQ, tmK, tmV, p, grid, stream);
    default: break;
  }
  set_last_error("prefill: query heads per kv head = %d not supported", G);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

pa_status launch_prefill(const PrefillArgs& a, cudaStream_t stream) {
  const int G = a.num_heads / a.num_kv_heads;
  const int QP = kBM / G;
  const int box_rows = a.block_size < kBN ? a.block_size : kBN;
  CUtensorMap tmQ, tmK, tmV;
  const uint64_t s1 = static_cast<uint64_t>(a.head_dim) * 2;
  const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.block_size;
  if (!encode_bf16_3d(&tmQ, a.q, a.head_dim, a.num_heads, a.total_q, s1, s1 * a.num_heads, 64, 1, QP,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16_3d(&tmK, a.k_cache, a.head_dim, a.num_kv_heads, rows, s1, s1 * a.num_kv_heads, 64, 1, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16_3d(&tmV, a.v_cache, a.head_dim, a.num_kv_heads, rows, s1, s1 * a.num_kv_heads, 64, 1, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return PA_ERR_INVALID_ARG;
  PrefillParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.cu_seqlens_q = a.cu_seqlens_q;
  p.cu_seqlens_k = a.cu_seqlens_k;
  p.block_tables = a.block_tables;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.num_heads = a.num_heads;
  p.block_size = a.block_size;
  p.box_rows = box_rows;
  p.causal = a.causal ? 1 : 0;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = current_device_info()->error_word;
  const dim3 grid(static_cast<unsigned>((a.max_seqlen_q + QP - 1) / QP), static_cast<unsigned>(a.num_kv_heads),
                  static_cast<unsigned>(a.num_seqs));
  return a.head_dim == 128 ? dispatch_group<128>(G, tmQ, tmK, tmV, p, grid, stream)
                           : dispatch_group<64>(G, tmQ, tmK, tmV, p, grid, stream);
}

}  // namespace pa
