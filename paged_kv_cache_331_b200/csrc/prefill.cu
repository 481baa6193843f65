// Varlen causal prefill over a paged KV cache with prefix-cache blocks,
// on the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM).
//
// ("Nano-vLLM 源碼學習" §二.2, prefill stage: varlen attention with prefix
// cache support; "Architektur im Überblick", "Prefill- und
// Decode-Vorbereitung": only uncached tokens are computed, their positions
// start at num_cached_tokens, so query i of a sequence with Lk keys and Lq
// new tokens sits at position Lk - Lq + i.)
//
// Work item = one CTA: two query tiles (A and B) of one (kv head g, sequence
// b).  The M = 128 rows of a tile pack the G query heads that share kv head
// g, QP = 128 / G query positions each (row r -> head g*G + r / QP,
// position qt*QP + r % QP), so every K/V tile loaded serves 2*G heads-tiles.
// Keys stream in tiles of 128 tokens gathered through the block table (TMA
// boxes whose row coordinate is block_id * block_size + offset).
//
// Roles (384 threads):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r of a
//              group owns row r (= TMEM lane r); it reads S from TMEM, masks,
//              runs the online softmax in the exp2 domain (part of the
//              exponentials on the FMA pipe), writes P as bf16 pairs over the
//              first half of its own S columns, rescales its O row in TMEM when
//              the running max grows, and does the epilogue.
//   warp 8     TMA producer: both Q tiles once, then K and V tiles in rings
//              (K one tile ahead).
//   warps 10-11 idle (they complete the third warpgroup, whose registers
//              the softmax warpgroups borrow through setmaxnreg).
//   warp 9     TMEM allocator and single-thread MMA issuer, in the order
//              QK_A0 QK_B0 | PV_A0 QK_A1 PV_B0 QK_B1 | PV_A1 QK_A2 PV_B1 ...
//              so that while one group runs its softmax the tensor core works
//              on the other tile (S = Q K^T: M128 N128 K=head_dim from shared
//              memory; O += P V: M128 N=head_dim K=128 with P from TMEM).
// MMAs of one CTA execute in issue order, so the commit that reports S_X(j+1)
// also reports PV_X(j): when a group sees its next S, its P columns and its O
// accumulator are free.
//
// The running max moves lazily (only when a row's max grows by more than
// 2^8), so O in TMEM is rarely corrected.
//
// Every wait is time-limited (pa_device.cuh); on a timeout the kernel records
// an error code, drains its copies and MMAs, frees TMEM and returns.
#include <cuda_runtime.h>

#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kBM = 128;            // rows per query tile (G heads x QP positions)
constexpr int kBN = 128;            // kv tokens per tile
constexpr int kKStages = 2;         // K ring depth
constexpr int kSoftmaxWarps = 8;    // two groups of four: tile A, tile B
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;   // third warpgroup: producer, MMA, two idle warps
// Registers: the block launches with 168 per thread (384 x 168 = 64512); the
// third warpgroup gives most of its share to the two softmax warpgroups:
// 256 x 216 + 128 x 72 = 64512.
constexpr uint32_t kSoftmaxRegs = 216;
constexpr uint32_t kControlRegs = 72;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= 384 * 168, "register split exceeds the launch budget");
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
  static constexpr int kVStages = D == 128 ? 3 : 4;    // V ring depth
  static constexpr size_t q_off = 0;                    // Q_A then Q_B
  static constexpr size_t k_off = q_off + 2 * kChunks * kChunkBytes;
  static constexpr size_t v_off = k_off + kKStages * kChunks * kChunkBytes;
  static constexpr size_t bar_off = v_off + kVStages * kChunks * kChunkBytes;
  // barriers: q_full, k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2], o_done[2], mma_done
  static constexpr int kNumBars = 1 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1;
  static constexpr size_t tmem_slot_off = bar_off + kNumBars * 8;
  static constexpr size_t bytes = tmem_slot_off + 16;
  static_assert(bytes <= 232448, "shared memory budget (227 KB per CTA)");
  // epilogue staging: group A in the K ring, group B in the V ring, 128 rows of D*2+16 bytes
  static_assert(kKStages * kChunks * kChunkBytes >= kBM * (D * 2 + 16), "staging A");
  static_assert(kVStages * kChunks * kChunkBytes >= kBM * (D * 2 + 16), "staging B");
};

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

// 2^x on the FMA pipe, for the share of the softmax exponentials that the
// MUFU unit (16 results per clock per SM) cannot absorb.  Cody-Waite style:
// x = n + f with n = round(x) (added to 1.5*2^23 so that n lands in the low
// mantissa bits), f in [-1/2, 1/2]; 2^f from a cubic whose coefficients were
// fitted here by iteratively reweighted least squares on Chebyshev nodes of
// [-1/2, 1/2] (max relative error 7.5e-5, below bf16 resolution); n is then
// added to the exponent field.  x is clamped to -125 so the exponent stays
// normal; such inputs give ~2^-125 instead of 0, far below anything that can
// change a bf16 result.
constexpr float kExpC0 = 0.9999280571937561f;
constexpr float kExpC1 = 0.6932609677314758f;
constexpr float kExpC2 = 0.2426111251115799f;
constexpr float kExpC3 = 0.055171653628349304f;
constexpr float kRoundMagic = 12582912.0f;   // 1.5 * 2^23

__device__ __forceinline__ void exp2_poly2(float& y0, float& y1, float x0, float x1) {
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  float t0 = kRoundMagic, t1 = kRoundMagic;
  fadd2(t0, t1, x0, x1);                             // t = x + magic (round to nearest integer)
  float f0 = x0, f1 = x1;
  ffma2(f0, f1, t0 - kRoundMagic, t1 - kRoundMagic, -1.f, -1.f);   // f = x - n
  float p0 = kExpC2, p1 = kExpC2;
  ffma2(p0, p1, f0, f1, kExpC3, kExpC3);
  float q0 = kExpC1, q1 = kExpC1;
  ffma2(q0, q1, p0, p1, f0, f1);
  float r0 = kExpC0, r1 = kExpC0;
  ffma2(r0, r1, q0, q1, f0, f1);
  y0 = __int_as_float(__float_as_int(r0) + (__float_as_int(t0) << 23));
  y1 = __int_as_float(__float_as_int(r1) + (__float_as_int(t1) << 23));
}

// Every kEmuEvery-th pair of softmax exponentials uses exp2_poly2.
constexpr int kEmuEvery = 8;   // pairs k with k % kEmuEvery >= kEmuFrom are emulated
constexpr int kEmuFrom = 5;

__device__ __forceinline__ void bulk_store_s2g(void* gdst, const void* ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(smem_u32(ssrc)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

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
  constexpr int kVStages = Smem::kVStages;
  constexpr uint32_t kIdescS = idesc_bf16_f32(kBM, kBN, 0, 0);
  constexpr uint32_t kIdescO = idesc_bf16_f32(kBM, D, 0, 1);
  // TMEM columns: S_A [0,128), S_B [128,256), O_A [256, 256+D), O_B [256+D, 256+2D);
  // P_X (bf16 pairs) overwrites the first 64 columns of S_X.
  constexpr uint32_t kColO = 2 * kBN;
  static_assert(kColO + 2 * D <= kTmemCols, "TMEM budget");

  // 128B-swizzled TMA tiles and MMA operands need 1024-byte alignment; the
  // kernel declares no static shared memory, so the dynamic window starts
  // aligned.  Checked anyway: a misaligned base is reported, never used.
  extern __shared__ __align__(1024) uint8_t smem[];
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_error(p.err, kErrSmemAlign);
    return;
  }
  uint8_t* sQ = smem + Smem::q_off;
  uint8_t* sK = smem + Smem::k_off;
  uint8_t* sV = smem + Smem::v_off;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Smem::bar_off);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  uint64_t* s_full = v_empty + kVStages;     // [2]: tile A, tile B
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_done = p_full + 2;             // [2]
  uint64_t* mma_done = o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::tmem_slot_off);

  const int b = blockIdx.z, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cq0 = __ldg(p.cu_seqlens_q), cq_b = __ldg(p.cu_seqlens_q + b), cq_b1 = __ldg(p.cu_seqlens_q + b + 1);
  const int Lq = cq_b1 - cq_b;
  const int Lk = __ldg(p.cu_seqlens_k + b + 1) - __ldg(p.cu_seqlens_k + b);
  const int ntq = (Lq + QP - 1) / QP;                     // query tiles of this sequence
  const int npairs = (ntq + 1) / 2;
  const int pair = npairs - 1 - static_cast<int>(blockIdx.x);   // longest pairs of a sequence first
  if (pair < 0 || Lk < Lq || Lk <= 0) return;
  // tile A is the later (longer) one of the pair; a pair of one tile has no B
  const bool has_b = 2 * pair + 1 < ntq;
  const int qt[2] = {has_b ? 2 * pair + 1 : 2 * pair, 2 * pair};
  const int q_row0 = cq_b - cq0;                            // first q/out row of this sequence
  const int pos_off = Lk - Lq;                              // position of query 0
  int nt[2], full_keys[2];
  for (int x = 0; x < 2; ++x) {
    const int i_last = min(Lq, (qt[x] + 1) * QP) - 1;
    const int n_keys = p.causal ? min(Lk, pos_off + i_last + 1) : Lk;
    nt[x] = (n_keys + kBN - 1) / kBN;
    full_keys[x] = p.causal ? min(Lk, pos_off + qt[x] * QP + 1) : Lk;   // keys every row of the tile sees
  }
  if (!has_b) nt[1] = 0;
  const int ntA = nt[0], ntB = nt[1];        // ntB <= ntA

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kKStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < kVStages; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 128);
      mbar_init(&o_done[x], 1);
    }
    mbar_init(mma_done, 1);
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp >= kSoftmaxWarps) {
   regs_decrease<kControlRegs>();
   if (warp == kProducerWarp) {
    // ---------------------------------------------------------------- producer --
    if (lane == 0) {
      prefetch_tensormap(&tmQ);
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const int ntiles_q = has_b ? 2 : 1;
      mbar_arrive_expect_tx(q_full, ntiles_q * kChunks * kChunkBytes);
      for (int x = 0; x < ntiles_q; ++x)
        for (int hh = 0; hh < G; ++hh)
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(sQ + (x * kChunks + c) * kChunkBytes + hh * QP * 128, &tmQ, q_full, c * 64, g * G + hh,
                        q_row0 + qt[x] * QP);
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
          for (int c = 0; c < kChunks; ++c)
            tma_load_3d(dst + c * kChunkBytes + k * p.box_rows * 128, map, bar, c * 64, g, row);
        }
      };
      // K runs one tile ahead of V.
      int k_issued = 0, v_issued = 0;
      bool ok = true;
      if (ntA > 0 && (ok = mbar_wait(&k_empty[0], 1, p.err))) {
        load_tile(&tmK, sK, &k_full[0], 0);
        k_issued = 1;
      }
      for (int j = 0; ok && j < ntA; ++j) {
        if (j + 1 < ntA) {
          const int s1 = (j + 1) % kKStages;
          if (!(ok = mbar_wait(&k_empty[s1], (((j + 1) / kKStages) & 1) ^ 1, p.err))) break;
          load_tile(&tmK, sK + s1 * kChunks * kChunkBytes, &k_full[s1], j + 1);
          k_issued = j + 2;
        }
        const int s = j % kVStages;
        if (!(ok = mbar_wait(&v_empty[s], ((j / kVStages) & 1) ^ 1, p.err))) break;
        load_tile(&tmV, sV + s * kChunks * kChunkBytes, &v_full[s], j);
        v_issued = j + 1;
      }
      mbar_wait(q_full, 0, p.err, kErrDrainTimeout);
      for (int j = max(0, k_issued - kKStages); j < k_issued; ++j)
        mbar_wait(&k_full[j % kKStages], (j / kKStages) & 1, p.err, kErrDrainTimeout);
      for (int j = max(0, v_issued - kVStages); j < v_issued; ++j)
        mbar_wait(&v_full[j % kVStages], (j / kVStages) & 1, p.err, kErrDrainTimeout);
    }
   } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      bool ok = mbar_wait(q_full, 0, p.err);
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      auto issue_s = [&](int x, int j) {   // S_X = Q_X K_j^T
        const int s = j % kKStages;
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = smem_desc(q_base + (x * kChunks + c) * kChunkBytes + kk * 32, 16, 1024, 2);
            const uint64_t bd = smem_desc(k_base + (s * kChunks + c) * kChunkBytes + kk * 32, 16, 1024, 2);
            tc_mma_ss(tmem + x * kBN, ad, bd, kIdescS, (c | kk) != 0);
          }
        tc_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int j) {   // O_X += P_X V_j, P_X from TMEM
        const int s = j % kVStages;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t bd = smem_desc(v_base + s * kChunks * kChunkBytes + kk * 2048, kChunkBytes, 1024, 2);
          tc_mma_ts(tmem + kColO + x * D, tmem + x * kBN + kk * 8, bd, kIdescO, (j | kk) != 0);
        }
        tc_commit(&o_done[x]);
      };
      if (ok && ntA > 0 && (ok = mbar_wait(&k_full[0], 0, p.err))) {
        tc_fence_after();
        issue_s(0, 0);
        if (ntB > 0) issue_s(1, 0);
        tc_commit(&k_empty[0]);
      }
      for (int j = 0; ok && j < ntA; ++j) {
        const int sv = j % kVStages;
        if (!(ok = mbar_wait(&v_full[sv], (j / kVStages) & 1, p.err))) break;
        const bool more = j + 1 < ntA;
        if (more && !(ok = mbar_wait(&k_full[(j + 1) % kKStages], ((j + 1) / kKStages) & 1, p.err))) break;
        // tile A
        if (!(ok = mbar_wait(&p_full[0], j & 1, p.err))) break;
        tc_fence_after();
        issue_pv(0, j);
        if (more) issue_s(0, j + 1);
        // tile B
        if (j < ntB) {
          if (!(ok = mbar_wait(&p_full[1], j & 1, p.err))) break;
          tc_fence_after();
          issue_pv(1, j);
          if (j + 1 < ntB) issue_s(1, j + 1);
        }
        tc_commit(&v_empty[sv]);
        if (more) tc_commit(&k_empty[(j + 1) % kKStages]);
      }
      // wait for every MMA this thread issued before TMEM can be released
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, p.err, kErrDrainTimeout);
    }
   }   // warps 10-11: nothing to do
  } else {
    // ------------------------------------------------------------------ softmax --
    regs_increase<kSoftmaxRegs>();
    const int x = warp >> 2;                   // 0: tile A, 1: tile B
    const int r = threadIdx.x & (kBM - 1);     // row / TMEM lane
    const int ntx = nt[x];
    const int hh = r / QP;
    const int i = qt[x] * QP + (r % QP);       // query index within the sequence
    const bool row_valid = i < Lq && (x == 0 || has_b);
    const int p_row = p.causal ? min(pos_off + i, Lk - 1) : Lk - 1;   // last visible key
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = x * kBN, colO = kColO + x * D;
    const float sl2 = p.scale_log2;
    float m_run = -INFINITY;                   // running max in raw score units
    float l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < ntx; ++j) {
      // S_X(j) complete implies PV_X(j-1) complete: P columns and O are free
      if (!(ok = mbar_wait_warp(&s_full[x], j & 1, p.err))) break;
      tc_fence_after();
      float xs[kBN];
      {
        uint32_t v[kBN / 32][32];
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c) tmem_ld32(lane_base + colS + c * 32, v[c]);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < kBN / 32; ++c)
#pragma unroll
          for (int e = 0; e < 32; ++e) xs[c * 32 + e] = __uint_as_float(v[c][e]);
      }
      const int col0 = j * kBN;
      if (col0 + kBN > full_keys[x]) {   // tile reaches past some row's last visible key
#pragma unroll
        for (int e = 0; e < kBN; ++e)
          if (col0 + e > p_row) xs[e] = -INFINITY;
      }
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = fmaxf(xs[u], xs[u + 8]);
#pragma unroll
      for (int e = 16; e < kBN; e += 16)
#pragma unroll
        for (int u = 0; u < 8; u += 2) {
          mx8[u] = max3(mx8[u], xs[e + u], xs[e + u + 8]);
          mx8[u + 1] = max3(mx8[u + 1], xs[e + u + 1], xs[e + u + 9]);
        }
      const float mt = fmaxf(fmaxf(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5])), fmaxf(mx8[6], mx8[7]));
      // lazy rescale: move the max only when it grew by more than 2^kRescaleLog2
      const bool grow = (mt - m_run) * sl2 > kRescaleLog2;
      const float m_new = grow ? mt : m_run;
      const float alpha = grow ? fast_exp2((m_run - m_new) * sl2) : 1.f;
      const float nms = -m_new * sl2;
      float rs[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      uint32_t pk[kBN / 2];
#pragma unroll
      for (int e = 0; e < kBN; e += 2) {
        float a0 = nms, a1 = nms;
        ffma2(a0, a1, xs[e], xs[e + 1], sl2, sl2);
        float p0, p1;
        if ((e / 2) % kEmuEvery >= kEmuFrom) {
          exp2_poly2(p0, p1, a0, a1);
        } else {
          p0 = fast_exp2(a0);
          p1 = fast_exp2(a1);
        }
        const int k = (e / 2) & 3;
        fadd2(rs[2 * k], rs[2 * k + 1], p0, p1);
        pk[e / 2] = pack_bf16x2(p0, p1);
      }
      l_run = l_run * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
      tmem_st32(lane_base + colS, *reinterpret_cast<const uint32_t(*)[32]>(&pk[0]));
      tmem_st32(lane_base + colS + 32, *reinterpret_cast<const uint32_t(*)[32]>(&pk[32]));
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        // rescale O rows whose max moved (alpha = 1 elsewhere)
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t v[32];
          tmem_ld32(lane_base + colO + c * 32, v);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
          tmem_st32(lane_base + colO + c * 32, v);
        }
      }
      tc_wait_st();
      m_run = m_new;
      if (x == 0 && col0 + kBN > Lk) {
        // the last tile reaches past the context: zero V rows >= Lk before any
        // PV reads them (group A's PV of this tile comes first; 0 * NaN would
        // poison the product)
        const int s = j % kVStages;
        if (!(ok = mbar_wait_warp(&v_full[s], (j / kVStages) & 1, p.err))) break;
        if (col0 + r >= Lk) {
#pragma unroll
          for (int c = 0; c < kChunks; ++c)
#pragma unroll
            for (int u = 0; u < 8; ++u)
              *reinterpret_cast<uint4*>(sV + (s * kChunks + c) * kChunkBytes + r * 128 + u * 16) =
                  make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
      }
      tc_fence_before();
      mbar_arrive(&p_full[x]);
    }
    if (ok && ntx > 0) ok = mbar_wait_warp(&o_done[x], (ntx - 1) & 1, p.err);
    // Group B stages its rows in the V ring, which tile A's remaining PVs may
    // still read when B has fewer key tiles: wait for every MMA of the CTA.
    if (ok && ntx > 0 && x == 1) ok = mbar_wait_warp(mma_done, 0, p.err);
    tc_fence_after();
    if (ok && ntx > 0) {   // warp-uniform: every lane takes part in the TMEM loads
      // O row -> bf16 -> shared memory, then one bulk copy per valid row to its
      // place in out.  Group A stages in the K ring (every QK has completed once
      // PV_A of the last tile has), group B in the V ring (after every MMA of
      // the CTA).  Rows are padded by 16 bytes so the 16-byte writes of a warp
      // hit distinct banks.
      const float inv = 1.f / l_run;
      uint8_t* srow = (x == 0 ? sK : sV) + r * (D * 2 + 16);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {   // 32 columns of O at a time
        uint32_t v[32];
        tmem_ld32(lane_base + colO + c * 32, v);
        tc_wait_ld();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          uint4 w;
          w.x = pack_bf16x2(__uint_as_float(v[8 * u + 0]) * inv, __uint_as_float(v[8 * u + 1]) * inv);
          w.y = pack_bf16x2(__uint_as_float(v[8 * u + 2]) * inv, __uint_as_float(v[8 * u + 3]) * inv);
          w.z = pack_bf16x2(__uint_as_float(v[8 * u + 4]) * inv, __uint_as_float(v[8 * u + 5]) * inv);
          w.w = pack_bf16x2(__uint_as_float(v[8 * u + 6]) * inv, __uint_as_float(v[8 * u + 7]) * inv);
          *reinterpret_cast<uint4*>(srow + (c * 4 + u) * 16) = w;
        }
      }
      fence_proxy_async_smem();
      if (row_valid) {
        __nv_bfloat16* orow = p.out + (static_cast<int64_t>(q_row0 + i) * p.num_heads + g * G + hh) * D;
        bulk_store_s2g(orow, srow, D * 2);
        bulk_commit();
        bulk_wait_read();
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
}

template <int D, int G>
pa_status launch_typed(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                       const PrefillParams& p, dim3 grid, cudaStream_t stream) {
  using Smem = PrefillSmem<D>;
  static int configured_device = -1;
  const DeviceInfo* di = current_device_info();
  if (configured_device != di->device) {
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D, G>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Smem::bytes));
    if (e != cudaSuccess) {
      set_last_error("cudaFuncSetAttribute(prefill): %s", cudaGetErrorString(e));
      return PA_ERR_CUDA;
    }
    configured_device = di->device;
  }
  prefill_kernel<D, G><<<grid, kThreads, Smem::bytes, stream>>>(tmQ, tmK, tmV, p);
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
  const int max_tiles = (a.max_seqlen_q + QP - 1) / QP;
  const dim3 grid(static_cast<unsigned>((max_tiles + 1) / 2), static_cast<unsigned>(a.num_kv_heads),
                  static_cast<unsigned>(a.num_seqs));
  return a.head_dim == 128 ? dispatch_group<128>(G, tmQ, tmK, tmV, p, grid, stream)
                           : dispatch_group<64>(G, tmQ, tmK, tmV, p, grid, stream);
}

}  // namespace pa
