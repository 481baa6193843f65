// Varlen causal prefill over a paged KV cache with prefix-cache blocks,
// on the sm_100a tensor cores (tcgen05.mma, accumulators in TMEM).
//
// ("Nano-vLLM 源碼學習" §二.2, prefill stage: varlen attention with prefix
// cache support; "Architektur im Überblick", "Prefill- und
// Decode-Vorbereitung": only uncached tokens are computed, their positions
// start at num_cached_tokens, so query i of a sequence with Lk keys and Lq
// new tokens sits at position Lk - Lq + i.)
//
// Persistent: one CTA per SM takes work items from a device counter until
// none are left; a work item is two query tiles (A and B) of one (kv head g,
// sequence b).  The M = 128 rows of a tile pack the G query heads that share
// kv head g, QP = 128 / G query positions each (row r -> head g*G + r / QP,
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
//   warp 8     TMA producer: takes the next item, decodes it and publishes
//              the decoded item to the other warps through a shared-memory
//              queue, loads its two Q tiles, then its K and V tiles in rings
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

#include <atomic>
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
// 256 x 208 + 128 x 88 = 64512.
constexpr uint32_t kSoftmaxRegs = 208;
constexpr uint32_t kControlRegs = 88;
static_assert(256 * kSoftmaxRegs + 128 * kControlRegs <= 384 * 168, "register split exceeds the launch budget");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kChunkBytes = kBM * 128;   // one 64-element-wide, 128-row swizzled chunk

// Dynamic work distribution: each launch uses one of kSchedSlots counter
// pairs {next item, CTAs finished}; CTAs take items with atomicAdd, and the
// last CTA to finish puts both counters back to zero for the next launch that
// uses the slot.  The host rotates slots between launches so that launches in
// flight at the same time (on different streams) do not share one, as long as
// fewer than kSchedSlots are in flight.  A captured CUDA graph keeps the slot
// it was captured with: a replay overlapping (on another stream) a launch that
// drew the same slot is outside the contract.
constexpr int kSchedSlots = 64;
__device__ unsigned int g_prefill_sched[kSchedSlots][2];

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
  int32_t sched_slot;
  int32_t out_v8;            // out is 32-byte aligned: write 32-byte vectors
  int32_t total_q;           // rows of q / out
  int32_t max_seqlen_q;
  int32_t max_seqlen_k;
  int32_t num_blocks;
};

template <int D>
struct PrefillSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kVStages = D == 128 ? 3 : 4;    // V ring depth
  static constexpr size_t q_off = 0;                    // Q_A then Q_B
  static constexpr size_t k_off = q_off + 2 * kChunks * kChunkBytes;
  static constexpr size_t v_off = k_off + kKStages * kChunks * kChunkBytes;
  static constexpr size_t bar_off = v_off + kVStages * kChunks * kChunkBytes;
  // barriers: q_full, q_empty[2], k_full[KS], k_empty[KS], v_full[VS], v_empty[VS], s_full[2], p_full[2],
  // o_done[2], mma_done, work_full[QN], work_empty[QN]
  static constexpr int kWorkQ = 4;                      // work-item queue depth
  static constexpr int kNumBars = 1 + 2 + 2 * kKStages + 2 * kVStages + 2 + 2 + 2 + 1 + 2 * kWorkQ;
  static constexpr size_t tmem_slot_off = bar_off + kNumBars * 8;
  static constexpr size_t queue_off = tmem_slot_off + 16;
  static constexpr size_t kItemBytes = 64;              // one decoded work item (struct Item)
  static constexpr size_t items_off = queue_off + kWorkQ * 4;
  static constexpr size_t bytes = items_off + kWorkQ * kItemBytes;
  static_assert(bytes <= 232448, "shared memory budget (227 KB per CTA)");
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
  float n0 = -kRoundMagic, n1 = -kRoundMagic;
  fadd2(n0, n1, t0, t1);                             // n = t - magic, exact
  float f0 = x0, f1 = x1;
  ffma2(f0, f1, n0, n1, -1.f, -1.f);                 // f = x - n
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
constexpr int kEmuFrom = 6;


// A row's running max only moves when the tile max exceeds it by more than
// 2^kRescaleLog2 (in exp2 units); until then the stale max keeps every
// probability <= 2^kRescaleLog2, exact after the final division, and the O
// accumulator in TMEM needs no correction.
constexpr float kRescaleLog2 = 8.0f;

// One work item: a pair of query tiles (A = the later one, B) of one
// (kv head, sequence).  Items are numbered pair-rank-major (rank 0 = the last
// pair of each sequence, which sees the most keys), so the costliest items
// are handed out first and items of similar cost run side by side.
struct Item {
  int b, g;
  int Lq, Lk, q_row0, pos_off;
  bool valid, has_b;
  bool bad;                               // the sequence's metadata breaks the call's contract: skipped
  int qtA, qtB, ntA, ntB, fullA, fullB;   // query tile, key tiles, keys every row sees
};

template <int QP>
__device__ __forceinline__ Item decode_item(int t, int num_seqs, int num_kv_heads, const PrefillParams& p) {
  Item it;
  const int per_rank = num_seqs * num_kv_heads;
  const int rank = t / per_rank;
  it.b = (t % per_rank) / num_kv_heads;
  it.g = t % num_kv_heads;
  const int64_t cq0 = __ldg(p.cu_seqlens_q);
  const int64_t cqb = __ldg(p.cu_seqlens_q + it.b);
  const int64_t lq = __ldg(p.cu_seqlens_q + it.b + 1) - cqb;
  const int64_t lk = __ldg(p.cu_seqlens_k + it.b + 1) - __ldg(p.cu_seqlens_k + it.b);
  const int64_t row0 = cqb - cq0;
  // Metadata that would make the item read or write outside the caller's
  // buffers (rows past total_q, keys past the block-table row) or miss rows
  // (more query tokens than max_seqlen_q provides items for) is reported and
  // the sequence is skipped.
  it.bad = lq < 0 || lk < lq || lq > p.max_seqlen_q || lk > p.max_seqlen_k ||
           lk > static_cast<int64_t>(p.max_blocks_per_seq) * p.block_size || row0 < 0 || row0 + lq > p.total_q;
  it.Lq = it.bad ? 0 : static_cast<int>(lq);
  it.Lk = it.bad ? 0 : static_cast<int>(lk);
  it.q_row0 = it.bad ? 0 : static_cast<int>(row0);
  it.pos_off = it.Lk - it.Lq;
  const int ntq = (it.Lq + QP - 1) / QP;
  const int npairs = (ntq + 1) / 2;
  const int pair = npairs - 1 - rank;
  it.valid = !it.bad && pair >= 0 && it.Lk >= it.Lq && it.Lk > 0;
  it.has_b = it.valid && 2 * pair + 1 < ntq;
  it.qtA = it.has_b ? 2 * pair + 1 : 2 * pair;
  it.qtB = 2 * pair;
  auto tiles = [&](int qt) {
    const int i_last = min(it.Lq, (qt + 1) * QP) - 1;
    const int n_keys = p.causal ? min(it.Lk, it.pos_off + i_last + 1) : it.Lk;
    return it.valid ? (n_keys + kBN - 1) / kBN : 0;
  };
  it.ntA = tiles(it.qtA);
  it.ntB = it.has_b ? tiles(it.qtB) : 0;
  it.fullA = p.causal ? min(it.Lk, it.pos_off + it.qtA * QP + 1) : it.Lk;
  it.fullB = p.causal ? min(it.Lk, it.pos_off + it.qtB * QP + 1) : it.Lk;
  return it;
}

template <int D, int G>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                   const __grid_constant__ CUtensorMap tmV, const PrefillParams p, int32_t num_seqs,
                   int32_t num_kv_heads, int32_t num_items) {
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
  uint64_t* q_empty = q_full + 1;            // [2]: Q_A, Q_B free again (their last QK has completed)
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + kKStages;
  uint64_t* v_full = k_empty + kKStages;
  uint64_t* v_empty = v_full + kVStages;
  uint64_t* s_full = v_empty + kVStages;     // [2]: tile A, tile B
  uint64_t* p_full = s_full + 2;             // [2]
  uint64_t* o_done = p_full + 2;             // [2]
  uint64_t* mma_done = o_done + 2;
  uint64_t* work_full = mma_done + 1;        // [kWorkQ]: queue entry written (producer)
  uint64_t* work_empty = work_full + Smem::kWorkQ;   // [kWorkQ]: entry read by the MMA thread and 8 softmax warps
  // queue entries: the item number (-1: no more work) and the item as the
  // producer decoded it, so that the other roles do not decode it again
  int32_t* work_queue = reinterpret_cast<int32_t*>(smem + Smem::queue_off);
  Item* work_items = reinterpret_cast<Item*>(smem + Smem::items_off);
  static_assert(sizeof(Item) <= Smem::kItemBytes && Smem::items_off % alignof(Item) == 0, "work item slot");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Smem::tmem_slot_off);
  constexpr int kWorkQ = Smem::kWorkQ;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(&q_empty[0], 1);
    mbar_init(&q_empty[1], 1);
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
    for (int q = 0; q < kWorkQ; ++q) {
      mbar_init(&work_full[q], 1);
      mbar_init(&work_empty[q], 1 + kSoftmaxWarps);
    }
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
      const int bs_shift = __ffs(p.block_size) - 1;
      int kc = 0, vc = 0;            // K / V tiles issued so far (ring positions)
      int qn[2] = {0, 0};            // Q tiles loaded so far per group
      bool ok = true;
      unsigned int* next_item = &g_prefill_sched[p.sched_slot][0];
      for (int n = 0; ok; ++n) {
        // take the next non-empty item and publish it to the MMA and softmax warps
        int t;
        Item it;
        do {
          t = static_cast<int>(atomicAdd(next_item, 1u));
          if (t >= num_items) break;
          it = decode_item<QP>(t, num_seqs, num_kv_heads, p);
          if (it.bad) record_error(p.err, kErrPrefillMeta);
        } while (!it.valid);
        const int q = n % kWorkQ;
        if (!(ok = mbar_wait(&work_empty[q], ((n / kWorkQ) & 1) ^ 1, p.err))) break;
        work_queue[q] = t < num_items ? t : -1;
        if (t < num_items) work_items[q] = it;
        mbar_arrive(&work_full[q]);   // release: the entry is visible to waiters of this phase
        if (t >= num_items) break;
        const int32_t* bt = p.block_tables + static_cast<int64_t>(it.b) * p.max_blocks_per_seq;
        const int nblk_valid = (it.Lk + p.block_size - 1) >> bs_shift;
        // One K or V tile: boxes past the last block of the sequence are skipped
        // (their table entries may be -1).
        auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* bar, int j) {
          int nbox = kBN / p.box_rows;
          while (nbox > 0 && ((j * kBN + (nbox - 1) * p.box_rows) >> bs_shift) >= nblk_valid) --nbox;
          mbar_arrive_expect_tx(bar, static_cast<uint32_t>(nbox * p.box_rows * 128 * kChunks));
          for (int k = 0; k < nbox; ++k) {
            const int tok = j * kBN + k * p.box_rows;
            const int blk = __ldg(bt + (tok >> bs_shift));
            // a table entry outside the cache is reported; TMA fills rows
            // outside the tensor map with zeros, so nothing outside is read
            if (static_cast<unsigned>(blk) >= static_cast<unsigned>(p.num_blocks)) record_error(p.err, kErrOutOfCache);
            const int row = (blk << bs_shift) + (tok & (p.block_size - 1));
            for (int c = 0; c < kChunks; ++c)
              tma_load_3d(dst + c * kChunkBytes + k * p.box_rows * 128, map, bar, c * 64, it.g, row);
          }
        };
        auto load_k = [&](int j) {
          const int s = kc % kKStages;
          if (!(ok = mbar_wait(&k_empty[s], ((kc / kKStages) & 1) ^ 1, p.err))) return;
          load_tile(&tmK, sK + s * kChunks * kChunkBytes, &k_full[s], j);
          ++kc;
        };
        auto load_v = [&](int j) {
          const int s = vc % kVStages;
          if (!(ok = mbar_wait(&v_empty[s], ((vc / kVStages) & 1) ^ 1, p.err))) return;
          load_tile(&tmV, sV + s * kChunks * kChunkBytes, &v_full[s], j);
          ++vc;
        };
        load_k(0);   // the first K tile goes ahead of Q: its slot may already be free
        if (!ok) break;
        const int nq = it.has_b ? 2 : 1;
        for (int x = 0; ok && x < nq; ++x)
          ok = mbar_wait(&q_empty[x], (qn[x] & 1) ^ 1, p.err);
        if (!ok) break;
        mbar_arrive_expect_tx(q_full, nq * kChunks * kChunkBytes);
        for (int x = 0; x < nq; ++x) {
          const int qt = x == 0 ? it.qtA : it.qtB;
          for (int hh = 0; hh < G; ++hh)
            for (int c = 0; c < kChunks; ++c)
              tma_load_3d(sQ + (x * kChunks + c) * kChunkBytes + hh * QP * 128, &tmQ, q_full, c * 64,
                          it.g * G + hh, it.q_row0 + qt * QP);
          ++qn[x];
        }
        for (int j = 0; ok && j < it.ntA; ++j) {   // K runs one tile ahead of V
          if (j + 1 < it.ntA) load_k(j + 1);
          if (ok) load_v(j);
        }
      }
      // never leave with copies in flight (time-limited; these have normally long landed)
      for (int n = max(0, kc - kKStages); n < kc; ++n)
        mbar_wait(&k_full[n % kKStages], (n / kKStages) & 1, p.err, kErrDrainTimeout);
      for (int n = max(0, vc - kVStages); n < vc; ++n)
        mbar_wait(&v_full[n % kVStages], (n / kVStages) & 1, p.err, kErrDrainTimeout);
      const int items_q = qn[0];
      if (items_q > 0) mbar_wait(q_full, (items_q - 1) & 1, p.err, kErrDrainTimeout);
    }
   } else if (warp == kMmaWarp) {
    // -------------------------------------------------------------- MMA issuer --
    if (lane == 0) {
      const uint32_t q_base = smem_u32(sQ), k_base = smem_u32(sK), v_base = smem_u32(sV);
      int kc = 0, vc = 0, nitems = 0;
      int sx[2] = {0, 0};      // p_full waits so far per group
      bool ok = true;
      // Descriptors differ only in their start-address field (bits 0-13, in
      // 16-byte units): build one base per operand and add offsets.
      const uint64_t q_desc = smem_desc(q_base, 16, 1024, 2);
      const uint64_t k_desc = smem_desc(k_base, 16, 1024, 2);
      const uint64_t v_desc = smem_desc(v_base, kChunkBytes, 1024, 2);
      auto issue_s = [&](int x, int ks) {   // S_X = Q_X K^T, K from ring slot ks
        const uint64_t qa = q_desc + ((x * kChunks * kChunkBytes) >> 4);
        const uint64_t kb = k_desc + ((ks * kChunks * kChunkBytes) >> 4);
#pragma unroll
        for (int c = 0; c < kChunks; ++c)
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t off = (c * kChunkBytes + kk * 32) >> 4;
            tc_mma_ss(tmem + x * kBN, qa + off, kb + off, kIdescS, (c | kk) != 0);
          }
        tc_commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int vs, bool first) {   // O_X (+)= P_X V, P_X from TMEM
        const uint64_t vb = v_desc + ((vs * kChunks * kChunkBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk)
          tc_mma_ts(tmem + kColO + x * D, tmem + x * kBN + kk * 8, vb + ((kk * 2048) >> 4), kIdescO,
                    !(first && kk == 0));
        tc_commit(&o_done[x]);
      };
      for (int n = 0; ok; ++n) {
        const int q = n % kWorkQ;
        if (!(ok = mbar_wait(&work_full[q], (n / kWorkQ) & 1, p.err))) break;
        const int t = work_queue[q];
        Item it;
        if (t >= 0) it = work_items[q];
        mbar_arrive(&work_empty[q]);
        if (t < 0) break;
        const int ntA = it.ntA, ntB = it.ntB;
        if (!(ok = mbar_wait(q_full, nitems & 1, p.err))) break;
        ++nitems;
        {
          const int ks = kc % kKStages;
          if (!(ok = mbar_wait(&k_full[ks], (kc / kKStages) & 1, p.err))) break;
          tc_fence_after();
          issue_s(0, ks);
          if (ntA == 1) tc_commit(&q_empty[0]);
          if (ntB > 0) {
            issue_s(1, ks);
            if (ntB == 1) tc_commit(&q_empty[1]);
          }
          tc_commit(&k_empty[ks]);
          ++kc;
        }
        for (int j = 0; ok && j < ntA; ++j) {
          const int vs = vc % kVStages;
          if (!(ok = mbar_wait(&v_full[vs], (vc / kVStages) & 1, p.err))) break;
          const bool more = j + 1 < ntA;
          const int ks = kc % kKStages;
          if (more && !(ok = mbar_wait(&k_full[ks], (kc / kKStages) & 1, p.err))) break;
          // tile A
          if (!(ok = mbar_wait(&p_full[0], sx[0] & 1, p.err))) break;
          ++sx[0];
          tc_fence_after();
          issue_pv(0, vs, j == 0);
          if (more) {
            issue_s(0, ks);
            if (j + 2 == ntA) tc_commit(&q_empty[0]);
          }
          // tile B
          if (j < ntB) {
            if (!(ok = mbar_wait(&p_full[1], sx[1] & 1, p.err))) break;
            ++sx[1];
            tc_fence_after();
            issue_pv(1, vs, j == 0);
            if (j + 1 < ntB) {
              issue_s(1, ks);
              if (j + 2 == ntB) tc_commit(&q_empty[1]);
            }
          }
          tc_commit(&v_empty[vs]);
          ++vc;
          if (more) {
            tc_commit(&k_empty[ks]);
            ++kc;
          }
        }
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
    const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
    const uint32_t colS = x * kBN, colO = kColO + x * D;
    const float sl2 = p.scale_log2;
    int ns = 0;                  // S tiles consumed so far (s_full phases)
    int no = 0;                  // PVs of this group issued so far (o_done phases)
    bool ok = true;
    for (int n = 0; ok; ++n) {
      const int q = n % kWorkQ;
      if (!(ok = mbar_wait_warp(&work_full[q], (n / kWorkQ) & 1, p.err))) break;
      const int t = work_queue[q];
      Item it;
      if (t >= 0) it = work_items[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(&work_empty[q]);
      if (t < 0) break;
      const int ntx = x == 0 ? it.ntA : it.ntB;
      if (ntx == 0) continue;
      const int full_keys = x == 0 ? it.fullA : it.fullB;
      const int hh = r / QP;
      const int i = (x == 0 ? it.qtA : it.qtB) * QP + (r % QP);  // query index within the sequence
      const bool row_valid = i < it.Lq;
      const int p_row = p.causal ? min(it.pos_off + i, it.Lk - 1) : it.Lk - 1;   // last visible key
      float m_run = -INFINITY;                 // running max in raw score units
      float l_run = 0.f;
      for (int j = 0; j < ntx; ++j) {
        // S_X(j) complete implies PV_X(j-1) complete: P columns and O are free
        if (!(ok = mbar_wait_warp(&s_full[x], ns & 1, p.err))) break;
        ++ns;
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
        if (col0 + kBN > full_keys) {   // tile reaches past some row's last visible key
          const int lim = p_row - col0;   // keys past it are masked in this row
#pragma unroll
          for (int e = 0; e < kBN; ++e) xs[e] = e > lim ? -INFINITY : xs[e];
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
        const float mt =
            fmaxf(fmaxf(max3(mx8[0], mx8[1], mx8[2]), max3(mx8[3], mx8[4], mx8[5])), fmaxf(mx8[6], mx8[7]));
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
        if (x == 0 && col0 + kBN > it.Lk) {
          // the last tile reaches past the context: zero V rows >= Lk before any
          // PV reads them (group A's PV of this tile comes first; 0 * NaN would
          // poison the product).  This tile's V slot is the one the MMA warp
          // consumes for tile j of this item.
          const int vs = (no + j) % kVStages;
          if (!(ok = mbar_wait_warp(&v_full[vs], ((no + j) / kVStages) & 1, p.err))) break;
          if (col0 + r >= it.Lk) {
#pragma unroll
            for (int c = 0; c < kChunks; ++c)
#pragma unroll
              for (int u = 0; u < 8; ++u)
                *reinterpret_cast<uint4*>(sV + (vs * kChunks + c) * kChunkBytes + r * 128 + u * 16) =
                    make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
        }
        tc_fence_before();
        mbar_arrive(&p_full[x]);
      }
      if (!ok) break;
      no += ntx;
      ok = mbar_wait_warp(&o_done[x], (no - 1) & 1, p.err);
      if (!ok) break;
      tc_fence_after();
      // Epilogue: O row -> bf16 -> out (16-byte stores of this thread's row).
      const float inv = 1.f / l_run;
      __nv_bfloat16* orow = p.out + (static_cast<int64_t>(it.q_row0 + i) * p.num_heads + it.g * G + hh) * D;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t v[32];
        tmem_ld32(lane_base + colO + c * 32, v);
        tc_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * inv, __uint_as_float(v[2 * e + 1]) * inv);
        if (row_valid) {
          if (p.out_v8) {   // full 32-byte sectors: half the store transactions of 16-byte vectors
            st_v8(orow + c * 32, *reinterpret_cast<const uint32_t(*)[8]>(&w[0]));
            st_v8(orow + c * 32 + 16, *reinterpret_cast<const uint32_t(*)[8]>(&w[8]));
          } else {
#pragma unroll
            for (int u = 0; u < 4; ++u)
              *reinterpret_cast<uint4*>(orow + c * 32 + u * 8) = make_uint4(w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
          }
        }
      }
      tc_fence_before();     // TMEM reads of O done before the next item's PV_X(0) may overwrite it
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kMmaWarp) tmem_dealloc(tmem, kTmemCols);
  if (threadIdx.x == 0) {
    // the last CTA of the launch returns the scheduling slot to zero
    __threadfence();
    if (atomicAdd(&g_prefill_sched[p.sched_slot][1], 1u) == gridDim.x - 1) {
      g_prefill_sched[p.sched_slot][0] = 0;
      g_prefill_sched[p.sched_slot][1] = 0;
      __threadfence();
    }
  }
}

template <int D, int G>
pa_status launch_typed(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                       const PrefillParams& p, dim3 grid, int32_t num_seqs, int32_t num_kv_heads, int32_t num_items,
                       cudaStream_t stream) {
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
  prefill_kernel<D, G><<<grid, kThreads, Smem::bytes, stream>>>(tmQ, tmK, tmV, p, num_seqs, num_kv_heads, num_items);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("prefill launch: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

template <int D>
pa_status dispatch_group(int G, const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                         const PrefillParams& p, dim3 grid, int32_t ns, int32_t nkv, int32_t ni, cudaStream_t stream) {
  switch (G) {
    case 1: return launch_typed<D, 1>(tmQ, tmK, tmV, p, grid, ns, nkv, ni, stream);
    case 2: return launch_typed<D, 2>(tmQ, tmK, tmV, p, grid, ns, nkv, ni, stream);
    case 4: return launch_typed<D, 4>(tmQ, tmK, tmV, p, grid, ns, nkv, ni, stream);
    case 8: return launch_typed<D, 8>(tmQ, tmK, tmV, p, grid, ns, nkv, ni, stream);
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
  p.out_v8 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
  p.total_q = a.total_q;
  p.max_seqlen_q = a.max_seqlen_q;
  p.max_seqlen_k = a.max_seqlen_k;
  p.num_blocks = a.num_blocks;
  static std::atomic<uint32_t> launches{0};
  p.sched_slot = static_cast<int32_t>(launches.fetch_add(1) % kSchedSlots);
  // persistent grid: at most one CTA per SM, each walking every gridDim.x-th work item
  const int max_tiles = (a.max_seqlen_q + QP - 1) / QP;
  const int64_t items64 = static_cast<int64_t>((max_tiles + 1) / 2) * a.num_kv_heads * a.num_seqs;
  if (items64 > INT32_MAX) {
    set_last_error("prefill: too many work items");
    return PA_ERR_UNSUPPORTED;
  }
  const int32_t items = static_cast<int32_t>(items64);
  const int sms = current_device_info()->sm_count;
  const dim3 grid(static_cast<unsigned>(items < sms ? items : sms));
  return a.head_dim == 128 ? dispatch_group<128>(G, tmQ, tmK, tmV, p, grid, a.num_seqs, a.num_kv_heads, items, stream)
                           : dispatch_group<64>(G, tmQ, tmK, tmV, p, grid, a.num_seqs, a.num_kv_heads, items, stream);
}

}  // namespace pa
