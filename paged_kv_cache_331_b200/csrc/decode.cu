// Paged GQA decode with split-KV, for sm_100a.
//
// ("Nano-vLLM 源碼學習" §二.2, decode stage; the lshu.cn essay on Nano-vLLM
// §3.2: attention gathers K/V of position j from page j / block_size, offset
// j % block_size of the sequence's page table.)
//
// The decode step reads every cached K/V row of every sequence once and does
// 4*G*D flops per row pair (G = query heads per kv head): about 2-4 flops per
// byte, so it is bound by HBM bandwidth, not by arithmetic.  Design:
//
//  * One CTA per (chunk of a sequence's keys, kv head, sequence).  The CTA
//    handles all G query heads that share the kv head, so each K/V byte
//    crosses HBM once.  Long sequences are cut into several chunks; their
//    partial results (running max m, sum l, unnormalised weighted V) go to a
//    workspace and a second kernel merges them (log-sum-exp rescaling).
//  * A producer warp streams 64-token K and V tiles of the kv head into
//    shared memory with TMA (a 3-D tensor map over [num_blocks*block_size,
//    kv_heads, head_dim] makes the physical block id just a row
//    coordinate), kStages deep, signalled through mbarriers.
//  * Four consumer warps each own 16 tokens of a tile.  QK: 8 lanes per
//    token, each lane holding D/8 query elements per head in registers,
//    three xor-shuffles per head finish the dot product.  Online softmax in
//    the exp2 domain (q pre-scaled by scale*log2 e) per warp.  PV: each lane
//    owns D/32 output dims of every head and walks the warp's tokens, reading
//    the probabilities as a shared-memory broadcast.  Warps merge their
//    (m, l, acc) at the end through shared memory.
#include <cuda_runtime.h>

#include <atomic>

#include <math.h>

#include "pa_device.cuh"
#include "pa_internal.h"

namespace pa {
namespace {

constexpr int kTile = kDecodeTile;         // tokens per stage
constexpr int kWarps = 4;                  // consumer warps
constexpr int kTPW = kTile / kWarps;       // tokens per consumer warp per tile
constexpr int kRounds = kTPW / 4;          // QK rounds (4 tokens per warp per round)
constexpr int kThreads = (kWarps + 1) * 32;

// Split-KV merge inside the split kernel: each launch uses one of
// kMergeSlots arrays of per-(sequence, kv head) counters; the CTA whose
// increment completes the count merges every chunk's partial and puts the
// counter back to zero for the next launch that uses the slot.  The host
// rotates slots between launches, so launches in flight at the same time on
// different streams do not share one as long as fewer than kMergeSlots are
// in flight.  A captured CUDA graph keeps the slot it was captured with: a
// replay overlapping (on another stream) a launch that drew the same slot is
// outside the contract.
constexpr int kMergeSlots = 16;
constexpr int kMergeCounters = 16384;   // sequences x kv heads per launch; above it a merge kernel runs
__device__ unsigned int g_decode_merge_cnt[kMergeSlots][kMergeCounters];

// Longest sequences first.  CTAs start roughly in the order of their index,
// and a launch whose last wave holds long sequences ends with most SMs idle.
// So, for launches of kOrderMinSeqs..kOrderMaxSeqs sequences and at most
// kOrderMaxCtas CTAs, split or not (the chunks of a long sequence are full,
// those of a short one few or partial), the CTAs of the first wave
// (blockIdx.z below order_first) take their sequences in index order and
// start at once, and CTA 0 sorts the other sequences by decreasing tile count
// and writes, for every later CTA, the sequence its blockIdx.z position
// stands for, with that sequence's context length:
// ((uint64)length << 32) | (sequence + 1).  Each CTA waits for its own entry
// (0 = not yet written), reads it once and puts 0 back, so the array is
// clean for the next launch that uses the slot; the host rotates
// kOrderSlots slots between launches, as for the merge counters.
constexpr int kOrderMinSeqs = 2;
constexpr int kOrderMaxSeqs = 512;
constexpr int kOrderMaxCtas = 8192;
constexpr int kOrderSlots = 16;
__device__ unsigned long long g_decode_order[kOrderSlots][kOrderMaxCtas];

struct DecodeParams {
  __nv_bfloat16* out;
  const __nv_bfloat16* q;
  const int32_t* block_tables;
  const int32_t* context_lens;
  float* ws_acc;
  float* ws_ml;
  float* o_part;            // partial mode: normalised fp32 output [B, Hq, D] instead of out
  float* lse_part;          //               log2-sum-exp of the scaled scores [B, Hq]
  int32_t max_blocks_per_seq;
  int32_t max_context_len;
  int32_t num_heads;
  int32_t block_size;
  int32_t box_rows;
  int32_t chunk_tokens;
  int32_t max_chunks;
  float scale_log2;
  unsigned int* err;
  int32_t num_kv_heads;
  int32_t merge_slot;       // >= 0: the last chunk CTA merges (counters of this slot); -1: merge kernel
  int32_t o_stride;         // head_dim (row stride of out / o_part)
  // fused store (slot_mapping != null): new K/V rows [num_seqs, Hkv, D] with row strides in elements
  const __nv_bfloat16* new_k;
  const __nv_bfloat16* new_v;
  int64_t new_k_stride;
  int64_t new_v_stride;
  const int32_t* slot_mapping;
  __nv_bfloat16* k_cache;
  __nv_bfloat16* v_cache;
  int64_t num_slots;        // num_blocks * block_size: a slot at or past it is outside the cache
  int32_t num_blocks;
  int32_t order_slot;       // >= 0: longest sequences first, through g_decode_order[order_slot]; -1: index order
  int32_t order_first;      // blockIdx.z positions below it (the first wave) take their sequence in index order
};

// CTAs per SM of a launch.  Unsplit launches at head_dim 128 with up to four
// query heads per kv head run three (two stages each): the extra consumer
// warps hide more of the arithmetic's latency.  Split launches keep two CTAs
// of three stages, which stream their long chunks faster.
constexpr int decode_ctas_per_sm(int head_dim, int G, int max_chunks) {
  return head_dim == 64 ? 2 : (G <= 4 ? (max_chunks == 1 ? 3 : 2) : 1);
}

// Per-shape configuration.  B CTAs share an SM (as many as shared memory and
// registers allow), so that each SM has 4*B consumer warps to hide latency;
// decode_ctas_per_sm picks B for a launch.
template <int D, int G, int B>
struct DecodeCfg {
  static constexpr int GP = G <= 1 ? 1 : (G <= 2 ? 2 : (G <= 4 ? 4 : 8));   // group padded to a power of two
  static constexpr int HB = GP == 1 ? 0 : (GP == 2 ? 1 : (GP == 4 ? 2 : 3)); // log2(GP)
  static_assert(D == 64 ? B == 2 : (G <= 4 ? (B == 2 || B == 3) : B == 1), "CTAs per SM for this shape");
  // three CTAs per SM fit only with two stages each
  static constexpr int kStages = (D == 64) ? 4 : (G <= 4 ? (B == 3 ? 2 : 3) : 4);
  static constexpr int kMinBlocks = B;
  static constexpr size_t kv_stage_elems = static_cast<size_t>(kTile) * D;
  static constexpr size_t k_off = 0;
  static constexpr size_t v_off = k_off + kStages * kv_stage_elems * 2;
  static constexpr size_t p_off = v_off + kStages * kv_stage_elems * 2;
  static constexpr size_t bar_off = p_off + static_cast<size_t>(kWarps) * kTPW * G * 2 * 4;
  static constexpr size_t bytes = bar_off + 2 * kStages * 8;
  // the cross-warp merge area reuses the K stages once every tile is consumed
  static constexpr size_t merge_bytes = static_cast<size_t>(kWarps) * G * (D + 2) * 4;
  static_assert(merge_bytes <= kStages * kv_stage_elems * 2, "merge area must fit in the K stages");
  static_assert(bar_off % 8 == 0, "alignment");
};

// One output element of a finished row: bf16 out, or in partial mode the
// normalised fp32 value (and, once per row, its log2-sum-exp).
__device__ __forceinline__ void write_row(const DecodeParams& p, int64_t row, int d, float o, float M, float lsum) {
  if (p.o_part) {
    p.o_part[row * (p.o_stride) + d] = o / lsum;
    if (d == 0) p.lse_part[row] = M + log2f(lsum);
  } else {
    p.out[row * p.o_stride + d] = __float2bfloat16(o / lsum);
  }
}

__device__ __forceinline__ int clamp_context(int L, const DecodeParams& p) {
  L = min(L, p.max_context_len);
  L = min(L, p.max_blocks_per_seq * p.block_size);
  return max(L, 0);
}

// Butterfly reduce-scatter over the 8 lanes of a token group: on entry every
// lane holds CNT partial dot products (one per head); on exit v[0] holds the
// full sum for one head, selected by the lane's bits (lane & 4, 2, 1 pick the
// upper half at each halving step), with CNT-1 fewer shuffles than reducing
// every head separately.
template <int CNT, int MASK>
__device__ __forceinline__ void reduce_scatter(float* v, int lane) {
  if constexpr (MASK == 0) {
    return;
  } else if constexpr (CNT > 1) {
    constexpr int H = CNT / 2;
    const bool up = (lane & MASK) != 0;
#pragma unroll
    for (int i = 0; i < H; ++i) {
      const float send = up ? v[i] : v[H + i];
      const float keep = up ? v[H + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
    }
    reduce_scatter<H, MASK / 2>(v, lane);
  } else {
    v[0] += __shfl_xor_sync(0xffffffffu, v[0], MASK);
    reduce_scatter<1, MASK / 2>(v, lane);
  }
}

// Head held by lane-in-group li after reduce_scatter<GP, 4>, and the lane that
// is the canonical holder of head h (its non-head bits zero).
template <int GP, int HB>
__device__ __forceinline__ int head_of_lane(int li) {
  int h = 0;
#pragma unroll
  for (int k = 0; k < HB; ++k)
    if (li & (4 >> k)) h += GP >> (k + 1);
  return h;
}
template <int HB>
__device__ __forceinline__ int lane_of_head(int h) {
  int li = 0;
#pragma unroll
  for (int k = 0; k < HB; ++k)
    if ((h >> (HB - 1 - k)) & 1) li |= 4 >> k;
  return li;
}

// The work of one CTA: chunk blockIdx.x of kv head blockIdx.y of sequence b,
// whose context_lens entry is L_raw.
template <int D, int G, int B>
__device__ __forceinline__ void decode_cta(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p,
                                           const int b, const int L_raw) {
  using Cfg = DecodeCfg<D, G, B>;
  constexpr int kStages = Cfg::kStages;
  constexpr int GP = Cfg::GP, HB = Cfg::HB;
  constexpr int DPL = D / 8;    // query/key dims per lane in QK (8 lanes per token)
  constexpr int DPV = D / 32;   // output dims per lane in PV
  static_assert(D == 64 || D == 128, "head_dim");

  extern __shared__ __align__(128) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem + Cfg::k_off);
  __nv_bfloat16* sV = reinterpret_cast<__nv_bfloat16*>(smem + Cfg::v_off);
  float* pbuf = reinterpret_cast<float*>(smem + Cfg::p_off);
  float* mrg = reinterpret_cast<float*>(smem + Cfg::k_off);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + Cfg::bar_off);
  uint64_t* empty = full + kStages;

  const int chunk = blockIdx.x, g = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = clamp_context(L_raw, p);
  if (L != L_raw && chunk == 0 && g == 0 && threadIdx.x == 0) record_error(p.err, kErrContextLen);
  const int hq0 = g * G;

  if (L == 0) {   // no keys: the output is defined as zero (a partial: 0 with lse = -inf)
    if (chunk == 0) {
      const int64_t base = (static_cast<int64_t>(b) * p.num_heads + hq0) * D;
      for (int i = threadIdx.x; i < G * D; i += kThreads) {
        if (p.o_part) p.o_part[base + i] = 0.f;
        else p.out[base + i] = __float2bfloat16(0.f);
      }
      if (p.lse_part && threadIdx.x < G) p.lse_part[static_cast<int64_t>(b) * p.num_heads + hq0 + threadIdx.x] = -INFINITY;
    }
    return;
  }
  const int start = chunk * p.chunk_tokens;
  if (start >= L) return;
  const int end = min(L, start + p.chunk_tokens);
  const int nchunks = (L + p.chunk_tokens - 1) / p.chunk_tokens;
  const int ntiles = (end - start + kTile - 1) / kTile;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kWarps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  if (warp == kWarps) {
    // ------------------------------------------------------------ producer --
    if (lane == 0) {
      prefetch_tensormap(&tmK);
      prefetch_tensormap(&tmV);
      const int32_t* bt = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq;
      const uint64_t pol = policy_evict_first();
      const int bs_shift = __ffs(p.block_size) - 1;
      int issued = 0;
      for (int it = 0; it < ntiles; ++it) {
        const int s = it % kStages;
        if (!mbar_wait(&empty[s], ((it / kStages) & 1) ^ 1, p.err)) break;
        const int t0 = start + it * kTile;
        const int valid = min(kTile, end - t0);
        const int nbox = (valid + p.box_rows - 1) / p.box_rows;
        mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nbox * p.box_rows * D * 2 * 2));
        for (int k = 0; k < nbox; ++k) {
          const int tok = t0 + k * p.box_rows;
          const int blk = __ldg(bt + (tok >> bs_shift));
          // a table entry outside the cache is reported; TMA fills the box's
          // rows outside the tensor map with zeros, so nothing outside the
          // cache is read
          if (static_cast<unsigned>(blk) >= static_cast<unsigned>(p.num_blocks)) record_error(p.err, kErrOutOfCache);
          const int row = (blk << bs_shift) + (tok & (p.block_size - 1));
          const size_t soff = (static_cast<size_t>(s) * kTile + static_cast<size_t>(k) * p.box_rows) * D;
          tma_load_3d_hint(sK + soff, &tmK, &full[s], 0, g, row, pol);
          tma_load_3d_hint(sV + soff, &tmV, &full[s], 0, g, row, pol);
        }
        ++issued;
      }
      // Never leave with copies in flight: wait (time-limited) for the last
      // loads of every stage.  On the normal path these have long landed.
      for (int it = max(0, issued - kStages); it < issued; ++it)
        mbar_wait(&full[it % kStages], (it / kStages) & 1, p.err, kErrDrainTimeout);
    }
    return;
  }

  // -------------------------------------------------------------- consumers --
  // Fused store: this CTA is the only reader of position L-1 (in its last
  // tile).  The consumer warp whose tokens include it loads the new token's
  // K/V row of kv head g into registers, writes it to the cache slot (nothing
  // in this launch reads that slot from global memory, so the store needs no
  // ordering), and once the last tile has landed overwrites that row of the
  // staged tile in shared memory, which its TMA load may have read before
  // the store.  The slot must be that position's (any other slot but -1 is
  // reported and not written) and lie inside the cache (a table entry past
  // the cache is reported, not followed).
  constexpr int kRowPieces = D / 8;   // 16-byte pieces of one head row
  int patch_row = -1;                 // row of position L-1 in the last tile, if this warp owns it
  uint4 new_piece = make_uint4(0, 0, 0, 0);   // lanes < kRowPieces: K piece lane; next kRowPieces: V pieces
  if (p.slot_mapping && chunk == nchunks - 1) {
    const int32_t slot = __ldg(p.slot_mapping + b);
    const int32_t* btb = p.block_tables + static_cast<int64_t>(b) * p.max_blocks_per_seq;
    const int pos = L - 1;
    const int64_t expect = static_cast<int64_t>(__ldg(btb + pos / p.block_size)) * p.block_size + pos % p.block_size;
    if (slot == expect && slot >= 0 && slot < p.num_slots) {
      const int idx = pos - (start + (ntiles - 1) * kTile);   // position within the last tile
      if (idx / kTPW == warp) {
        patch_row = idx;
        if (lane < 2 * kRowPieces) {
          const bool is_v = lane >= kRowPieces;
          const int piece = is_v ? lane - kRowPieces : lane;
          new_piece = ld_nc_v4((is_v ? p.new_v + b * p.new_v_stride : p.new_k + b * p.new_k_stride) +
                               static_cast<int64_t>(g) * D + piece * 8);
          *reinterpret_cast<uint4*>((is_v ? p.v_cache : p.k_cache) +
                                    (static_cast<int64_t>(slot) * p.num_kv_heads + g) * D + piece * 8) = new_piece;
        }
      }
    } else if (slot != -1 && warp == 0 && lane == 0) {
      record_error(p.err, slot == expect ? kErrOutOfCache : kErrBadSlot);
    }
  }
  const int li = lane & 7, gi = lane >> 3;
  const int hsel = head_of_lane<GP, HB>(li);            // head whose score this lane ends up with
  constexpr int kHeadBits = (7 << (3 - HB)) & 7;
  const bool owner = (li & ~kHeadBits & 7) == 0 && hsel < G;   // one lane per (token, head) writes p

  // q in registers as (even, odd) dim pairs, pre-scaled by scale * log2(e)
  float qf[G][DPL];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    const __nv_bfloat16* qp = p.q + (static_cast<int64_t>(b) * p.num_heads + hq0 + h) * D;
#pragma unroll
    for (int part = 0; part < DPL / 8; ++part) {
      const uint4 v = *reinterpret_cast<const uint4*>(qp + part * 64 + li * 8);
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        qf[h][part * 8 + 2 * e] = bf16lo(w[e]) * p.scale_log2;
        qf[h][part * 8 + 2 * e + 1] = bf16hi(w[e]) * p.scale_log2;
      }
    }
  }
  float m[G], acc[G][DPV];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
#pragma unroll
    for (int c = 0; c < DPV; ++c) acc[h][c] = 0.f;
  }
  float m_own = -INFINITY, l_own = 0.f;   // running max / sum of this lane's head (lane-group partial)
  float* pw = pbuf + warp * kTPW * G * 2;
  const int wbase = warp * kTPW;

  for (int it = 0; it < ntiles; ++it) {
    const int s = it % kStages;
    if (!mbar_wait(&full[s], (it / kStages) & 1, p.err)) break;
    if (it == ntiles - 1 && patch_row >= 0) {   // the new row replaces what TMA staged for position L-1
      if (lane < 2 * kRowPieces) {
        const bool is_v = lane >= kRowPieces;
        const int piece = is_v ? lane - kRowPieces : lane;
        *reinterpret_cast<uint4*>((is_v ? sV : sK) + (static_cast<size_t>(s) * kTile + patch_row) * D + piece * 8) =
            new_piece;
      }
      __syncwarp();
    }
    const int valid = min(kTile, end - (start + it * kTile));
    const int nw = min(kTPW, valid - wbase);
    if (nw > 0) {
      const __nv_bfloat16* Ks = sK + static_cast<size_t>(s) * kTile * D;
      float sc[kRounds];
#pragma unroll
      for (int r = 0; r < kRounds; ++r) {
        const __nv_bfloat16* kr = Ks + (wbase + r * 4 + gi) * D;
        uint32_t kw[DPL / 2];
#pragma unroll
        for (int part = 0; part < DPL / 8; ++part) {
          const uint4 v = *reinterpret_cast<const uint4*>(kr + part * 64 + li * 8);
          kw[part * 4 + 0] = v.x; kw[part * 4 + 1] = v.y; kw[part * 4 + 2] = v.z; kw[part * 4 + 3] = v.w;
        }
        float kf[DPL];
#pragma unroll
        for (int e = 0; e < DPL / 2; ++e) {
          kf[2 * e] = bf16lo(kw[e]);
          kf[2 * e + 1] = bf16hi(kw[e]);
        }
        float v[GP];
#pragma unroll
        for (int h = 0; h < GP; ++h) {
          if (h < G) {
            float e0 = 0.f, e1 = 0.f;
#pragma unroll
            for (int e = 0; e < DPL / 2; ++e) ffma2(e0, e1, qf[h][2 * e], qf[h][2 * e + 1], kf[2 * e], kf[2 * e + 1]);
            v[h] = e0 + e1;
          } else {
            v[h] = 0.f;
          }
        }
        reduce_scatter<GP, 4>(v, lane);
        sc[r] = (r * 4 + gi < nw && hsel < G) ? v[0] : -INFINITY;
      }
      // tile max of every head, visible in every lane
      float mx = sc[0];
#pragma unroll
      for (int r = 1; r < kRounds; ++r) mx = fmaxf(mx, sc[r]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mh = __shfl_sync(0xffffffffu, mx, lane_of_head<HB>(h));
        const float mnew = fmaxf(m[h], mh);
        const float alpha = fast_exp2(m[h] - mnew);
        m[h] = mnew;
#pragma unroll
        for (int c = 0; c < DPV; c += 2) fmul2(acc[h][c], acc[h][c + 1], alpha, alpha);
      }
      const float m_own_new = fmaxf(m_own, mx);
      const float a_own = fast_exp2(m_own - m_own_new);
      m_own = m_own_new;
      float psum = 0.f;
#pragma unroll
      for (int r = 0; r < kRounds; ++r) {
        const float pr = fast_exp2(sc[r] - m_own_new);
        psum += pr;
        if (owner) *reinterpret_cast<float2*>(pw + ((r * 4 + gi) * G + hsel) * 2) = make_float2(pr, pr);
      }
      l_own = l_own * a_own + psum;
      __syncwarp();
      const __nv_bfloat16* Vs = sV + (static_cast<size_t>(s) * kTile + wbase) * D + lane * DPV;
#pragma unroll 4
      for (int t = 0; t < nw; ++t) {
        float pv[2 * G];
        if constexpr (G % 2 == 0) {
#pragma unroll
          for (int h = 0; h < G; h += 2) {
            const float4 x = *reinterpret_cast<const float4*>(pw + (t * G + h) * 2);
            pv[2 * h] = x.x; pv[2 * h + 1] = x.y; pv[2 * h + 2] = x.z; pv[2 * h + 3] = x.w;
          }
        } else {
#pragma unroll
          for (int h = 0; h < G; ++h) {
            const float2 x = *reinterpret_cast<const float2*>(pw + (t * G + h) * 2);
            pv[2 * h] = x.x; pv[2 * h + 1] = x.y;
          }
        }
        float vf[DPV];
        if constexpr (DPV == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(Vs + t * D);
          vf[0] = bf16lo(v.x); vf[1] = bf16hi(v.x); vf[2] = bf16lo(v.y); vf[3] = bf16hi(v.y);
        } else {
          const uint32_t v = *reinterpret_cast<const uint32_t*>(Vs + t * D);
          vf[0] = bf16lo(v); vf[1] = bf16hi(v);
        }
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
          for (int c = 0; c < DPV; c += 2) ffma2(acc[h][c], acc[h][c + 1], pv[2 * h], pv[2 * h + 1], vf[c], vf[c + 1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  }

  // ---------------------------------------------------- merge the four warps --
  // every tile has been consumed, so the K stages are free for the merge area
  l_own += __shfl_xor_sync(0xffffffffu, l_own, 8);
  l_own += __shfl_xor_sync(0xffffffffu, l_own, 16);
  float lh[G];
#pragma unroll
  for (int h = 0; h < G; ++h) lh[h] = __shfl_sync(0xffffffffu, l_own, lane_of_head<HB>(h));
  named_barrier_sync(1, kWarps * 32);   // all warps are past their last read of the K stages
  float* mw = mrg + warp * G * (D + 2);
#pragma unroll
  for (int h = 0; h < G; ++h)
#pragma unroll
    for (int c = 0; c < DPV; ++c) mw[h * D + lane * DPV + c] = acc[h][c];
  if (lane == 0) {
#pragma unroll
    for (int h = 0; h < G; ++h) {
      mw[G * D + 2 * h] = m[h];
      mw[G * D + 2 * h + 1] = lh[h];
    }
  }
  named_barrier_sync(1, kWarps * 32);
  for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
    const int h = i / D, d = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mrg[w * G * (D + 2) + G * D + 2 * h]);
    float lsum = 0.f, o = 0.f;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
      const float* mwv = mrg + w * G * (D + 2);
      const float f = fast_exp2(mwv[G * D + 2 * h] - M);
      lsum += mwv[G * D + 2 * h + 1] * f;
      o += mwv[h * D + d] * f;
    }
    const int64_t row = static_cast<int64_t>(b) * p.num_heads + hq0 + h;
    if (nchunks == 1) {
      write_row(p, row, d, o, M, lsum);
    } else {
      const int64_t idx = row * p.max_chunks + chunk;
      p.ws_acc[idx * D + d] = o;
      if (d == 0) {
        p.ws_ml[2 * idx] = M;
        p.ws_ml[2 * idx + 1] = lsum;
      }
    }
  }
  if (nchunks == 1 || p.merge_slot < 0) return;

  // ------------------------------------- the last chunk of (b, g) merges all --
  // The barrier orders every consumer's partial writes before thread 0's
  // device-scope fence (fences are cumulative), which publishes them before
  // its increment; the last CTA's fence after its increment orders the
  // partials of the other chunks before the reads that follow the barrier.
  __shared__ int s_last;
  named_barrier_sync(1, kWarps * 32);
  if (threadIdx.x == 0) {
    __threadfence();
    unsigned int* cnt = &g_decode_merge_cnt[p.merge_slot][b * p.num_kv_heads + g];
    const unsigned int prev = atomicAdd(cnt, 1u);
    s_last = prev == static_cast<unsigned int>(nchunks - 1);
    if (s_last) {
      *cnt = 0u;                         // every chunk has counted: ready for the next launch
      __threadfence();
    }
  }
  named_barrier_sync(1, kWarps * 32);
  if (!s_last) return;
  for (int i = threadIdx.x; i < G * D; i += kWarps * 32) {
    const int h = i / D, d = i % D;
    const int64_t row = static_cast<int64_t>(b) * p.num_heads + hq0 + h;
    const float* ml = p.ws_ml + row * p.max_chunks * 2;
    const float* ac = p.ws_acc + row * p.max_chunks * D + d;
    float M = -INFINITY;
    for (int c = 0; c < nchunks; ++c) M = fmaxf(M, __ldcg(ml + 2 * c));
    float lsum = 0.f, o = 0.f;
    for (int c = 0; c < nchunks; ++c) {
      const float f = fast_exp2(__ldcg(ml + 2 * c) - M);
      lsum += __ldcg(ml + 2 * c + 1) * f;
      o += __ldcg(ac + static_cast<int64_t>(c) * D) * f;
    }
    write_row(p, row, d, o, M, lsum);
  }
}

// The sequence this CTA works on, as a packed order entry (see g_decode_order).
template <int D, int G, int B>
__device__ __forceinline__ unsigned long long decode_order_entry(const DecodeParams& p) {
  using Cfg = DecodeCfg<D, G, B>;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ unsigned long long s_entry;
  unsigned long long* entries = g_decode_order[p.order_slot];
  const int nseq = static_cast<int>(gridDim.z);
  const int lin = static_cast<int>((blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x);
  if (lin == 0) {
    // A counting sort by tile count, descending, in shared memory that the
    // TMA ring does not use yet.  (The order within a tile count is whatever
    // the shared-memory atomics give: only this CTA computes it.)
    constexpr int kPerThread = (kOrderMaxSeqs + kThreads - 1) / kThreads;
    constexpr int kBins = 1024;
    int* hist = reinterpret_cast<int*>(smem + Cfg::k_off);
    int* seq_at = hist + kBins;
    int* raw_at = seq_at + kOrderMaxSeqs;
    const int first = p.order_first;   // sequences [first, nseq) are sorted into positions [first, nseq)
    int shift = 0;   // tile counts past kBins share bins
    while ((((p.max_context_len + kTile - 1) / kTile) >> shift) >= kBins) ++shift;
    for (int i = threadIdx.x; i < kBins; i += kThreads) hist[i] = 0;
    __syncthreads();
    int bin[kPerThread], raw[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      const int i = first + threadIdx.x + u * kThreads;
      bin[u] = -1;
      if (i < nseq) {
        raw[u] = __ldg(p.context_lens + i);
        const int tiles = (clamp_context(raw[u], p) + kTile - 1) / kTile;
        bin[u] = kBins - 1 - min(tiles >> shift, kBins - 1);   // longest first
        atomicAdd(&hist[bin[u]], 1);
      }
    }
    __syncthreads();
    if (threadIdx.x < 32) {   // exclusive prefix sum of the bins, 32 consecutive bins per lane
      constexpr int kPerLane = kBins / 32;
      int run = 0;
      for (int k = 0; k < kPerLane; ++k) run += hist[threadIdx.x * kPerLane + k];
      int incl = run;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (static_cast<int>(threadIdx.x) >= o) incl += v;
      }
      int off = incl - run;
      for (int k = 0; k < kPerLane; ++k) {
        const int c = hist[threadIdx.x * kPerLane + k];
        hist[threadIdx.x * kPerLane + k] = off;
        off += c;
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
      if (bin[u] >= 0) {
        const int pos = atomicAdd(&hist[bin[u]], 1);
        seq_at[pos] = first + threadIdx.x + u * kThreads;
        raw_at[pos] = raw[u];
      }
    }
    __syncthreads();
    const int per_seq = static_cast<int>(gridDim.x * gridDim.y);
    for (int e = first * per_seq + threadIdx.x; e < nseq * per_seq; e += kThreads) {
      const int z = e / per_seq - first;
      entries[e] = (static_cast<unsigned long long>(static_cast<unsigned int>(raw_at[z])) << 32) |
                   static_cast<unsigned int>(seq_at[z] + 1);
    }
    __syncthreads();   // the sort's shared memory is free again
    return (static_cast<unsigned long long>(static_cast<unsigned int>(__ldg(p.context_lens))) << 32) | 1u;
  }
  if (threadIdx.x == 0) {
    volatile unsigned long long* mine = entries + lin;
    unsigned long long e = *mine;
    if (e == 0ull) {   // CTA 0 (resident: the first to be dispatched) has not written it yet
      const uint64_t t0 = global_timer_ns();
      while ((e = *mine) == 0ull) {
        if (global_timer_ns() - t0 > PA_WAIT_LIMIT_NS) {   // never on a working device: fall back to index order
          record_error(p.err, kErrWaitTimeout);
          e = (static_cast<unsigned long long>(static_cast<unsigned int>(__ldg(p.context_lens + blockIdx.z))) << 32) |
              (blockIdx.z + 1u);
          break;
        }
      }
    }
    *mine = 0ull;      // read once: clean for the next launch that uses the slot
    s_entry = e;
  }
  __syncthreads();
  return s_entry;
}

template <int D, int G, int B>
__global__ void __launch_bounds__(kThreads, DecodeCfg<D, G, B>::kMinBlocks)
    decode_split_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                        const DecodeParams p) {
  if (p.order_slot >= 0 && (blockIdx.z >= static_cast<unsigned>(p.order_first) ||
                            (blockIdx.x | blockIdx.y | blockIdx.z) == 0)) {
    const unsigned long long e = decode_order_entry<D, G, B>(p);
    const unsigned int seq = static_cast<unsigned int>(e) - 1u;
    if (seq < gridDim.z) {
      decode_cta<D, G, B>(tmK, tmV, p, static_cast<int>(seq), static_cast<int>(static_cast<unsigned int>(e >> 32)));
    } else {   // an entry no launch of this shape wrote (a launch on this slot was cut short): index order
      if (threadIdx.x == 0) record_error(p.err, kErrWaitTimeout);
      decode_cta<D, G, B>(tmK, tmV, p, static_cast<int>(blockIdx.z), __ldg(p.context_lens + blockIdx.z));
    }
  } else {
    decode_cta<D, G, B>(tmK, tmV, p, static_cast<int>(blockIdx.z), __ldg(p.context_lens + blockIdx.z));
  }
}

// Merge of split-KV partials: one warp per (sequence, query head).
//   M = max_c m_c,  out = sum_c 2^(m_c - M) acc_c / sum_c 2^(m_c - M) l_c
template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeParams p, int32_t num_rows) {
  constexpr int DPV = D / 32;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= num_rows) return;
  const int b = row / p.num_heads;
  const int L = clamp_context(__ldg(p.context_lens + b), p);
  const int n = (L + p.chunk_tokens - 1) / p.chunk_tokens;
  if (n <= 1) return;   // written directly by the split kernel (or zero)
  const float* ml = p.ws_ml + static_cast<int64_t>(row) * p.max_chunks * 2;
  const float* acc = p.ws_acc + static_cast<int64_t>(row) * p.max_chunks * D;
  float M = -INFINITY;
  for (int c = lane; c < n; c += 32) M = fmaxf(M, ml[2 * c]);
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float lsum = 0.f, o[DPV];
#pragma unroll
  for (int c = 0; c < DPV; ++c) o[c] = 0.f;
  for (int c = 0; c < n; ++c) {
    const float f = fast_exp2(ml[2 * c] - M);
    lsum += ml[2 * c + 1] * f;
    if constexpr (DPV == 4) {
      const float4 a = *reinterpret_cast<const float4*>(acc + static_cast<int64_t>(c) * D + lane * 4);
      o[0] += a.x * f; o[1] += a.y * f; o[2] += a.z * f; o[3] += a.w * f;
    } else {
      const float2 a = *reinterpret_cast<const float2*>(acc + static_cast<int64_t>(c) * D + lane * 2);
      o[0] += a.x * f; o[1] += a.y * f;
    }
  }
  const float inv = 1.f / lsum;
  if (p.o_part) {   // partial mode: keep the normalised output in fp32, with its log2-sum-exp
    float* op = p.o_part + static_cast<int64_t>(row) * D + lane * DPV;
#pragma unroll
    for (int c = 0; c < DPV; ++c) op[c] = o[c] * inv;
    if (lane == 0) p.lse_part[row] = M + log2f(lsum);
    return;
  }
  __nv_bfloat16* out = p.out + static_cast<int64_t>(row) * D + lane * DPV;
#pragma unroll
  for (int c = 0; c < DPV; c += 2)
    *reinterpret_cast<uint32_t*>(out + c) = pack_bf16x2(o[c] * inv, o[c + 1] * inv);
}

// Combination of R partials per (sequence, head) row (one warp per row):
//   M = max_r lse_r,  out = sum_r 2^(lse_r - M) o_r / sum_r 2^(lse_r - M)
// (a row whose partials all hold no keys, lse = -inf everywhere, is 0).
template <int D>
__global__ void __launch_bounds__(128) merge_lse_kernel(__nv_bfloat16* __restrict__ out,
                                                        const float* __restrict__ o_parts,
                                                        const float* __restrict__ lse_parts, int32_t num_parts,
                                                        int32_t num_rows) {
  constexpr int DPV = D / 32;
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= num_rows) return;
  float M = -INFINITY;
  for (int r = lane; r < num_parts; r += 32) M = fmaxf(M, __ldg(lse_parts + static_cast<int64_t>(r) * num_rows + row));
#pragma unroll
  for (int o = 16; o; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  float o[DPV];
#pragma unroll
  for (int c = 0; c < DPV; ++c) o[c] = 0.f;
  float wsum = 0.f;
  if (M != -INFINITY) {
    for (int r = 0; r < num_parts; ++r) {
      const float l = __ldg(lse_parts + static_cast<int64_t>(r) * num_rows + row);
      if (l == -INFINITY) continue;
      const float w = fast_exp2(l - M);
      wsum += w;
      const float* src = o_parts + (static_cast<int64_t>(r) * num_rows + row) * D + lane * DPV;
#pragma unroll
      for (int c = 0; c < DPV; ++c) o[c] += w * __ldg(src + c);
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = out + static_cast<int64_t>(row) * D + lane * DPV;
#pragma unroll
  for (int c = 0; c < DPV; c += 2)
    *reinterpret_cast<uint32_t*>(dst + c) = pack_bf16x2(o[c] * inv, o[c + 1] * inv);
}

template <int D, int G, int B>
pa_status launch_cfg(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, dim3 grid,
                       cudaStream_t stream) {
  using Cfg = DecodeCfg<D, G, B>;
  static int configured_device = -1;
  const DeviceInfo* di = current_device_info();
  if (configured_device != di->device) {
    cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<D, G, B>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(Cfg::bytes));
    if (e != cudaSuccess) {
      set_last_error("cudaFuncSetAttribute(decode): %s", cudaGetErrorString(e));
      return PA_ERR_CUDA;
    }
    configured_device = di->device;
  }
  decode_split_kernel<D, G, B><<<grid, kThreads, Cfg::bytes, stream>>>(tmK, tmV, p);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("decode launch: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

// The configuration decode_ctas_per_sm names for this launch.
template <int D, int G>
pa_status launch_split(const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, dim3 grid,
                       cudaStream_t stream) {
  if constexpr (D == 128 && G <= 4) {
    return decode_ctas_per_sm(D, G, p.max_chunks) == 3 ? launch_cfg<D, G, 3>(tmK, tmV, p, grid, stream)
                                                       : launch_cfg<D, G, 2>(tmK, tmV, p, grid, stream);
  } else {
    return launch_cfg<D, G, (D == 64 ? 2 : 1)>(tmK, tmV, p, grid, stream);
  }
}

template <int D>
pa_status dispatch_group(int G, const CUtensorMap& tmK, const CUtensorMap& tmV, const DecodeParams& p, dim3 grid,
                         cudaStream_t stream) {
  switch (G) {
    case 1: return launch_split<D, 1>(tmK, tmV, p, grid, stream);
    case 2: return launch_split<D, 2>(tmK, tmV, p, grid, stream);
    case 3: return launch_split<D, 3>(tmK, tmV, p, grid, stream);
    case 4: return launch_split<D, 4>(tmK, tmV, p, grid, stream);
    case 5: return launch_split<D, 5>(tmK, tmV, p, grid, stream);
    case 6: return launch_split<D, 6>(tmK, tmV, p, grid, stream);
    case 7: return launch_split<D, 7>(tmK, tmV, p, grid, stream);
    case 8: return launch_split<D, 8>(tmK, tmV, p, grid, stream);
    default: break;
  }
  set_last_error("decode: query heads per kv head = %d is not supported (1..8)", G);
  return PA_ERR_UNSUPPORTED;
}

}  // namespace

int32_t decode_auto_chunk(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int sm_count) {
  // Enough CTAs to fill every CTA slot (two per SM, as split launches run) several times over,
  // without chunks so short that per-CTA set-up dominates.
  constexpr int kMinChunk = 512;
  constexpr int kWavesTarget = 4;
  const int64_t units = static_cast<int64_t>(num_seqs) * num_kv_heads;
  if (max_context_len <= kMinChunk || units <= 0) return ((max(max_context_len, 1) + kTile - 1) / kTile) * kTile;
  const int64_t want = static_cast<int64_t>(kWavesTarget) * 2 * sm_count;
  if (units >= want) return ((max_context_len + kTile - 1) / kTile) * kTile;   // enough CTAs unsplit
  int64_t splits = (want + units - 1) / units;
  const int64_t max_splits = (max_context_len + kMinChunk - 1) / kMinChunk;
  splits = splits < 1 ? 1 : (splits > max_splits ? max_splits : splits);
  // Among one split fewer or more, prefer the count whose chunks (whole
  // tiles) cover the longest context with the least overhang: a short last
  // chunk leaves its CTA idle for most of a wave.  Ties go to fewer CTAs:
  // with the longest sequences dispatched first, fewer merges and CTA
  // set-ups pay more than the finer balance of smaller chunks.
  int64_t best_chunk = 0, best_waste = INT64_MAX;
  for (int64_t s2 = splits - 1; s2 <= splits + 1; ++s2) {
    if (s2 < 1 || s2 > max_splits) continue;
    const int64_t per = (max_context_len + s2 - 1) / s2;
    const int64_t chunk = ((per + kTile - 1) / kTile) * kTile;
    const int64_t waste = ((max_context_len + chunk - 1) / chunk) * chunk - max_context_len;
    if (waste < best_waste) {
      best_waste = waste;
      best_chunk = chunk;
    }
  }
  return static_cast<int32_t>(best_chunk);
}

pa_status launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int G = a.num_heads / a.num_kv_heads;
  const int box_rows = a.block_size < kTile ? a.block_size : kTile;
  CUtensorMap tmK, tmV;
  const uint64_t rows = static_cast<uint64_t>(a.num_blocks) * a.block_size;
  const uint64_t s1 = static_cast<uint64_t>(a.head_dim) * 2;
  const uint64_t s2 = s1 * a.num_kv_heads;
  if (!encode_bf16_3d(&tmK, a.k_cache, a.head_dim, a.num_kv_heads, rows, s1, s2, a.head_dim, 1, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !encode_bf16_3d(&tmV, a.v_cache, a.head_dim, a.num_kv_heads, rows, s1, s2, a.head_dim, 1, box_rows,
                      CU_TENSOR_MAP_SWIZZLE_NONE))
    return PA_ERR_INVALID_ARG;
  DecodeParams p;
  p.out = static_cast<__nv_bfloat16*>(a.out);
  p.q = static_cast<const __nv_bfloat16*>(a.q);
  p.block_tables = a.block_tables;
  p.context_lens = a.context_lens;
  p.ws_acc = a.ws_acc;
  p.ws_ml = a.ws_ml;
  p.o_part = a.o_part;
  p.lse_part = a.lse_part;
  p.max_blocks_per_seq = a.max_blocks_per_seq;
  p.max_context_len = a.max_context_len;
  p.num_heads = a.num_heads;
  p.block_size = a.block_size;
  p.box_rows = box_rows;
  p.chunk_tokens = a.chunk_tokens;
  p.max_chunks = a.max_chunks;
  p.scale_log2 = a.scale * 1.4426950408889634f;
  p.err = current_device_info()->error_word;
  p.num_kv_heads = a.num_kv_heads;
  p.o_stride = a.head_dim;
  p.new_k = static_cast<const __nv_bfloat16*>(a.new_k);
  p.new_v = static_cast<const __nv_bfloat16*>(a.new_v);
  p.new_k_stride = a.new_k_stride;
  p.new_v_stride = a.new_v_stride;
  p.slot_mapping = a.slot_mapping;
  p.k_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(a.k_cache));
  p.v_cache = static_cast<__nv_bfloat16*>(const_cast<void*>(a.v_cache));
  p.num_slots = static_cast<int64_t>(a.num_blocks) * a.block_size;
  p.num_blocks = a.num_blocks;
  static std::atomic<uint32_t> order_launches{0};
  const int64_t ctas = static_cast<int64_t>(a.max_chunks) * a.num_kv_heads * a.num_seqs;
  // the sequence positions whose CTAs all start in the first wave (at the
  // CTAs per SM that decode_ctas_per_sm gives this launch)
  const int per_sm = decode_ctas_per_sm(a.head_dim, G, a.max_chunks);
  // At least position 0 keeps its own sequence: CTA 0, which sorts the rest,
  // works on sequence 0 whatever the order says, so the sorted order must
  // start at position 1 even when one position's CTAs fill a whole wave.
  const int64_t wave_positions = static_cast<int64_t>(current_device_info()->sm_count) * per_sm /
                                 (static_cast<int64_t>(a.num_kv_heads) * a.max_chunks);
  p.order_first = static_cast<int32_t>(wave_positions > 1 ? wave_positions : 1);
  // only when some sequences come after the first wave
  p.order_slot = (a.num_seqs >= kOrderMinSeqs && a.num_seqs <= kOrderMaxSeqs &&
                  ctas <= kOrderMaxCtas && p.order_first < a.num_seqs)
                     ? static_cast<int32_t>(order_launches.fetch_add(1) % kOrderSlots)
                     : -1;
  static std::atomic<uint32_t> launches{0};
  const bool fused_merge = static_cast<int64_t>(a.num_seqs) * a.num_kv_heads <= kMergeCounters;
  p.merge_slot = (a.max_chunks > 1 && fused_merge) ? static_cast<int32_t>(launches.fetch_add(1) % kMergeSlots) : -1;
  const dim3 grid(static_cast<unsigned>(a.max_chunks), static_cast<unsigned>(a.num_kv_heads),
                  static_cast<unsigned>(a.num_seqs));
  pa_status st = a.head_dim == 128 ? dispatch_group<128>(G, tmK, tmV, p, grid, stream)
                                   : dispatch_group<64>(G, tmK, tmV, p, grid, stream);
  if (st != PA_OK || a.max_chunks <= 1 || p.merge_slot >= 0) return st;
  const int32_t rows_out = a.num_seqs * a.num_heads;
  const unsigned mblocks = static_cast<unsigned>((rows_out + 3) / 4);
  if (a.head_dim == 128)
    decode_merge_kernel<128><<<mblocks, 128, 0, stream>>>(p, rows_out);
  else
    decode_merge_kernel<64><<<mblocks, 128, 0, stream>>>(p, rows_out);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    set_last_error("decode merge launch: %s", cudaGetErrorString(e));
    return PA_ERR_CUDA;
  }
  return PA_OK;
}

}  // namespace pa

namespace pa {

cudaError_t launch_merge_lse(void* out, const float* o_parts, const float* lse_parts, int32_t num_parts,
                             int32_t num_rows, int32_t head_dim, cudaStream_t stream) {
  const unsigned blocks = static_cast<unsigned>((num_rows + 3) / 4);
  if (head_dim == 128)
    merge_lse_kernel<128><<<blocks, 128, 0, stream>>>(static_cast<__nv_bfloat16*>(out), o_parts, lse_parts,
                                                      num_parts, num_rows);
  else
    merge_lse_kernel<64><<<blocks, 128, 0, stream>>>(static_cast<__nv_bfloat16*>(out), o_parts, lse_parts,
                                                     num_parts, num_rows);
  return cudaGetLastError();
}

}  // namespace pa
