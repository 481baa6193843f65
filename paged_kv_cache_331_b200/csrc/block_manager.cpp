// Host-side KV-cache block manager: reference-counted cache blocks, chained
// full-block hashes for prefix caching, growth during decode, and the
// metadata arrays the attention kernels consume.
//
// ("Architektur im Überblick", "Block Manager und KV-Cache-Verwaltung",
// "Hash-basiertes Prefix Caching", "Dynamische Block-Erweiterung",
// "Kern-Designentscheidungen" 2 and "Prefill- und Decode-Vorbereitung"; the
// semantics the pages leave open are stated in pa_block_manager.h.)
//
// Layout: blocks live in flat arrays indexed by block id.  Free blocks form an
// intrusive doubly linked FIFO list (prev/next arrays), so taking the first
// free block, taking a specific block (a cache hit on a freed block) and
// releasing a block are all O(1).  The hash dictionary maps a 64-bit block
// hash to a block id (std::unordered_map).  A sequence holds its token ids, its
// number of cached tokens and its block table.
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <new>
#include <unordered_map>
#include <vector>

#include "pa_block_manager.h"

namespace pa {
void set_last_error(const char* fmt, ...);
}

namespace {

using pa::set_last_error;

pa_status bm_fail(pa_status st, const char* fmt, ...) {
  char buf[400];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_last_error("%s", buf);
  return st;
}

// ---------------------------------------------------------------- XXH64 --
// The 64-bit algorithm of the xxHash specification: four accumulators over
// 32-byte stripes, then the remaining 8-, 4- and 1-byte lanes, then the
// avalanche.
constexpr uint64_t kP1 = 0x9E3779B185EBCA87ull;
constexpr uint64_t kP2 = 0xC2B2AE3D27D4EB4Full;
constexpr uint64_t kP3 = 0x165667B19E3779F9ull;
constexpr uint64_t kP4 = 0x85EBCA77C2B2AE63ull;
constexpr uint64_t kP5 = 0x27D4EB2F165667C5ull;

inline uint64_t rotl64(uint64_t x, int r) { return (x << r) | (x >> (64 - r)); }
inline uint64_t read64(const unsigned char* p) {
  uint64_t v = 0;
  for (int i = 7; i >= 0; --i) v = (v << 8) | p[i];   // little-endian regardless of the host
  return v;
}
inline uint32_t read32(const unsigned char* p) {
  return static_cast<uint32_t>(p[0]) | (static_cast<uint32_t>(p[1]) << 8) | (static_cast<uint32_t>(p[2]) << 16) |
         (static_cast<uint32_t>(p[3]) << 24);
}
inline uint64_t xxh_round(uint64_t acc, uint64_t lane) { return rotl64(acc + lane * kP2, 31) * kP1; }
inline uint64_t xxh_merge(uint64_t acc, uint64_t v) { return (acc ^ xxh_round(0, v)) * kP1 + kP4; }

uint64_t xxh64(const unsigned char* p, size_t len, uint64_t seed) {
  const unsigned char* const end = p + len;
  uint64_t acc;
  if (len >= 32) {
    uint64_t v1 = seed + kP1 + kP2, v2 = seed + kP2, v3 = seed, v4 = seed - kP1;
    const unsigned char* const last_stripe = end - 32;
    do {
      v1 = xxh_round(v1, read64(p));
      v2 = xxh_round(v2, read64(p + 8));
      v3 = xxh_round(v3, read64(p + 16));
      v4 = xxh_round(v4, read64(p + 24));
      p += 32;
    } while (p <= last_stripe);
    acc = rotl64(v1, 1) + rotl64(v2, 7) + rotl64(v3, 12) + rotl64(v4, 18);
    acc = xxh_merge(acc, v1);
    acc = xxh_merge(acc, v2);
    acc = xxh_merge(acc, v3);
    acc = xxh_merge(acc, v4);
  } else {
    acc = seed + kP5;
  }
  acc += static_cast<uint64_t>(len);
  for (; p + 8 <= end; p += 8) acc = rotl64(acc ^ xxh_round(0, read64(p)), 27) * kP1 + kP4;
  if (p + 4 <= end) {
    acc = rotl64(acc ^ (static_cast<uint64_t>(read32(p)) * kP1), 23) * kP2 + kP3;
    p += 4;
  }
  for (; p < end; ++p) acc = rotl64(acc ^ (static_cast<uint64_t>(*p) * kP5), 11) * kP1;
  acc ^= acc >> 33;
  acc *= kP2;
  acc ^= acc >> 29;
  acc *= kP3;
  acc ^= acc >> 32;
  return acc;
}

uint64_t block_hash(const int32_t* tokens, int32_t n, bool has_prefix, uint64_t prefix,
                    std::vector<unsigned char>& scratch) {
  scratch.resize((has_prefix ? 8 : 0) + 4 * static_cast<size_t>(n));
  unsigned char* w = scratch.data();
  if (has_prefix)
    for (int i = 0; i < 8; ++i) *w++ = static_cast<unsigned char>(prefix >> (8 * i));
  for (int32_t t = 0; t < n; ++t) {
    const uint32_t v = static_cast<uint32_t>(tokens[t]);
    for (int i = 0; i < 4; ++i) *w++ = static_cast<unsigned char>(v >> (8 * i));
  }
  return xxh64(scratch.data(), scratch.size(), 0);
}

struct Sequence {
  std::vector<int32_t> tokens;
  int32_t num_cached_tokens = 0;
  std::vector<int32_t> table;
};

}  // namespace

struct pa_block_manager {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  // per block
  std::vector<int32_t> ref_count;
  std::vector<uint8_t> has_hash;
  std::vector<uint64_t> hash;
  std::vector<int32_t> tokens;      // num_blocks x block_size: the tokens a hashed block holds
  std::vector<int32_t> prev, next;  // free list links (-1 = none)
  std::vector<uint8_t> is_free;
  int32_t free_head = -1, free_tail = -1, num_free = 0;
  std::unordered_map<uint64_t, int32_t> hash_to_block;
  std::unordered_map<int64_t, Sequence> seqs;
  std::vector<unsigned char> scratch;

  int32_t nblocks_of(const Sequence& s) const {
    return static_cast<int32_t>((s.tokens.size() + block_size - 1) / block_size);
  }

  void push_free(int32_t b) {   // append at the tail
    prev[b] = free_tail;
    next[b] = -1;
    if (free_tail >= 0) next[free_tail] = b; else free_head = b;
    free_tail = b;
    is_free[b] = 1;
    ++num_free;
  }
  void unlink_free(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else free_head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else free_tail = prev[b];
    prev[b] = next[b] = -1;
    is_free[b] = 0;
    --num_free;
  }
  // Give a free block a new owner: its old dictionary entry goes, it starts unhashed.
  void take(int32_t b) {
    if (has_hash[b]) {
      auto it = hash_to_block.find(hash[b]);
      if (it != hash_to_block.end() && it->second == b) hash_to_block.erase(it);
    }
    unlink_free(b);
    ref_count[b] = 1;
    has_hash[b] = 0;
  }
  void seal(int32_t b, uint64_t h, const int32_t* toks) {   // record a full block's hash and tokens
    has_hash[b] = 1;
    hash[b] = h;
    std::memcpy(&tokens[static_cast<size_t>(b) * block_size], toks, sizeof(int32_t) * block_size);
    hash_to_block[h] = b;
  }
  bool same_tokens(int32_t b, const int32_t* toks) const {
    return has_hash[b] && std::memcmp(&tokens[static_cast<size_t>(b) * block_size], toks,
                                      sizeof(int32_t) * block_size) == 0;
  }
};

namespace {

Sequence* find_seq(pa_block_manager* bm, int64_t id) {
  auto it = bm->seqs.find(id);
  return it == bm->seqs.end() ? nullptr : &it->second;
}
const Sequence* find_seq(const pa_block_manager* bm, int64_t id) {
  auto it = bm->seqs.find(id);
  return it == bm->seqs.end() ? nullptr : &it->second;
}

void release_table(pa_block_manager* bm, Sequence& s) {
  for (auto it = s.table.rbegin(); it != s.table.rend(); ++it)
    if (--bm->ref_count[*it] == 0) bm->push_free(*it);
  s.table.clear();
  s.num_cached_tokens = 0;
}

}  // namespace

extern "C" {

uint64_t pa_xxh64(const void* data, size_t len, uint64_t seed) {
  return xxh64(static_cast<const unsigned char*>(data), data ? len : 0, seed);
}

uint64_t pa_bm_block_hash(const int32_t* token_ids, int32_t n, int32_t has_prefix, uint64_t prefix) {
  std::vector<unsigned char> scratch;
  return block_hash(token_ids, n > 0 && token_ids ? n : 0, has_prefix != 0, prefix, scratch);
}

pa_block_manager* pa_bm_create(int32_t num_blocks, int32_t block_size) {
  set_last_error("");
  if (num_blocks <= 0 || block_size < 2) {
    bm_fail(PA_ERR_INVALID_ARG, "pa_bm_create: need num_blocks > 0 and block_size >= 2");
    return nullptr;
  }
  pa_block_manager* bm = new (std::nothrow) pa_block_manager;
  if (!bm) return nullptr;
  try {
    bm->num_blocks = num_blocks;
    bm->block_size = block_size;
    bm->ref_count.assign(num_blocks, 0);
    bm->has_hash.assign(num_blocks, 0);
    bm->hash.assign(num_blocks, 0);
    bm->tokens.assign(static_cast<size_t>(num_blocks) * block_size, 0);
    bm->prev.assign(num_blocks, -1);
    bm->next.assign(num_blocks, -1);
    bm->is_free.assign(num_blocks, 0);
    for (int32_t b = 0; b < num_blocks; ++b) bm->push_free(b);
  } catch (...) {
    delete bm;
    bm_fail(PA_ERR_INVALID_ARG, "pa_bm_create: out of memory");
    return nullptr;
  }
  return bm;
}

void pa_bm_destroy(pa_block_manager* bm) { delete bm; }

int32_t pa_bm_num_free_blocks(const pa_block_manager* bm) { return bm ? bm->num_free : -1; }

pa_status pa_bm_add_sequence(pa_block_manager* bm, int64_t seq_id, const int32_t* token_ids, int32_t num_tokens) {
  set_last_error("");
  if (!bm || num_tokens <= 0 || !token_ids) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_add_sequence: need tokens");
  if (bm->seqs.count(seq_id)) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_add_sequence: sequence %lld exists",
                                             static_cast<long long>(seq_id));
  Sequence& s = bm->seqs[seq_id];
  s.tokens.assign(token_ids, token_ids + num_tokens);
  return PA_OK;
}

pa_status pa_bm_append_token(pa_block_manager* bm, int64_t seq_id, int32_t token_id) {
  set_last_error("");
  Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_append_token: unknown sequence");
  s->tokens.push_back(token_id);
  return PA_OK;
}

pa_status pa_bm_remove_sequence(pa_block_manager* bm, int64_t seq_id) {
  set_last_error("");
  Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_remove_sequence: unknown sequence");
  release_table(bm, *s);
  bm->seqs.erase(seq_id);
  return PA_OK;
}

int32_t pa_bm_can_allocate(const pa_block_manager* bm, int64_t seq_id) {
  const Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return -1;
  return bm->num_free >= bm->nblocks_of(*s) ? 1 : 0;
}

pa_status pa_bm_allocate(pa_block_manager* bm, int64_t seq_id) {
  set_last_error("");
  Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_allocate: unknown sequence");
  if (!s->table.empty()) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_allocate: sequence already holds blocks");
  const int32_t bs = bm->block_size, nb = bm->nblocks_of(*s);
  // Fresh blocks needed = blocks after the leading run of hits, plus hits on
  // freed blocks (they leave the free list too): check before changing state.
  {
    int32_t need = 0;
    bool has = false, miss = false;
    uint64_t h = 0;
    for (int32_t i = 0; i < nb; ++i) {
      const int32_t* toks = s->tokens.data() + static_cast<size_t>(i) * bs;
      const bool full = static_cast<int64_t>(i + 1) * bs <= static_cast<int64_t>(s->tokens.size());
      if (full) h = block_hash(toks, bs, has, h, bm->scratch);
      has = full;
      if (!miss) {
        auto it = has ? bm->hash_to_block.find(h) : bm->hash_to_block.end();
        if (it == bm->hash_to_block.end() || !bm->same_tokens(it->second, toks)) miss = true;
        else if (bm->ref_count[it->second] == 0) ++need;
      }
      if (miss) ++need;
    }
    if (need > bm->num_free)
      return bm_fail(PA_ERR_NO_FREE_BLOCK, "pa_bm_allocate: %d free blocks, %d needed", bm->num_free, need);
  }
  bool has = false, miss = false;
  uint64_t h = 0;
  for (int32_t i = 0; i < nb; ++i) {
    const int32_t* toks = s->tokens.data() + static_cast<size_t>(i) * bs;
    const bool full = static_cast<int64_t>(i + 1) * bs <= static_cast<int64_t>(s->tokens.size());
    if (full) h = block_hash(toks, bs, has, h, bm->scratch);
    has = full;
    int32_t b = -1;
    if (!miss) {
      auto it = has ? bm->hash_to_block.find(h) : bm->hash_to_block.end();
      if (it != bm->hash_to_block.end() && bm->same_tokens(it->second, toks)) b = it->second;
      else miss = true;
    }
    if (miss) {
      b = bm->free_head;
      bm->take(b);
    } else {
      s->num_cached_tokens += bs;
      if (bm->ref_count[b] > 0) ++bm->ref_count[b];
      else bm->take(b);   // freed but still holding this content: revive it
    }
    if (has) bm->seal(b, h, toks);
    s->table.push_back(b);
  }
  return PA_OK;
}

pa_status pa_bm_deallocate(pa_block_manager* bm, int64_t seq_id) {
  set_last_error("");
  Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_deallocate: unknown sequence");
  release_table(bm, *s);
  return PA_OK;
}

int32_t pa_bm_can_append(const pa_block_manager* bm, int64_t seq_id) {
  const Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return -1;
  const bool needs = s->tokens.size() % bm->block_size == 1;
  return bm->num_free >= (needs ? 1 : 0) ? 1 : 0;
}

pa_status pa_bm_may_append(pa_block_manager* bm, int64_t seq_id) {
  set_last_error("");
  Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_may_append: unknown sequence");
  if (s->table.empty()) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_may_append: sequence holds no blocks");
  const int32_t bs = bm->block_size;
  const size_t n = s->tokens.size();
  const int32_t last = s->table.back();
  if (n % bs == 1) {
    if (static_cast<int32_t>(s->table.size()) != bm->nblocks_of(*s) - 1 || !bm->has_hash[last])
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_may_append: table does not end in a full block");
    if (bm->num_free == 0) return bm_fail(PA_ERR_NO_FREE_BLOCK, "pa_bm_may_append: no free block");
    const int32_t b = bm->free_head;
    bm->take(b);
    s->table.push_back(b);
  } else if (n % bs == 0) {
    if (static_cast<int32_t>(s->table.size()) != bm->nblocks_of(*s) || bm->has_hash[last])
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_may_append: last block already sealed or table short");
    const size_t k = s->table.size();
    const bool has_prefix = k > 1;
    const uint64_t prefix = has_prefix ? bm->hash[s->table[k - 2]] : 0;
    const int32_t* toks = s->tokens.data() + (k - 1) * bs;
    bm->seal(last, block_hash(toks, bs, has_prefix, prefix, bm->scratch), toks);
  } else {
    if (static_cast<int32_t>(s->table.size()) != bm->nblocks_of(*s) || bm->has_hash[last])
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_may_append: table out of step with the tokens");
  }
  return PA_OK;
}

pa_status pa_bm_sequence_info(const pa_block_manager* bm, int64_t seq_id, int32_t* num_tokens,
                              int32_t* num_cached_tokens, int32_t* num_table_blocks) {
  set_last_error("");
  const Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_sequence_info: unknown sequence");
  if (num_tokens) *num_tokens = static_cast<int32_t>(s->tokens.size());
  if (num_cached_tokens) *num_cached_tokens = s->num_cached_tokens;
  if (num_table_blocks) *num_table_blocks = static_cast<int32_t>(s->table.size());
  return PA_OK;
}

pa_status pa_bm_block_table(const pa_block_manager* bm, int64_t seq_id, int32_t* out, int32_t capacity) {
  set_last_error("");
  const Sequence* s = bm ? find_seq(bm, seq_id) : nullptr;
  if (!s) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_block_table: unknown sequence");
  if (!out || capacity < static_cast<int32_t>(s->table.size()))
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_block_table: buffer of %d entries for %zu blocks", capacity,
                   s->table.size());
  std::memcpy(out, s->table.data(), sizeof(int32_t) * s->table.size());
  return PA_OK;
}

pa_status pa_bm_block_info(const pa_block_manager* bm, int32_t block_id, int32_t* ref_count, int32_t* has_hash,
                           uint64_t* hash) {
  set_last_error("");
  if (!bm || block_id < 0 || block_id >= bm->num_blocks)
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_block_info: block id out of range");
  if (ref_count) *ref_count = bm->ref_count[block_id];
  if (has_hash) *has_hash = bm->has_hash[block_id];
  if (hash) *hash = bm->hash[block_id];
  return PA_OK;
}

pa_status pa_bm_prepare_prefill(const pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                                int32_t max_blocks_per_seq, int32_t token_capacity, int32_t* block_tables,
                                int32_t* cu_seqlens_q, int32_t* cu_seqlens_k, int32_t* slot_mapping,
                                int32_t* positions, int32_t* total_q) {
  set_last_error("");
  if (!bm || num_seqs < 0 || (num_seqs > 0 && (!seq_ids || !block_tables)) || !cu_seqlens_q || !cu_seqlens_k ||
      !total_q || max_blocks_per_seq <= 0 || token_capacity < 0)
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_prefill: bad arguments");
  // validate everything first, so that nothing is written on failure
  int64_t need = 0, keys = 0;
  for (int32_t r = 0; r < num_seqs; ++r) {
    const Sequence* s = find_seq(bm, seq_ids[r]);
    if (!s || s->table.empty()) return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_prefill: sequence %d not allocated", r);
    if (static_cast<int32_t>(s->table.size()) > max_blocks_per_seq)
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_prefill: %zu blocks exceed max_blocks_per_seq",
                     s->table.size());
    need += static_cast<int64_t>(s->tokens.size()) - s->num_cached_tokens;
    keys += static_cast<int64_t>(s->tokens.size());
  }
  if (need > token_capacity || keys > INT32_MAX)
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_prefill: %lld new tokens, capacity %d",
                   static_cast<long long>(need), token_capacity);
  if (need > 0 && (!slot_mapping || !positions))
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_prefill: null slot_mapping or positions");
  const int32_t bs = bm->block_size;
  cu_seqlens_q[0] = cu_seqlens_k[0] = 0;
  int32_t t = 0;
  for (int32_t r = 0; r < num_seqs; ++r) {
    const Sequence& s = *find_seq(bm, seq_ids[r]);
    const int32_t n = static_cast<int32_t>(s.tokens.size());
    int32_t* row = block_tables + static_cast<int64_t>(r) * max_blocks_per_seq;
    for (int32_t i = 0; i < max_blocks_per_seq; ++i)
      row[i] = i < static_cast<int32_t>(s.table.size()) ? s.table[i] : -1;
    for (int32_t p = s.num_cached_tokens; p < n; ++p, ++t) {
      positions[t] = p;
      slot_mapping[t] = s.table[p / bs] * bs + p % bs;
    }
    cu_seqlens_q[r + 1] = cu_seqlens_q[r] + (n - s.num_cached_tokens);
    cu_seqlens_k[r + 1] = cu_seqlens_k[r] + n;
  }
  *total_q = t;
  return PA_OK;
}

pa_status pa_bm_prepare_decode(const pa_block_manager* bm, const int64_t* seq_ids, int32_t num_seqs,
                               int32_t max_blocks_per_seq, int32_t* block_tables, int32_t* context_lens,
                               int32_t* slot_mapping, int32_t* positions) {
  set_last_error("");
  if (!bm || num_seqs < 0 || max_blocks_per_seq <= 0 ||
      (num_seqs > 0 && (!seq_ids || !block_tables || !context_lens || !slot_mapping || !positions)))
    return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_decode: bad arguments");
  for (int32_t r = 0; r < num_seqs; ++r) {
    const Sequence* s = find_seq(bm, seq_ids[r]);
    if (!s || static_cast<int32_t>(s->table.size()) != bm->nblocks_of(*s))
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_decode: sequence %d has no block for its last token", r);
    if (static_cast<int32_t>(s->table.size()) > max_blocks_per_seq)
      return bm_fail(PA_ERR_INVALID_ARG, "pa_bm_prepare_decode: %zu blocks exceed max_blocks_per_seq",
                     s->table.size());
  }
  const int32_t bs = bm->block_size;
  for (int32_t r = 0; r < num_seqs; ++r) {
    const Sequence& s = *find_seq(bm, seq_ids[r]);
    const int32_t n = static_cast<int32_t>(s.tokens.size());
    int32_t* row = block_tables + static_cast<int64_t>(r) * max_blocks_per_seq;
    for (int32_t i = 0; i < max_blocks_per_seq; ++i)
      row[i] = i < static_cast<int32_t>(s.table.size()) ? s.table[i] : -1;
    context_lens[r] = n;
    positions[r] = n - 1;
    slot_mapping[r] = s.table[(n - 1) / bs] * bs + (n - 1) % bs;
  }
  return PA_OK;
}

}  // extern "C"
