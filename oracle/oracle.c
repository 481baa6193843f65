/*
 * Oracle for attention over a paged KV cache -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct CPU restatement of what the hot path computes.
 * Only the tests, the package's smoke check and the bench's CPU-baseline leg
 * may load this library; the product path never does.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Arithmetic: bf16 inputs are widened exactly to double; scores, softmax and
 * the weighted sum are computed in double; outputs are rounded once to bf16
 * (nearest, ties to even).  No blocking, fusion or reordering: every output
 * row walks its block table token by token.
 *
 * Sources (web pages about nano-vllm):
 *  - "Architektur im Überblick", section "Dynamische KV-Cache-Allokation":
 *    per layer the cache is k_cache/v_cache [num_blocks, block_size,
 *    num_kv_heads, head_dim].
 *  - same page, "Prefill- und Decode-Vorbereitung": one slot per new token,
 *    slots are consecutive within each non-cached block; positions of the
 *    computed tokens start at num_cached_tokens.
 *  - same page, "Block-Berechnung und Token-Appending": num_blocks =
 *    ceil(num_tokens / block_size).
 *  - lshu.cn essay on Nano-vLLM, §3.2 (memory manager and paged attention):
 *    a logical position maps to page pos / page_size and offset
 *    pos % page_size of that sequence's page table; attention gathers K/V
 *    from those scattered pages.
 *  - "Nano-vLLM 源碼學習", §二.2 (attention layer): a store_kvcache kernel
 *    writes new K/V into the cache, prefill runs varlen attention with prefix
 *    cache support, decode runs attention against the cache.
 *  - "Architektur im Überblick", "Attention-Mechanismus": GQA through a
 *    separate num_kv_heads; query head h reads kv head h / (num_heads /
 *    num_kv_heads).
 *  - "Nano-vLLM 源碼學習", layers, 7 (rotary_embedding.py): rotary position
 *    embedding of q and k from sines and cosines of the position.
 *
 * Every function validates its arguments and returns 0 on success or a
 * negative code: -1 bad argument, -2 block id, slot or position out of range.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Planted-mistake builds (-DORACLE_MUTANT=k) exist only so that the tests
 * can show each pin catches a plausible error.  The default build has none. */
#ifndef ORACLE_MUTANT
#define ORACLE_MUTANT 0
#endif

/* ---------------------------------------------------------------- bf16 --- */

static double bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Round a double to the nearest bf16 (8 significant bits, float's exponent
 * range), ties to even, in one step: scale to the bf16 quantum of x's binade
 * and round to an integer with nearbyint (default mode: nearest-even). */
static uint16_t double_to_bf16(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int e;
    frexp(a, &e);                    /* a = m * 2^e, m in [0.5, 1) */
    if (e < -125) e = -125;          /* below 2^-126 the quantum is fixed (subnormals) */
#if ORACLE_MUTANT == 8
    double r = floor(a / ldexp(1.0, e - 8)) * ldexp(1.0, e - 8);     /* truncation */
#else
    double quantum = ldexp(1.0, e - 8);
    double r = nearbyint(a / quantum) * quantum;
#endif
    if (r >= ldexp(1.0, 128)) return sign | 0x7F80;
    float rf = (float)r;             /* exact: r has at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &rf, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

int oracle_bf16_round(const double* x, uint16_t* out, int64_t n)
{
    if (n < 0 || (n && (!x || !out))) return -1;
    for (int64_t i = 0; i < n; ++i) out[i] = double_to_bf16(x[i]);
    return 0;
}

/* ------------------------------------------------------ page-table walk --- */

/* Physical (block, offset) of logical position pos of sequence b: the
 * page index is pos / block_size, the offset pos % block_size (lshu.cn §3.2). */
int oracle_kv_location(const int32_t* block_tables, int32_t max_blocks_per_seq, int32_t b, int32_t pos,
                       int32_t block_size, int32_t num_blocks, int32_t* blk_out, int32_t* off_out)
{
    if (!block_tables || block_size <= 0 || pos < 0 || b < 0) return -1;
#if ORACLE_MUTANT == 6
    int32_t page = pos >> 8;                           /* block size hard-wired to 256 */
#else
    int32_t page = pos / block_size;
#endif
#if ORACLE_MUTANT == 4
    int32_t off = (pos + 1) % block_size;
#else
    int32_t off = pos % block_size;
#endif
    if (page >= max_blocks_per_seq) return -2;
    int32_t blk = block_tables[(int64_t)b * max_blocks_per_seq + page];
    if (blk < 0 || blk >= num_blocks) return -2;
    *blk_out = blk;
    *off_out = off;
    return 0;
}

static const uint16_t* kv_row(const uint16_t* cache, int32_t blk, int32_t off, int32_t block_size,
                              int32_t num_kv_heads, int32_t head_dim, int32_t kvh)
{
    return cache + (((int64_t)blk * block_size + off) * num_kv_heads + kvh) * head_dim;
}

static int32_t kv_head_of(int32_t h, int32_t num_heads, int32_t num_kv_heads)
{
#if ORACLE_MUTANT == 1
    (void)num_heads;
    return h % num_kv_heads;
#else
    return h / (num_heads / num_kv_heads);
#endif
}

/* ---------------------------------------------------------------- store --- */

/* store_kvcache ("Nano-vLLM 源碼學習" §二.2): for every new token t whose slot
 * is not -1, copy its K and V rows (num_kv_heads * head_dim values) into row
 * slot of the cache viewed as [num_blocks * block_size, num_kv_heads, head_dim],
 * i.e. block slot / block_size, offset slot % block_size.  A bit copy. */
int oracle_store_kvcache(const uint16_t* key, const uint16_t* value, int64_t key_row_stride,
                         int64_t value_row_stride, uint16_t* k_cache, uint16_t* v_cache,
                         const int32_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, int32_t num_blocks)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0) return -1;
    if (num_tokens == 0) return 0;
    if (!key || !value || !k_cache || !v_cache || !slot_mapping) return -1;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (key_row_stride < row || value_row_stride < row) return -1;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int32_t slot = slot_mapping[t];
#if ORACLE_MUTANT == 7
        if (slot == -1) slot = 0;                      /* skip rule lost */
#endif
        if (slot == -1) continue;
        if (slot < 0 || (int64_t)slot >= (int64_t)num_blocks * block_size) return -2;
        int32_t blk = slot / block_size, off = slot % block_size;
        uint16_t* kd = k_cache + ((int64_t)blk * block_size + off) * row;
        uint16_t* vd = v_cache + ((int64_t)blk * block_size + off) * row;
        memcpy(kd, key + (int64_t)t * key_row_stride, (size_t)row * sizeof(uint16_t));
        memcpy(vd, value + (int64_t)t * value_row_stride, (size_t)row * sizeof(uint16_t));
    }
    return 0;
}

/* ------------------------------------------------------------ attention --- */

/* Softmax attention of one query row over logical keys [0, n) of sequence b:
 *   s_j = scale * <q, k_j>,  p_j = exp(s_j - max s),  o = sum_j p_j v_j / sum_j p_j
 * with k_j, v_j gathered through the block table.  Writes head_dim doubles.
 * n == 0 gives o = 0.  Returns 0 or a negative code. */
static int attend_row(double* o, const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                      const int32_t* block_tables, int32_t max_blocks_per_seq, int32_t b, int32_t n,
                      int32_t kvh, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int32_t num_blocks, double scale, double* s /* scratch, n doubles */)
{
    for (int32_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    if (n <= 0) return 0;
    double m = -INFINITY;
    for (int32_t j = 0; j < n; ++j) {
        int32_t blk, off;
        int rc = oracle_kv_location(block_tables, max_blocks_per_seq, b, j, block_size, num_blocks, &blk, &off);
        if (rc) return rc;
        const uint16_t* k = kv_row(k_cache, blk, off, block_size, num_kv_heads, head_dim, kvh);
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) dot += bf16_to_double(q[d]) * bf16_to_double(k[d]);
#if ORACLE_MUTANT == 3
        s[j] = dot;
#else
        s[j] = scale * dot;
#endif
        if (s[j] > m) m = s[j];
    }
    double denom = 0.0;
    for (int32_t j = 0; j < n; ++j) {
        int32_t blk, off;
        oracle_kv_location(block_tables, max_blocks_per_seq, b, j, block_size, num_blocks, &blk, &off);
        const uint16_t* v = kv_row(v_cache, blk, off, block_size, num_kv_heads, head_dim, kvh);
        double p = exp(s[j] - m);
        denom += p;
        for (int32_t d = 0; d < head_dim; ++d) o[d] += p * bf16_to_double(v[d]);
    }
#if ORACLE_MUTANT != 9
    for (int32_t d = 0; d < head_dim; ++d) o[d] /= denom;
#endif
    return 0;
}

static int set_threads(int nthreads)
{
#ifdef _OPENMP
    int n = nthreads > 0 ? nthreads : omp_get_max_threads();
    return n;
#else
    (void)nthreads;
    return 1;
#endif
}

/* Decode ("Nano-vLLM 源碼學習" §二.2, decode stage): one query token per
 * sequence attends keys 0 .. context_lens[b]-1 of its own block table; the
 * newest token (position context_lens[b]-1) was stored beforehand.
 * q, out: [num_seqs, num_heads, head_dim].  out_f64 (optional) receives the
 * unrounded result. */
int oracle_decode(uint16_t* out, double* out_f64, const uint16_t* q, const uint16_t* k_cache,
                  const uint16_t* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                  const int32_t* context_lens, int32_t num_seqs, int32_t num_heads, int32_t num_kv_heads,
                  int32_t head_dim, int32_t block_size, int32_t num_blocks, double scale, int nthreads)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return -1;
    if (num_heads % num_kv_heads) return -1;
    if (num_seqs == 0) return 0;
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || (!out && !out_f64)) return -1;
    int32_t maxL = 0;
    for (int32_t b = 0; b < num_seqs; ++b) {
        if (context_lens[b] < 0) return -1;
        if (context_lens[b] > maxL) maxL = context_lens[b];
    }
    int err = 0;
    int nt = set_threads(nthreads);
    const int64_t rows = (int64_t)num_seqs * num_heads;
#pragma omp parallel num_threads(nt)
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(maxL > 0 ? maxL : 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)head_dim);
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < rows; ++r) {
            int32_t b = (int32_t)(r / num_heads), h = (int32_t)(r % num_heads);
            int32_t kvh = kv_head_of(h, num_heads, num_kv_heads);
            int rc = attend_row(o, q + r * head_dim, k_cache, v_cache, block_tables, max_blocks_per_seq, b,
                                context_lens[b], kvh, num_kv_heads, head_dim, block_size, num_blocks, scale, s);
            if (rc) {
#pragma omp atomic write
                err = rc;
            }
            for (int32_t d = 0; d < head_dim; ++d) {
                if (out) out[r * head_dim + d] = double_to_bf16(o[d]);
                if (out_f64) out_f64[r * head_dim + d] = o[d];
            }
        }
        free(s);
        free(o);
    }
    return err;
}

/* Split-KV partials: the keys of each sequence are cut into chunks of
 * chunk_len tokens; for chunk c (keys [c*chunk_len, min((c+1)*chunk_len, L)))
 * and head h: m = max_j s_j, l = sum_j exp(s_j - m), acc = sum_j exp(s_j - m) v_j.
 * Empty chunks get m = -inf, l = 0, acc = 0.  Layout: m, l [B, H, C];
 * acc [B, H, C, D] with C = num_chunks. */
int oracle_decode_partials(double* m_out, double* l_out, double* acc_out, const uint16_t* q,
                           const uint16_t* k_cache, const uint16_t* v_cache, const int32_t* block_tables,
                           int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_seqs,
                           int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                           int32_t num_blocks, double scale, int32_t chunk_len, int32_t num_chunks)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return -1;
    if (chunk_len <= 0 || num_chunks <= 0 || num_heads % num_kv_heads) return -1;
    for (int32_t b = 0; b < num_seqs; ++b)
        if (context_lens[b] < 0 || context_lens[b] > (int64_t)chunk_len * num_chunks) return -1;
    for (int32_t b = 0; b < num_seqs; ++b) {
        for (int32_t h = 0; h < num_heads; ++h) {
            int32_t kvh = kv_head_of(h, num_heads, num_kv_heads);
            const uint16_t* qr = q + ((int64_t)b * num_heads + h) * head_dim;
            for (int32_t c = 0; c < num_chunks; ++c) {
                int64_t idx = ((int64_t)b * num_heads + h) * num_chunks + c;
                double* acc = acc_out + idx * head_dim;
                int32_t j0 = c * chunk_len, j1 = j0 + chunk_len;
                if (j1 > context_lens[b]) j1 = context_lens[b];
                double m = -INFINITY, l = 0.0;
                for (int32_t d = 0; d < head_dim; ++d) acc[d] = 0.0;
                for (int32_t j = j0; j < j1; ++j) {
                    int32_t blk, off;
                    int rc = oracle_kv_location(block_tables, max_blocks_per_seq, b, j, block_size, num_blocks,
                                                &blk, &off);
                    if (rc) return rc;
                    const uint16_t* k = kv_row(k_cache, blk, off, block_size, num_kv_heads, head_dim, kvh);
                    double dot = 0.0;
                    for (int32_t d = 0; d < head_dim; ++d) dot += bf16_to_double(qr[d]) * bf16_to_double(k[d]);
                    if (scale * dot > m) m = scale * dot;
                }
                for (int32_t j = j0; j < j1; ++j) {
                    int32_t blk, off;
                    oracle_kv_location(block_tables, max_blocks_per_seq, b, j, block_size, num_blocks, &blk, &off);
                    const uint16_t* k = kv_row(k_cache, blk, off, block_size, num_kv_heads, head_dim, kvh);
                    const uint16_t* v = kv_row(v_cache, blk, off, block_size, num_kv_heads, head_dim, kvh);
                    double dot = 0.0;
                    for (int32_t d = 0; d < head_dim; ++d) dot += bf16_to_double(qr[d]) * bf16_to_double(k[d]);
                    double p = exp(scale * dot - m);
                    l += p;
                    for (int32_t d = 0; d < head_dim; ++d) acc[d] += p * bf16_to_double(v[d]);
                }
                m_out[idx] = m;
                l_out[idx] = l;
            }
        }
    }
    return 0;
}

/* Merge of split-KV partials (log-sum-exp rescaling):
 *   M = max_c m_c,  o = sum_c exp(m_c - M) acc_c / sum_c exp(m_c - M) l_c.
 * Chunks with l_c == 0 contribute nothing; a row with no keys gives o = 0. */
int oracle_merge_partials(uint16_t* out, double* out_f64, const double* m_in, const double* l_in,
                          const double* acc_in, int32_t num_rows, int32_t num_chunks, int32_t head_dim)
{
    if (num_rows < 0 || num_chunks <= 0 || head_dim <= 0) return -1;
    for (int32_t r = 0; r < num_rows; ++r) {
        double M = -INFINITY;
        for (int32_t c = 0; c < num_chunks; ++c)
            if (l_in[(int64_t)r * num_chunks + c] > 0.0 && m_in[(int64_t)r * num_chunks + c] > M)
                M = m_in[(int64_t)r * num_chunks + c];
        double denom = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) {
            double num = 0.0;
            for (int32_t c = 0; c < num_chunks; ++c) {
                int64_t idx = (int64_t)r * num_chunks + c;
#if ORACLE_MUTANT == 10
                if (l_in[idx] > 0.0) num += acc_in[idx * head_dim + d];        /* no rescaling */
#else
                if (l_in[idx] > 0.0) num += exp(m_in[idx] - M) * acc_in[idx * head_dim + d];
#endif
            }
            if (d == 0) {
                for (int32_t c = 0; c < num_chunks; ++c) {
                    int64_t idx = (int64_t)r * num_chunks + c;
#if ORACLE_MUTANT == 10
                    if (l_in[idx] > 0.0) denom += l_in[idx];
#else
                    if (l_in[idx] > 0.0) denom += exp(m_in[idx] - M) * l_in[idx];
#endif
                }
            }
            double o = denom > 0.0 ? num / denom : 0.0;
            if (out) out[(int64_t)r * head_dim + d] = double_to_bf16(o);
            if (out_f64) out_f64[(int64_t)r * head_dim + d] = o;
        }
    }
    return 0;
}

/* Varlen prefill with prefix cache ("Nano-vLLM 源碼學習" §二.2, prefill stage;
 * "Architektur im Überblick", "Prefill- und Decode-Vorbereitung"): sequence b
 * has Lq = cu_seqlens_q[b+1]-cu_seqlens_q[b] new query tokens and
 * Lk = cu_seqlens_k[b+1]-cu_seqlens_k[b] keys in the cache (cached prefix plus
 * the new tokens, stored beforehand).  The new tokens occupy the last Lq
 * positions, so query i sits at position Lk - Lq + i and, when causal, attends
 * keys 0 .. Lk - Lq + i; otherwise keys 0 .. Lk-1.
 * q, out: [total_q, num_heads, head_dim].  row_select (optional, total_q
 * bytes): compute only tokens whose byte is nonzero, leave the rest untouched. */
int oracle_prefill_varlen(uint16_t* out, double* out_f64, const uint16_t* q, const uint16_t* k_cache,
                          const uint16_t* v_cache, const int32_t* cu_seqlens_q, const int32_t* cu_seqlens_k,
                          const int32_t* block_tables, int32_t max_blocks_per_seq, int32_t num_seqs,
                          int32_t num_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                          int32_t num_blocks, double scale, int32_t causal, const uint8_t* row_select,
                          int nthreads)
{
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0) return -1;
    if (num_heads % num_kv_heads) return -1;
    if (num_seqs == 0) return 0;
    if (!q || !k_cache || !v_cache || !cu_seqlens_q || !cu_seqlens_k || !block_tables || (!out && !out_f64))
        return -1;
    int32_t maxLk = 0;
    for (int32_t b = 0; b < num_seqs; ++b) {
        int32_t Lq = cu_seqlens_q[b + 1] - cu_seqlens_q[b], Lk = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
        if (Lq < 0 || Lk < Lq) return -1;
        if (Lk > maxLk) maxLk = Lk;
    }
    const int32_t total_q = cu_seqlens_q[num_seqs] - cu_seqlens_q[0];
    int err = 0;
    int nt = set_threads(nthreads);
    const int64_t rows = (int64_t)total_q * num_heads;
#pragma omp parallel num_threads(nt)
    {
        double* s = (double*)malloc(sizeof(double) * (size_t)(maxLk > 0 ? maxLk : 1));
        double* o = (double*)malloc(sizeof(double) * (size_t)head_dim);
#pragma omp for schedule(dynamic, 4)
        for (int64_t r = 0; r < rows; ++r) {
            int32_t t = (int32_t)(r / num_heads), h = (int32_t)(r % num_heads);
            if (row_select && !row_select[t]) continue;
            int32_t b = 0;
            while (cu_seqlens_q[b + 1] - cu_seqlens_q[0] <= t) ++b;   /* sequence owning token t */
            int32_t Lq = cu_seqlens_q[b + 1] - cu_seqlens_q[b], Lk = cu_seqlens_k[b + 1] - cu_seqlens_k[b];
            int32_t i = t - (cu_seqlens_q[b] - cu_seqlens_q[0]);
#if ORACLE_MUTANT == 2
            int32_t n = causal ? (Lk - Lq + i) : Lk;        /* off by one: drops the diagonal */
#elif ORACLE_MUTANT == 5
            int32_t n = causal ? (i + 1) : Lk;              /* top-left alignment: ignores the prefix */
#else
            int32_t n = causal ? (Lk - Lq + i + 1) : Lk;
#endif
            int32_t kvh = kv_head_of(h, num_heads, num_kv_heads);
            int rc = attend_row(o, q + r * head_dim, k_cache, v_cache, block_tables, max_blocks_per_seq, b, n, kvh,
                                num_kv_heads, head_dim, block_size, num_blocks, scale, s);
            if (rc) {
#pragma omp atomic write
                err = rc;
            }
            for (int32_t d = 0; d < head_dim; ++d) {
                if (out) out[r * head_dim + d] = double_to_bf16(o[d]);
                if (out_f64) out_f64[r * head_dim + d] = o[d];
            }
        }
        free(s);
        free(o);
    }
    return err;
}

/* ----------------------------------------------------------------- rope --- */

/* Rotary position embedding.  "Nano-vLLM 源碼學習", layers, 7 (rotary_embedding.py):
 * the RotaryEmbedding class adds position information to the query and the key
 * through sines and cosines of the position; "Architektur im Überblick",
 * Attention-Mechanismus: the attention layer applies its rotary_emb to q and k
 * before attention.  The pages print no formula.  Read as RoFormer's rotation
 * over the whole head, element i paired with element i + D/2 (the layout of
 * the Qwen models the pages serve), for frequency index i in [0, D/2):
 *
 *   theta_i   = base^(-2i/D)
 *   y_i       = x_i cos(p theta_i) - x_{i+D/2} sin(p theta_i)
 *   y_{i+D/2} = x_{i+D/2} cos(p theta_i) + x_i sin(p theta_i)
 *
 * i.e. the complex number x_i + j x_{i+D/2} multiplied by e^{j p theta_i}. */

static double rope_theta(int32_t i, int32_t head_dim, double base)
{
#if ORACLE_MUTANT == 13
    return pow(base, -(double)i / head_dim);                   /* exponent halved */
#else
    return pow(base, -2.0 * i / head_dim);
#endif
}

/* The cos/sin cache: row p holds cos(p theta_i) for i in [0, D/2) followed by
 * sin(p theta_i), each computed in double and rounded once to float. */
int oracle_rope_table(float* table, int32_t max_position, int32_t head_dim, double base)
{
    if (!table || max_position <= 0 || head_dim <= 0 || head_dim % 2 || !(base > 1.0)) return -1;
    const int32_t half = head_dim / 2;
    for (int32_t p = 0; p < max_position; ++p)
        for (int32_t i = 0; i < half; ++i) {
            double a = (double)p * rope_theta(i, head_dim, base);
            table[(int64_t)p * head_dim + i] = (float)cos(a);
#if ORACLE_MUTANT == 12
            table[(int64_t)p * head_dim + half + i] = (float)-sin(a);   /* rotation by -angle */
#else
            table[(int64_t)p * head_dim + half + i] = (float)sin(a);
#endif
        }
    return 0;
}

/* Rotate one head row x (head_dim bf16) to position row cs of the table;
 * the products and sums in double, each output rounded once to bf16. */
static void rope_row(uint16_t* y, double* y64, const uint16_t* x, const float* cs, int32_t head_dim)
{
    const int32_t half = head_dim / 2;
    for (int32_t i = 0; i < half; ++i) {
#if ORACLE_MUTANT == 11
        int32_t lo = 2 * i, hi = 2 * i + 1;                    /* adjacent pairs */
#else
        int32_t lo = i, hi = i + half;
#endif
        double c = cs[i], s = cs[half + i];
        double a = bf16_to_double(x[lo]), b = bf16_to_double(x[hi]);
        double ylo = a * c - b * s, yhi = b * c + a * s;
        y[lo] = double_to_bf16(ylo);
        y[hi] = double_to_bf16(yhi);
        if (y64) { y64[lo] = ylo; y64[hi] = yhi; }
    }
}

/* Rotary embedding fused with store_kvcache: for every token t at position
 * positions[t], rotate its num_heads query rows into q_out ([num_tokens,
 * num_heads, head_dim], dense) and its num_kv_heads key rows; then, if
 * slot_mapping[t] != -1, store the rotated key rows and the unchanged value
 * rows exactly as oracle_store_kvcache does. */
int oracle_rope_store_kvcache(uint16_t* q_out, double* q_out_f64, const uint16_t* q, int64_t q_row_stride,
                              const uint16_t* key, const uint16_t* value, int64_t key_row_stride,
                              int64_t value_row_stride, const int32_t* positions, const float* table,
                              int32_t max_position, uint16_t* k_cache, uint16_t* v_cache,
                              const int32_t* slot_mapping, int32_t num_tokens, int32_t num_heads,
                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks)
{
    if (num_tokens < 0 || num_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || head_dim % 2 || block_size <= 0 ||
        num_blocks < 0 || max_position <= 0)
        return -1;
    if (num_tokens == 0) return 0;
    if (!q_out || !q || !key || !value || !positions || !table || !k_cache || !v_cache || !slot_mapping) return -1;
    const int64_t qrow = (int64_t)num_heads * head_dim, kvrow = (int64_t)num_kv_heads * head_dim;
    if (q_row_stride < qrow || key_row_stride < kvrow || value_row_stride < kvrow) return -1;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int32_t p = positions[t];
        if (p < 0 || p >= max_position) return -2;
    }
    uint16_t* krot = (uint16_t*)malloc((size_t)kvrow * sizeof(uint16_t));
    if (!krot) return -1;
    for (int32_t t = 0; t < num_tokens; ++t) {
#if ORACLE_MUTANT == 15
        const float* cs = table + (int64_t)(positions[t] + 1 < max_position ? positions[t] + 1 : positions[t]) * head_dim;
#else
        const float* cs = table + (int64_t)positions[t] * head_dim;
#endif
        for (int32_t h = 0; h < num_heads; ++h) {
            int64_t o = ((int64_t)t * num_heads + h) * head_dim;
            rope_row(q_out + o, q_out_f64 ? q_out_f64 + o : NULL, q + (int64_t)t * q_row_stride + (int64_t)h * head_dim,
                     cs, head_dim);
        }
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            const uint16_t* kx = key + (int64_t)t * key_row_stride + (int64_t)h * head_dim;
#if ORACLE_MUTANT == 14
            memcpy(krot + (int64_t)h * head_dim, kx, (size_t)head_dim * sizeof(uint16_t));   /* key not rotated */
#else
            rope_row(krot + (int64_t)h * head_dim, NULL, kx, cs, head_dim);
#endif
        }
        int rc = oracle_store_kvcache(krot, value + (int64_t)t * value_row_stride, kvrow, value_row_stride, k_cache,
                                      v_cache, slot_mapping + t, 1, num_kv_heads, head_dim, block_size, num_blocks);
        if (rc) {
            free(krot);
            return rc;
        }
    }
    free(krot);
    return 0;
}

int oracle_mutant_id(void) { return ORACLE_MUTANT; }

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
