/*
 * Paged KV-cache oracle: plain, slow, obviously correct fp64 CPU code.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg load this file's library.  The product path
 * (the CUDA library) never calls it, and it includes nothing from the
 * product: no header, table or helper is shared.
 *
 * What it follows:
 *  - "Inside vLLM: How PagedAttention Changes Python LLM Inference at the
 *    Systems Level", section "PagedAttention: What the OS Figured Out Decades
 *    Ago": the KV cache is cut into fixed-size blocks (16 tokens by default);
 *    a per-sequence block table maps logical block i to a physical block; the
 *    physical blocks need not be adjacent, yet attention sees the sequence as
 *    if it were contiguous.  So decode attention over a paged cache is plain
 *    scaled dot-product attention over the tokens gathered in logical order.
 *  - same page, section "Copy-on-Write Makes Beam Search Cheap": branches
 *    share prompt blocks by reference count, and a write into a shared block
 *    first copies that one block.
 *  - "vLLM PagedAttention: reducing KV cache memory waste", section "How
 *    PagedAttention Works": blocks are claimed as tokens arrive; only a
 *    sequence's last block can be partly filled.
 *  - "PagedAttention in vLLM: a throughput settings guide", section "Tuning
 *    Batching, Prefill, and Cache": with chunked prefill a step fills its
 *    token budget with chunks of prompts; a chunk's tokens attend to the
 *    cached tokens before them and causally to each other.
 *
 * Cache layout (a reading; the pages fix none): key_cache and value_cache are
 * each [num_blocks][num_kv_heads][block_size][head_dim] of 16-bit elements,
 * head_dim contiguous.  Element (block b, head h, row o, column i) sits at
 * ((b * num_kv_heads + h) * block_size + o) * head_dim + i.
 *
 * Storage types: dtype 0 = IEEE binary16 (fp16), dtype 1 = bfloat16.  Values
 * are widened to double exactly and all arithmetic is in double.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* IEEE 754 binary16: sign bit, 5 exponent bits with bias 15, 10 fraction
 * bits.  Exponent field 0 is a subnormal (fraction * 2^-24); 31 is inf/NaN. */
double oracle_f16_to_f64(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -24);
    else if (e == 31)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(f | 0x400), e - 25);
    return sign ? -mag : mag;
}

/* bfloat16: sign bit, 8 exponent bits with bias 127, 7 fraction bits (the top
 * half of an IEEE binary32).  Exponent 0 is subnormal (fraction * 2^-133). */
double oracle_bf16_to_f64(uint16_t b) {
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -133);
    else if (e == 255)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(f | 0x80), e - 134);
    return sign ? -mag : mag;
}

static double widen(uint16_t bits, int dtype) {
    return dtype == 0 ? oracle_f16_to_f64(bits) : oracle_bf16_to_f64(bits);
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Write each new token's K and V into its slot.  Slot s names physical block
 * s / block_size, row s % block_size (the logical-to-physical step of the
 * block table, resolved by the caller).  A negative slot is padding and is
 * skipped.  Bit copy: the cache holds exactly the input bits afterwards.
 * k, v: [num_tokens][num_kv_heads][head_dim].  Returns the number of slots
 * that were out of range (and skipped). */
int64_t oracle_reshape_and_cache(const uint16_t *k, const uint16_t *v, uint16_t *key_cache,
                                 uint16_t *value_cache, const int64_t *slot_mapping,
                                 int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int64_t num_blocks) {
    int64_t bad = 0;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_blocks * (int64_t)block_size) {
            ++bad;
            continue;
        }
        int64_t b = slot / block_size;
        int64_t o = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t dst = ((b * num_kv_heads + h) * block_size + o) * head_dim;
            int64_t src = ((int64_t)t * num_kv_heads + h) * head_dim;
            for (int32_t i = 0; i < head_dim; ++i) {
                key_cache[dst + i] = k[src + i];
                value_cache[dst + i] = v[src + i];
            }
        }
    }
    return bad;
}

/* Copy-on-write block copy: for each (src, dst) pair, the whole physical
 * block dst (every head, every row, K and V) becomes a copy of block src.
 * pairs: [num_pairs][2].  Returns the number of pairs skipped for an id out
 * of range. */
int64_t oracle_copy_blocks(uint16_t *key_cache, uint16_t *value_cache, const int32_t *pairs,
                           int32_t num_pairs, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int64_t num_blocks) {
    int64_t bad = 0;
    int64_t per_block = (int64_t)num_kv_heads * block_size * head_dim;
    for (int32_t p = 0; p < num_pairs; ++p) {
        int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) {
            ++bad;
            continue;
        }
        for (int64_t e = 0; e < per_block; ++e) {
            key_cache[dst * per_block + e] = key_cache[src * per_block + e];
            value_cache[dst * per_block + e] = value_cache[src * per_block + e];
        }
    }
    return bad;
}

/* Gather tokens [t0, t1) of sequence s, kv head kvh, into contiguous double
 * rows K[j - t0][i], V[j - t0][i], following the block table. */
static void gather(double *K, double *V, const uint16_t *key_cache, const uint16_t *value_cache,
                   const int32_t *table_row, int32_t t0, int32_t t1, int32_t kvh,
                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int dtype) {
    for (int32_t j = t0; j < t1; ++j) {
        int64_t b = table_row[j / block_size];
        int64_t o = j % block_size;
        int64_t base = ((b * num_kv_heads + kvh) * block_size + o) * head_dim;
        for (int32_t i = 0; i < head_dim; ++i) {
            K[(int64_t)(j - t0) * head_dim + i] = widen(key_cache[base + i], dtype);
            V[(int64_t)(j - t0) * head_dim + i] = widen(value_cache[base + i], dtype);
        }
    }
}

/* Scaled dot-product attention of one query row over n contiguous rows:
 * x_j = scale * q . K_j;  w_j = exp(x_j - max x);  o = sum_j w_j V_j / sum_j w_j.
 * Writes o (normalised) and returns log(sum_j exp(x_j)) = max + log(sum w).
 * n == 0 gives o = 0 and -inf. */
static double attend(double *o, const double *q, const double *K, const double *V, int32_t n,
                     int32_t head_dim, double scale) {
    for (int32_t i = 0; i < head_dim; ++i)
        o[i] = 0.0;
    if (n <= 0)
        return -INFINITY;
    double *x = (double *)malloc(sizeof(double) * (size_t)n);
    double m = -INFINITY;
    for (int32_t j = 0; j < n; ++j) {
        double dot = 0.0;
        for (int32_t i = 0; i < head_dim; ++i)
            dot += q[i] * K[(int64_t)j * head_dim + i];
        x[j] = scale * dot;
        if (x[j] > m)
            m = x[j];
    }
    double den = 0.0;
    for (int32_t j = 0; j < n; ++j) {
        double w = exp(x[j] - m);
        den += w;
        for (int32_t i = 0; i < head_dim; ++i)
            o[i] += w * V[(int64_t)j * head_dim + i];
    }
    for (int32_t i = 0; i < head_dim; ++i)
        o[i] /= den;
    free(x);
    return m + log(den);
}

/* Decode attention over the paged cache for tokens [t0, t1) of each
 * sequence (clipped to [0, context_len)); t1 < 0 means "to the end".
 * For sequence s and query head h the kv head is h / (num_q_heads /
 * num_kv_heads): consecutive query heads share one kv head.
 * q: [num_seqs][num_q_heads][head_dim] bits; block_tables:
 * [num_seqs][max_blocks_per_seq]; out: [num_sel][num_q_heads][head_dim]
 * doubles; lse (optional): [num_sel][num_q_heads].  seq_sel (optional)
 * lists which sequences to compute, in output order. */
void oracle_decode_range(double *out, double *lse, const uint16_t *q, const uint16_t *key_cache,
                         const uint16_t *value_cache, const int32_t *block_tables,
                         int32_t max_blocks_per_seq, const int32_t *context_lens,
                         int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                         int32_t head_dim, int32_t block_size, double scale, int32_t dtype,
                         const int32_t *seq_sel, int32_t num_sel, int32_t t0, int32_t t1) {
    int32_t group = num_q_heads / num_kv_heads;
    int32_t ns = seq_sel ? num_sel : num_seqs;
    int64_t jobs = (int64_t)ns * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t job = 0; job < jobs; ++job) {
        int32_t si = (int32_t)(job / num_q_heads);
        int32_t h = (int32_t)(job % num_q_heads);
        int32_t s = seq_sel ? seq_sel[si] : si;
        int32_t kvh = h / group;
        int32_t L = context_lens[s];
        int32_t a = t0 < 0 ? 0 : t0;
        int32_t b = (t1 < 0 || t1 > L) ? L : t1;
        int32_t n = b > a ? b - a : 0;
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        double *K = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(n ? n : 1));
        double *V = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(n ? n : 1));
        for (int32_t i = 0; i < head_dim; ++i)
            qd[i] = widen(q[((int64_t)s * num_q_heads + h) * head_dim + i], dtype);
        gather(K, V, key_cache, value_cache, block_tables + (int64_t)s * max_blocks_per_seq, a,
               a + n, kvh, num_kv_heads, head_dim, block_size, dtype);
        double r = attend(out + job * head_dim, qd, K, V, n, head_dim, scale);
        if (lse)
            lse[job] = r;
        free(qd);
        free(K);
        free(V);
    }
}

/* Chunked prefill over the paged cache.  Sequence s owns query rows
 * query_start[s] .. query_start[s + 1] - 1 of q ([num_q_tokens][num_q_heads]
 * [head_dim]); they are the last n_s = query_start[s + 1] - query_start[s]
 * tokens of its context of L = context_lens[s] tokens, whose K/V are already
 * in the cache.  Query row i of s sits at position p = L - n_s + i and
 * attends to tokens 0 .. p (causal): out row = softmax(scale q K^T) V over
 * those tokens, in double. */
void oracle_prefill(double *out, const uint16_t *q, const uint16_t *key_cache,
                    const uint16_t *value_cache, const int32_t *block_tables,
                    int32_t max_blocks_per_seq, const int32_t *context_lens,
                    const int32_t *query_start, int32_t num_seqs, int32_t num_q_heads,
                    int32_t num_kv_heads, int32_t head_dim, int32_t block_size, double scale,
                    int32_t dtype) {
    int32_t group = num_q_heads / num_kv_heads;
    int64_t rows = (int64_t)query_start[num_seqs] * num_q_heads;
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t job = 0; job < rows; ++job) {
        int32_t t = (int32_t)(job / num_q_heads);
        int32_t h = (int32_t)(job % num_q_heads);
        int32_t s = 0;
        while (query_start[s + 1] <= t) ++s;
        int32_t n_s = query_start[s + 1] - query_start[s];
        int32_t pos = context_lens[s] - n_s + (t - query_start[s]);
        int32_t n = pos + 1 > 0 ? pos + 1 : 0;
        double *qd = (double *)malloc(sizeof(double) * (size_t)head_dim);
        double *K = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(n ? n : 1));
        double *V = (double *)malloc(sizeof(double) * (size_t)head_dim * (size_t)(n ? n : 1));
        for (int32_t i = 0; i < head_dim; ++i)
            qd[i] = widen(q[((int64_t)t * num_q_heads + h) * head_dim + i], dtype);
        gather(K, V, key_cache, value_cache, block_tables + (int64_t)s * max_blocks_per_seq, 0, n,
               h / group, num_kv_heads, head_dim, block_size, dtype);
        attend(out + job * head_dim, qd, K, V, n, head_dim, scale);
        free(qd);
        free(K);
        free(V);
    }
}

/* Whole-context decode: oracle_decode_range over [0, context_len). */
void oracle_decode(double *out, const uint16_t *q, const uint16_t *key_cache,
                   const uint16_t *value_cache, const int32_t *block_tables,
                   int32_t max_blocks_per_seq, const int32_t *context_lens, int32_t num_seqs,
                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                   int32_t block_size, double scale, int32_t dtype, const int32_t *seq_sel,
                   int32_t num_sel) {
    oracle_decode_range(out, NULL, q, key_cache, value_cache, block_tables, max_blocks_per_seq,
                        context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                        scale, dtype, seq_sel, num_sel, 0, -1);
}

/* Merge attention results computed over disjoint token ranges of the same
 * row.  Range p gave the normalised output o_p and lse_p = log sum_j exp(x_j)
 * over its tokens; softmax over the union weighs range p by exp(lse_p), so
 * out = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M), M = max_p lse_p.
 * o_parts: [rows][P][head_dim]; lse_parts: [rows][P]; out: [rows][head_dim].
 * A row whose ranges are all empty (every lse -inf) gives 0. */
void oracle_lse_merge(double *out, const double *o_parts, const double *lse_parts, int64_t rows,
                      int32_t num_parts, int32_t head_dim) {
    for (int64_t r = 0; r < rows; ++r) {
        double M = -INFINITY;
        for (int32_t p = 0; p < num_parts; ++p)
            if (lse_parts[r * num_parts + p] > M)
                M = lse_parts[r * num_parts + p];
        for (int32_t i = 0; i < head_dim; ++i)
            out[r * head_dim + i] = 0.0;
        if (M == -INFINITY)
            continue;
        double den = 0.0;
        for (int32_t p = 0; p < num_parts; ++p) {
            double w = exp(lse_parts[r * num_parts + p] - M);
            den += w;
            for (int32_t i = 0; i < head_dim; ++i)
                out[r * head_dim + i] += w * o_parts[(r * num_parts + p) * head_dim + i];
        }
        for (int32_t i = 0; i < head_dim; ++i)
            out[r * head_dim + i] /= den;
    }
}
