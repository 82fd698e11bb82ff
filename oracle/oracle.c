/*
 * oracle.c -- plain, slow, fp64 CPU oracle for paged decode attention and the
 * slot-mapped KV-cache append.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU baseline
 * do.  It shares no code, header or constant with the CUDA library.
 *
 * What it computes (restated from the pages on PagedAttention):
 *   - "vLLM Fundamentals: Paged Attention and Batching", section "Paged
 *     Attention": the KV cache is split into blocks that are not contiguous;
 *     each sequence has a block table, and the paged kernel follows that table
 *     to gather the blocks.  Paging changes where keys and values live, not
 *     what attention computes.
 *   - "Deep Dive into vLLM", section 2.1: logical block -> physical block
 *     through the block table.
 *   - runbyai.xyz post 449 (an essay on vLLM and PagedAttention), section 1,
 *     Decoding: each decode step uses the keys and values of all previous
 *     tokens.
 * So the oracle is the plain definition of single-query softmax attention,
 * evaluated by walking the block table token by token in logical order:
 *
 *   for sequence s, query head j, kv head h = floor(j / (Hq / Hkv)):
 *     k_t = K[table[s][t / bs]][t % bs][h][:]   (likewise v_t), t = 0 .. L_s-1
 *     x_t = scale * sum_d q[s][j][d] * k_t[d]
 *     mu  = max_t x_t,  w_t = exp(x_t - mu)
 *     out[s][j][:] = sum_t w_t v_t / sum_t w_t         (0 when L_s == 0)
 *
 * All arithmetic is fp64; bf16 inputs are widened exactly.  The pages give no
 * formula, scale, head grouping or layout: the readings used here are the
 * plain softmax(scale * q K^T) V, q head j served by kv head floor(j / G), and
 * the pool layout [num_blocks][block_size][num_kv_heads][head_dim].
 *
 * The append follows the same pages: each decode step computes and caches the
 * new token's key and value (runbyai.xyz post 449, sections 1 and 2).
 * Token i goes to slot slot_mapping[i] = physical_block * bs + offset; a
 * negative slot means "no write".
 *
 * Chunked prefill / mixed batches ("vLLM Fundamentals", section "Continuous
 * Batching": long prefills are cut into chunks under a per-step token budget
 * and mixed with decodes; each request processes some number of tokens per
 * step): sequence s brings n_s query tokens, the last n_s of its L_s cached
 * tokens. Query i (position p = L_s - n_s + i) attends, causally, to the
 * cache positions 0 .. p -- the same plain definition over a shorter
 * context. n_s = 1 is the decode step.
 *
 * FP8 cache (runbyai post 449, section 5, names quantization among the means
 * for long contexts; the format is the task's reading): pools of e4m3 codes
 * (1 sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 15 with
 * mantissa 7 is NaN; exponent 0 is subnormal, m * 2^-9) and one fp32 scale
 * per kv head for K and one for V. A stored code c of head h stands for
 * e4m3(c) * scale[h]. The append quantizes x (bf16) as the e4m3 value nearest
 * to the fp32 quotient x / scale[h] (ties to an even mantissa), saturating at
 * +-448, the largest finite e4m3 value. The decode dequantizes exactly in
 * fp64 and is otherwise the plain definition above.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* bf16 bit pattern -> double, exactly (bf16 is the top half of an fp32). */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* e4m3 code -> its value, from the format's definition. */
double oracle_e4m3_to_double(uint8_t c)
{
    int e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
    double v = e == 0 ? ldexp((double)m, -9) : ldexp((double)(8 + m), e - 10); /* (1 + m/8) 2^(e-7) */
    return (c & 0x80) ? -v : v;
}

/* fp32 -> nearest e4m3 code, ties to an even mantissa, saturating at +-448. */
uint8_t oracle_e4m3_from_float(float xf)
{
    if (isnan(xf))
        return 0x7f;
    uint8_t sign = signbit(xf) ? 0x80 : 0;
    double a = fabs((double)xf);
    if (a >= 448.0)
        return sign | 0x7e;
    if (a < ldexp(1.0, -6)) {                  /* subnormal range: multiples of 2^-9 */
        double m = nearbyint(a * 512.0);       /* 8 is the smallest normal, code 0x08 */
        return sign | (uint8_t)m;
    }
    int e;
    frexp(a, &e);                              /* a = f 2^e, f in [0.5, 1) */
    int E = e - 1;                             /* a = 2^E (1 + mantissa) */
    double m = nearbyint((a / ldexp(1.0, E) - 1.0) * 8.0);
    if (m == 8.0) {
        m = 0.0;
        E += 1;
    }
    return sign | (uint8_t)((E + 7) << 3) | (uint8_t)m;
}

/* A KV pool as the decode reads it: bf16 values, or e4m3 codes with a scale per kv head. */
typedef struct {
    const uint16_t *bf16;
    const uint8_t *fp8;
    const float *scale;
} Pool;

static double pool_value(const Pool *P, int64_t elem, int h)
{
    if (P->bf16)
        return bf16_bits_to_double(P->bf16[elem]);
    return oracle_e4m3_to_double(P->fp8[elem]) * (double)P->scale[h];
}

/* Element offset of (physical block p, offset off, kv head h, dim 0) in the pool. */
static int64_t pool_row(int64_t p, int off, int h, int block_size, int num_kv_heads, int head_dim)
{
    return ((p * block_size + off) * num_kv_heads + h) * (int64_t)head_dim;
}

/*
 * One output row: out[0..head_dim) for sequence s, query head j.
 * x is scratch of at least context_len doubles.
 * Returns 0, or -2 when a table entry it needs is outside [0, num_blocks).
 */
static int decode_one(double *out, double *x,
                      const uint16_t *qrow, const Pool *K, const Pool *V,
                      const int32_t *block_tables, int context_len,
                      int s, int j, int num_q_heads, int num_kv_heads, int head_dim,
                      int block_size, int max_blocks_per_seq, int64_t num_blocks, double scale)
{
    const int group = num_q_heads / num_kv_heads;
    const int h = j / group;
    const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;

    for (int d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (context_len == 0)
        return 0;

    /* logits, walking the block table in logical token order */
    for (int t = 0; t < context_len; ++t) {
        int64_t p = table[t / block_size];
        if (p < 0 || p >= num_blocks)
            return -2;
        int64_t krow = pool_row(p, t % block_size, h, block_size, num_kv_heads, head_dim);
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += bf16_bits_to_double(qrow[d]) * pool_value(K, krow + d, h);
        x[t] = scale * dot;
    }

    double mu = x[0];
    for (int t = 1; t < context_len; ++t)
        if (x[t] > mu)
            mu = x[t];

    double z = 0.0;
    for (int t = 0; t < context_len; ++t) {
        double w = exp(x[t] - mu);
        int64_t p = table[t / block_size];
        int64_t vrow = pool_row(p, t % block_size, h, block_size, num_kv_heads, head_dim);
        for (int d = 0; d < head_dim; ++d)
            out[d] += w * pool_value(V, vrow + d, h);
        z += w;
    }
    for (int d = 0; d < head_dim; ++d)
        out[d] /= z;
    return 0;
}

/*
 * Paged decode attention, fp64.
 *
 * out           [num_pairs][head_dim] doubles; row k is the output of pair k.
 * q             bf16 bits [num_seqs][num_q_heads][head_dim]
 * k_cache/v_cache bf16 bits [num_blocks][block_size][num_kv_heads][head_dim]
 * block_tables  [num_seqs][max_blocks_per_seq]
 * context_lens  [num_seqs]
 * pairs         flat indices s * num_q_heads + j of the rows wanted, or NULL
 *               for all rows in order (num_pairs must then be num_seqs * num_q_heads)
 * num_threads   OpenMP threads (<= 0: the runtime's default)
 *
 * Returns 0; -1 for a bad argument; -2 for a table entry outside the pool;
 * -3 for a context length outside [0, max_blocks_per_seq * block_size].
 */
static int decode_pool(double *out, const uint16_t *q, const Pool *K, const Pool *V,
                       const int32_t *block_tables, const int32_t *context_lens,
                       int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                       int max_blocks_per_seq, int64_t num_blocks, double scale,
                       const int64_t *pairs, int64_t num_pairs, int num_threads)
{
    if (!out || !q || !block_tables || !context_lens)
        return -1;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 ||
        max_blocks_per_seq < 0 || num_blocks < 0 || num_q_heads % num_kv_heads != 0)
        return -1;
    if (!pairs && num_pairs != (int64_t)num_seqs * num_q_heads)
        return -1;

    int max_len = 0;
    for (int s = 0; s < num_seqs; ++s) {
        if (context_lens[s] < 0 || (int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * block_size)
            return -3;
        if (context_lens[s] > max_len)
            max_len = context_lens[s];
    }
    for (int64_t k = 0; pairs && k < num_pairs; ++k)
        if (pairs[k] < 0 || pairs[k] >= (int64_t)num_seqs * num_q_heads)
            return -1;

    int status = 0;
#ifdef _OPENMP
    if (num_threads <= 0)
        num_threads = omp_get_max_threads();
#pragma omp parallel num_threads(num_threads)
#endif
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        int mine = x ? 0 : -1;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
        for (int64_t k = 0; k < num_pairs; ++k) {
            int64_t flat = pairs ? pairs[k] : k;
            int s = (int)(flat / num_q_heads);
            int j = (int)(flat % num_q_heads);
            if (mine == 0)
                mine = decode_one(out + k * head_dim, x, q + ((int64_t)s * num_q_heads + j) * head_dim, K, V,
                                  block_tables,
                                  context_lens[s], s, j, num_q_heads, num_kv_heads, head_dim,
                                  block_size, max_blocks_per_seq, num_blocks, scale);
        }
        free(x);
#ifdef _OPENMP
#pragma omp critical
#endif
        if (mine != 0 && status == 0)
            status = mine;
    }
    return status;
}

int oracle_paged_decode(double *out, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                        const int32_t *block_tables, const int32_t *context_lens,
                        int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                        int max_blocks_per_seq, int64_t num_blocks, double scale,
                        const int64_t *pairs, int64_t num_pairs, int num_threads)
{
    if (!k_cache || !v_cache)
        return -1;
    Pool K = {k_cache, NULL, NULL}, V = {v_cache, NULL, NULL};
    return decode_pool(out, q, &K, &V, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
                       head_dim, block_size, max_blocks_per_seq, num_blocks, scale, pairs, num_pairs,
                       num_threads);
}

/*
 * The same over an e4m3 cache: k_cache / v_cache hold codes
 * [num_blocks][block_size][num_kv_heads][head_dim], k_scale / v_scale one fp32
 * per kv head; element e of head h stands for e4m3(code) * scale[h].
 */
int oracle_paged_decode_fp8(double *out, const uint16_t *q, const uint8_t *k_cache, const uint8_t *v_cache,
                            const float *k_scale, const float *v_scale,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                            int max_blocks_per_seq, int64_t num_blocks, double scale,
                            const int64_t *pairs, int64_t num_pairs, int num_threads)
{
    if (!k_cache || !v_cache || !k_scale || !v_scale)
        return -1;
    Pool K = {NULL, k_cache, k_scale}, V = {NULL, v_cache, v_scale};
    return decode_pool(out, q, &K, &V, block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
                       head_dim, block_size, max_blocks_per_seq, num_blocks, scale, pairs, num_pairs,
                       num_threads);
}

/*
 * Slot-mapped append: for every token i with slot_mapping[i] >= 0, copy
 * k[i][h][:] and v[i][h][:] into block slot / bs, offset slot % bs, for every
 * kv head h.  Later tokens win when two share a slot.
 *
 * Returns 0; -1 for a bad argument; -2 when a slot is at or past
 * num_blocks * block_size (nothing is written in that case).
 */
int oracle_kv_append(uint16_t *k_cache, uint16_t *v_cache, const uint16_t *k, const uint16_t *v,
                     const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads, int head_dim,
                     int block_size, int64_t num_blocks)
{
    if (!k_cache || !v_cache || !k || !v || (!slot_mapping && num_tokens > 0))
        return -1;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return -1;
    for (int64_t i = 0; i < num_tokens; ++i)
        if (slot_mapping[i] >= num_blocks * block_size)
            return -2;

    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t p = slot / block_size;
        int off = (int)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t dst = pool_row(p, off, h, block_size, num_kv_heads, head_dim);
            int64_t src = (i * num_kv_heads + h) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                k_cache[dst + d] = k[src + d];
                v_cache[dst + d] = v[src + d];
            }
        }
    }
    return 0;
}

/*
 * The append into an e4m3 cache: element d of token i, kv head h becomes the
 * code of (float) k[i][h][d] / k_scale[h] (and likewise for v), computed as one
 * fp32 division and then oracle_e4m3_from_float.  Same slots and returns as
 * oracle_kv_append.
 */
int oracle_kv_append_fp8(uint8_t *k_cache, uint8_t *v_cache, const uint16_t *k, const uint16_t *v,
                         const float *k_scale, const float *v_scale, const int64_t *slot_mapping,
                         int64_t num_tokens, int num_kv_heads, int head_dim, int block_size, int64_t num_blocks)
{
    if (!k_cache || !v_cache || !k || !v || !k_scale || !v_scale || (!slot_mapping && num_tokens > 0))
        return -1;
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks < 0)
        return -1;
    for (int64_t i = 0; i < num_tokens; ++i)
        if (slot_mapping[i] >= num_blocks * block_size)
            return -2;

    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        int64_t p = slot / block_size;
        int off = (int)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            int64_t dst = pool_row(p, off, h, block_size, num_kv_heads, head_dim);
            int64_t src = (i * num_kv_heads + h) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                float kq = (float)bf16_bits_to_double(k[src + d]) / k_scale[h];
                float vq = (float)bf16_bits_to_double(v[src + d]) / v_scale[h];
                k_cache[dst + d] = oracle_e4m3_from_float(kq);
                v_cache[dst + d] = oracle_e4m3_from_float(vq);
            }
        }
    }
    return 0;
}

/*
 * Multi-query paged attention (chunked prefill, mixed batches), fp64.
 *
 * out           [num_tokens][num_q_heads][head_dim] doubles
 * q             bf16 bits [num_tokens][num_q_heads][head_dim]; the queries of
 *               sequence s are rows query_start[s] .. query_start[s + 1] - 1
 * query_start   [num_seqs + 1], non-decreasing, query_start[0] = 0,
 *               query_start[num_seqs] = num_tokens; n_s = query_start[s+1] -
 *               query_start[s] <= context_lens[s]
 * the rest as oracle_paged_decode.  Query i of sequence s sits at position
 * p = context_lens[s] - n_s + i and attends to positions 0 .. p.
 *
 * Returns 0; -1 for a bad argument; -2 for a table entry outside the pool;
 * -3 for a context length outside [0, max_blocks_per_seq * block_size].
 */
int oracle_paged_prefill(double *out, const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                         const int32_t *block_tables, const int32_t *context_lens, const int32_t *query_start,
                         int num_seqs, int64_t num_tokens, int num_q_heads, int num_kv_heads, int head_dim,
                         int block_size, int max_blocks_per_seq, int64_t num_blocks, double scale, int num_threads)
{
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
        return -1;
    if (num_seqs < 0 || num_tokens < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || max_blocks_per_seq < 0 || num_blocks < 0 || num_q_heads % num_kv_heads != 0)
        return -1;
    if (query_start[0] != 0 || query_start[num_seqs] != num_tokens)
        return -1;
    int max_len = 0;
    for (int s = 0; s < num_seqs; ++s) {
        int64_t n = (int64_t)query_start[s + 1] - query_start[s];
        if (n < 0)
            return -1;
        if (context_lens[s] < 0 || (int64_t)context_lens[s] > (int64_t)max_blocks_per_seq * block_size)
            return -3;
        if (n > context_lens[s])
            return -1;
        if (context_lens[s] > max_len)
            max_len = context_lens[s];
    }
    Pool K = {k_cache, NULL, NULL}, V = {v_cache, NULL, NULL};
    int status = 0;
#ifdef _OPENMP
    if (num_threads <= 0)
        num_threads = omp_get_max_threads();
#pragma omp parallel num_threads(num_threads)
#endif
    {
        double *x = (double *)malloc(sizeof(double) * (size_t)(max_len > 0 ? max_len : 1));
        int mine = x ? 0 : -1;
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1) collapse(2)
#endif
        for (int s = 0; s < num_seqs; ++s) {
            for (int j = 0; j < num_q_heads; ++j) {
                int n = query_start[s + 1] - query_start[s];
                for (int i = 0; i < n && mine == 0; ++i) {
                    int64_t row = (int64_t)query_start[s] + i;
                    int p = context_lens[s] - n + i;           /* this query's position */
                    /* decode of this one query over the context 0 .. p of sequence s */
                    mine = decode_one(out + (row * num_q_heads + j) * head_dim, x,
                                      q + (row * num_q_heads + j) * (int64_t)head_dim, &K, &V, block_tables,
                                      p + 1, s, j, num_q_heads, num_kv_heads, head_dim, block_size,
                                      max_blocks_per_seq, num_blocks, scale);
                }
            }
        }
        free(x);
#ifdef _OPENMP
#pragma omp critical
#endif
        if (mine != 0 && status == 0)
            status = mine;
    }
    return status;
}
