/*
 * pa_oracle.c -- plain, slow, fp64 CPU reference for paged-KV-cache attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may link, load or call
 * this file; only the tests, the graft smoke check and the CPU-baseline leg of the
 * benchmark use it.  It shares no code, header, table or helper with the CUDA
 * library: it is written straight from the definitions on the source pages.
 *
 * Sources (page title, section):
 *   [P1] "vLLM 深度拆解：当大模型推理学会「分页注意力」" -- 1.1 (KV cache: K,V of
 *        every past token kept and attended to), 2.1 (fixed 16-token blocks, block
 *        table maps logical block -> physical block, possibly non-contiguous),
 *        3.1 (each step: generate a token and write it back into the KV cache).
 *   [P3] the devpress.csdn.net/amd teardown of vLLM v0.6.x (untitled in the
 *        extracted text; it opens "你跑过一个 70B 模型吗？") -- section
 *        "核心代码拆解" (the simplified kernel: layouts
 *        key/value_cache[num_blocks, num_heads, block_size, head_size],
 *        query/output[num_tokens, num_heads, head_size], block_table
 *        [num_requests, max_num_blocks], context_lens[num_requests]; physical
 *        block looked up through the table; score scaled by `scale`; softmax and
 *        a V-weighted sum "as in standard attention"), section "关键设计二"
 *        (Copy-on-Write copies a whole block from the shared one to a new one).
 *   [P1] 5.3 and the [P3] architecture figure -- an FP8 KV cache; the e4m3
 *        reading and its scale convention are stated above e4m3_value() below.
 *
 * Arithmetic: every element is widened exactly to double (bf16 is the upper half
 * of an IEEE binary32, so widening is exact) and all sums, the max, exp and the
 * division are done in double.  There is no blocking, no online softmax, no
 * split of the context: each sequence's blocks are gathered into a contiguous
 * [L, head_dim] array and textbook softmax attention is run over it.
 *
 * Parallelism: an OpenMP loop over independent (sequence, query head) outputs.
 * Each output is computed by exactly one thread with the same serial arithmetic,
 * so results do not depend on the thread count.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_FP8 2   /* e4m3 code; widen() gives its value, unscaled */

/*
 * FP8 KV cache.  The pages name FP8 without a format (chenxutan 5.3: FP8 is nearly
 * lossless and cuts memory and bandwidth; the devpress teardown's architecture
 * figure lists FP8/INT8 quantisation in the kernel layer).  Reading taken: the
 * E4M3 format of the OCP 8-bit floating point specification with one scale per
 * tensor -- sign, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 holds
 * the subnormals m * 2^-9; no infinities; S.1111.111 is NaN, so the largest
 * finite value is S.1111.110 = 448.
 */
static double e4m3_value(uint8_t c)
{
    const int sgn = c >> 7, e = (c >> 3) & 15, m = c & 7;
    if (e == 15 && m == 7)
        return NAN;
    const double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return sgn ? -v : v;
}

/* Nearest e4m3 code to x, ties to even mantissa, magnitudes beyond the largest
 * finite value (and infinities) saturated to +-448, NaN to 0x7F. */
static uint8_t e4m3_encode(float x)
{
    if (isnan(x))
        return 0x7F;
    const uint8_t sgn = signbit(x) ? 0x80 : 0x00;
    const double a = fabs((double)x);
    if (a >= 448.0)
        return sgn | 0x7E;
    if (a < ldexp(1.0, -6)) {                 /* subnormal range: a multiple of 2^-9 */
        const double m = nearbyint(a * 512.0); /* round to nearest, ties to even; 8 -> 2^-6 */
        return sgn | (uint8_t)m;
    }
    int e2;
    const double f = frexp(a, &e2);            /* a = f * 2^e2, f in [0.5, 1) */
    int ex = e2 - 1;                           /* a = (1 + frac) * 2^ex */
    double mq = nearbyint((2.0 * f - 1.0) * 8.0);
    if (mq == 8.0) {
        ex += 1;
        mq = 0.0;
    }
    const int biased = ex + 7;
    if (biased > 15 || (biased == 15 && mq == 7.0))
        return sgn | 0x7E;
    return sgn | (uint8_t)((biased << 3) | (int)mq);
}

/* Exact widening of one stored element to double. */
static double widen(const void *base, int64_t idx, int dtype)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[idx];
    if (dtype == ORACLE_FP8)
        return e4m3_value(((const uint8_t *)base)[idx]);
    uint32_t bits = (uint32_t)((const uint16_t *)base)[idx] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* Element offset of (physical block, kv head, slot in block, dim 0) in the pool
 * laid out [num_blocks, num_kv_heads, block_size, head_dim] ([P3] kernel sketch). */
static int64_t pool_offset(int64_t blk, int64_t kvh, int64_t off, int64_t nkv, int64_t bs, int64_t d)
{
    return ((blk * nkv + kvh) * bs + off) * d;
}

/*
 * Gather the first `len` tokens of one sequence, one kv head, from the paged pool
 * into contiguous double arrays kd, vd [len][d].  Logical token t lives in
 * physical block table[t / bs] at slot t % bs ([P1] 2.1, [P3] kernel sketch).
 * Returns 0, or -1 if a table entry is outside [0, num_blocks).
 */
static int gather_kv(const void *kc, const void *vc, int dtype, int64_t num_blocks, int64_t nkv,
                     int64_t bs, int64_t d, const int32_t *table, int64_t len, int64_t kvh,
                     double *kd, double *vd)
{
    for (int64_t t = 0; t < len; ++t) {
        int64_t blk = table[t / bs];
        if (blk < 0 || blk >= num_blocks)
            return -1;
        int64_t base = pool_offset(blk, kvh, t % bs, nkv, bs, d);
        for (int64_t i = 0; i < d; ++i) {
            kd[t * d + i] = widen(kc, base + i, dtype);
            vd[t * d + i] = widen(vc, base + i, dtype);
        }
    }
    return 0;
}

/*
 * Textbook attention of one query vector q[d] over n keys/values:
 *   x_t = scale * <q, K_t>,  w_t = exp(x_t - max x) / sum_u exp(x_u - max x),
 *   out = sum_t w_t V_t.
 * n == 0 gives out = 0.
 */
static void attend(const double *q, const double *kd, const double *vd, int64_t n, int64_t d,
                   double scale, double *x, double *out)
{
    for (int64_t i = 0; i < d; ++i)
        out[i] = 0.0;
    if (n == 0)
        return;
    double mx = -INFINITY;
    for (int64_t t = 0; t < n; ++t) {
        double dot = 0.0;
        for (int64_t i = 0; i < d; ++i)
            dot += q[i] * kd[t * d + i];
        x[t] = scale * dot;
        if (x[t] > mx)
            mx = x[t];
    }
    double z = 0.0;
    for (int64_t t = 0; t < n; ++t) {
        x[t] = exp(x[t] - mx);
        z += x[t];
    }
    for (int64_t t = 0; t < n; ++t) {
        double w = x[t] / z;
        for (int64_t i = 0; i < d; ++i)
            out[i] += w * vd[t * d + i];
    }
}

/*
 * Decode attention: one query token per sequence.
 *   query [num_seqs, num_q_heads, d] (dtype), out [num_seqs, num_q_heads, d] (double).
 * Query head h reads kv head h / (num_q_heads / num_kv_heads) (contiguous groups).
 * Returns 0, -1 on a bad table entry, -2 on a bad length, -3 on allocation failure.
 */
int oracle_decode(const void *query, const void *key_cache, const void *value_cache, int dtype,
                  int32_t num_blocks, int32_t num_kv_heads, int32_t block_size, int32_t head_dim,
                  const int32_t *block_tables, int32_t max_blocks_per_seq,
                  const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, double scale,
                  double *out)
{
    const int64_t d = head_dim, nkv = num_kv_heads, bs = block_size;
    const int64_t group = num_q_heads / num_kv_heads;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (context_lens[s] < 0 || context_lens[s] > (int64_t)max_blocks_per_seq * bs)
            return -2;
    int status = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t s = 0; s < num_seqs; ++s) {
        for (int32_t h = 0; h < num_q_heads; ++h) {
            const int64_t len = context_lens[s];
            double *kd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *vd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *x = malloc(sizeof(double) * (size_t)(len + 1));
            double *qd = malloc(sizeof(double) * (size_t)d);
            if (!kd || !vd || !x || !qd) {
#pragma omp atomic write
                status = -3;
            } else {
                const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;
                if (gather_kv(key_cache, value_cache, dtype, num_blocks, nkv, bs, d, table, len,
                              h / group, kd, vd) != 0) {
#pragma omp atomic write
                    status = -1;
                } else {
                    for (int64_t i = 0; i < d; ++i)
                        qd[i] = widen(query, ((int64_t)s * num_q_heads + h) * d + i, dtype);
                    attend(qd, kd, vd, len, d, scale, x,
                           out + ((int64_t)s * num_q_heads + h) * d);
                }
            }
            free(kd);
            free(vd);
            free(x);
            free(qd);
        }
    }
    return status;
}

/*
 * Chunked prefill: sequence s has chunk_lens[s] new query rows, the last ones of
 * its context, so row i sits at position p = context_lens[s] - chunk_lens[s] + i
 * and attends causally to keys 0..p ([P1] 2.3 and 5.1: a long prompt is split
 * into chunks; each chunk's queries attend to everything cached before them).
 *   query/out [num_seqs, max_chunk, num_q_heads, d]; out is double.
 * Only rows with row_mask[s * max_chunk + i] != 0 are computed (row_mask may be
 * NULL = all rows); other out rows are left untouched.
 * Returns 0, -1 bad table entry, -2 bad lengths, -3 allocation failure.
 */
int oracle_prefill(const void *query, const void *key_cache, const void *value_cache, int dtype,
                   int32_t num_blocks, int32_t num_kv_heads, int32_t block_size, int32_t head_dim,
                   const int32_t *block_tables, int32_t max_blocks_per_seq,
                   const int32_t *context_lens, const int32_t *chunk_lens, int32_t num_seqs,
                   int32_t max_chunk, int32_t num_q_heads, double scale, const uint8_t *row_mask,
                   double *out)
{
    const int64_t d = head_dim, nkv = num_kv_heads, bs = block_size;
    const int64_t group = num_q_heads / num_kv_heads;
    for (int32_t s = 0; s < num_seqs; ++s) {
        if (context_lens[s] < 0 || context_lens[s] > (int64_t)max_blocks_per_seq * bs)
            return -2;
        if (chunk_lens[s] < 0 || chunk_lens[s] > max_chunk || chunk_lens[s] > context_lens[s])
            return -2;
    }
    int status = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t s = 0; s < num_seqs; ++s) {
        for (int32_t kvh = 0; kvh < num_kv_heads; ++kvh) {
            const int64_t len = context_lens[s];
            const int64_t start = len - chunk_lens[s];
            double *kd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *vd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *x = malloc(sizeof(double) * (size_t)(len + 1));
            double *qd = malloc(sizeof(double) * (size_t)d);
            if (!kd || !vd || !x || !qd) {
#pragma omp atomic write
                status = -3;
            } else {
                const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;
                if (gather_kv(key_cache, value_cache, dtype, num_blocks, nkv, bs, d, table, len,
                              kvh, kd, vd) != 0) {
#pragma omp atomic write
                    status = -1;
                } else {
                    for (int64_t i = 0; i < chunk_lens[s]; ++i) {
                        if (row_mask && !row_mask[(int64_t)s * max_chunk + i])
                            continue;
                        for (int64_t h = kvh * group; h < (kvh + 1) * group; ++h) {
                            int64_t row = ((int64_t)s * max_chunk + i) * num_q_heads + h;
                            for (int64_t e = 0; e < d; ++e)
                                qd[e] = widen(query, row * d + e, dtype);
                            attend(qd, kd, vd, start + i + 1, d, scale, x, out + row * d);
                        }
                    }
                }
            }
            free(kd);
            free(vd);
            free(x);
            free(qd);
        }
    }
    return status;
}

/*
 * KV append through a slot mapping ([P1] 3.1: the new token's K,V are written
 * back into the cache; slot = physical block * block_size + offset in block).
 *   key/value [num_tokens, num_kv_heads, head_dim] elements of elem_bytes each.
 * slot < 0 is padding and is skipped.  Returns 0, or -1 if a slot is beyond the
 * pool (nothing after it is written).
 */
int oracle_cache_write(const void *key, const void *value, const int64_t *slot_mapping,
                       int32_t num_tokens, void *key_cache, void *value_cache, int32_t num_blocks,
                       int32_t num_kv_heads, int32_t block_size, int32_t head_dim,
                       int32_t elem_bytes)
{
    const int64_t row = (int64_t)head_dim * elem_bytes;
    for (int32_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size)
            return -1;
        int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            int64_t dst = pool_offset(blk, h, off, num_kv_heads, block_size, head_dim) * elem_bytes;
            int64_t src = ((int64_t)i * num_kv_heads + h) * row;
            memcpy((char *)key_cache + dst, (const char *)key + src, (size_t)row);
            memcpy((char *)value_cache + dst, (const char *)value + src, (size_t)row);
        }
    }
    return 0;
}

/*
 * Copy-on-Write block copy ([P3] 关键设计二: allocate a new block and copy the
 * shared block's contents into it).  pairs [num_pairs][2] = (src, dst); every
 * kv head, slot and dim of block src is copied to block dst, in K and in V.
 * Pairs are applied in order.  Returns 0, or -1 on an id outside the pool.
 */
int oracle_copy_blocks(void *key_cache, void *value_cache, const int32_t *pairs, int32_t num_pairs,
                       int32_t num_blocks, int64_t block_bytes)
{
    for (int32_t p = 0; p < num_pairs; ++p) {
        int64_t src = pairs[2 * p], dst = pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return -1;
        memmove((char *)key_cache + dst * block_bytes, (const char *)key_cache + src * block_bytes,
                (size_t)block_bytes);
        memmove((char *)value_cache + dst * block_bytes,
                (const char *)value_cache + src * block_bytes, (size_t)block_bytes);
    }
    return 0;
}

/* Number of OpenMP threads the attention loops use (1 without OpenMP). */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Set the OpenMP thread count for subsequent calls (ignored without OpenMP). */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/* out[i] = the e4m3 code of the binary32 quotient x[i] / scale (fp32 division). */
void oracle_e4m3_encode(const float *x, int64_t n, float scale, uint8_t *out)
{
    for (int64_t i = 0; i < n; ++i) {
        const float t = x[i] / scale;
        out[i] = e4m3_encode(t);
    }
}

/* out[i] = exact value of code c[i]. */
void oracle_e4m3_decode(const uint8_t *c, int64_t n, double *out)
{
    for (int64_t i = 0; i < n; ++i)
        out[i] = e4m3_value(c[i]);
}

/*
 * KV append into FP8 pools: key/value [num_tokens, num_kv_heads, head_dim] bf16;
 * each element x is stored as the e4m3 code of fl32(x) / k_scale (v_scale for V)
 * in pools of one byte per element, laid out as for oracle_cache_write.
 * Returns 0, or -1 if a slot is beyond the pool (nothing after it is written).
 */
int oracle_cache_write_fp8(const void *key, const void *value, const int64_t *slot_mapping,
                           int32_t num_tokens, uint8_t *key_cache, uint8_t *value_cache,
                           int32_t num_blocks, int32_t num_kv_heads, int32_t block_size,
                           int32_t head_dim, float k_scale, float v_scale)
{
    for (int32_t i = 0; i < num_tokens; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size)
            return -1;
        const int64_t blk = slot / block_size, off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            const int64_t dst = pool_offset(blk, h, off, num_kv_heads, block_size, head_dim);
            const int64_t src = ((int64_t)i * num_kv_heads + h) * head_dim;
            for (int32_t k = 0; k < head_dim; ++k) {
                const float kx = (float)widen(key, src + k, ORACLE_BF16);
                const float vx = (float)widen(value, src + k, ORACLE_BF16);
                key_cache[dst + k] = e4m3_encode(kx / k_scale);
                value_cache[dst + k] = e4m3_encode(vx / v_scale);
            }
        }
    }
    return 0;
}

/*
 * Decode attention over FP8 pools: as oracle_decode with bf16 queries, each
 * cached key element taken as its code's value times k_scale and each value
 * element times v_scale (products exact in double).
 */
int oracle_decode_fp8(const void *query, const uint8_t *key_cache, const uint8_t *value_cache,
                      int32_t num_blocks, int32_t num_kv_heads, int32_t block_size, int32_t head_dim,
                      const int32_t *block_tables, int32_t max_blocks_per_seq,
                      const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads, double scale,
                      double k_scale, double v_scale, double *out)
{
    const int64_t d = head_dim, nkv = num_kv_heads, bs = block_size;
    const int64_t group = num_q_heads / num_kv_heads;
    for (int32_t s = 0; s < num_seqs; ++s)
        if (context_lens[s] < 0 || context_lens[s] > (int64_t)max_blocks_per_seq * bs)
            return -2;
    int status = 0;
#pragma omp parallel for collapse(2) schedule(dynamic, 1)
    for (int32_t s = 0; s < num_seqs; ++s) {
        for (int32_t h = 0; h < num_q_heads; ++h) {
            const int64_t len = context_lens[s];
            double *kd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *vd = malloc(sizeof(double) * (size_t)(len * d + 1));
            double *x = malloc(sizeof(double) * (size_t)(len + 1));
            double *qd = malloc(sizeof(double) * (size_t)d);
            if (!kd || !vd || !x || !qd) {
#pragma omp atomic write
                status = -3;
            } else {
                const int32_t *table = block_tables + (int64_t)s * max_blocks_per_seq;
                if (gather_kv(key_cache, value_cache, ORACLE_FP8, num_blocks, nkv, bs, d, table, len,
                              h / group, kd, vd) != 0) {
#pragma omp atomic write
                    status = -1;
                } else {
                    for (int64_t i = 0; i < len * d; ++i) {
                        kd[i] *= k_scale;
                        vd[i] *= v_scale;
                    }
                    for (int64_t i = 0; i < d; ++i)
                        qd[i] = widen(query, ((int64_t)s * num_q_heads + h) * d + i, ORACLE_BF16);
                    attend(qd, kd, vd, len, d, scale, x, out + ((int64_t)s * num_q_heads + h) * d);
                }
            }
            free(kd);
            free(vd);
            free(x);
            free(qd);
        }
    }
    return status;
}

