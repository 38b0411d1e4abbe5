/*
 * Oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Plain, slow, obviously correct CPU code in fp64.  Only tests/, the smoke check
 * in __graft_entry__ and the CPU-baseline leg of bench.py may load it.  It shares
 * no code, header or constant with the GPU library.
 *
 * What it computes (the plain definition; paging changes only where keys and
 * values are read from, never the result):
 *   "What problem does PagedAttention solve, and what is continuous batching?",
 *   section "How PagedAttention works": a block table maps a request's logical
 *   block number to a physical block, and the attention kernel follows that table
 *   when it reads keys and values, so physical blocks 12, 87, 301, 44 still stand
 *   for positions 0..49 in order.  Section "Common misconception": paging is not
 *   compression, it changes layout and allocation only.
 *
 * So for sequence s of length L and query head h (KV head g = h / (Hq / Hkv)):
 *   K_s[j] = pool_K[table[s][j / B]][g][j % B][:]      j = 0..L-1   (gather)
 *   z_j    = scale * sum_i q[s][h][i] * K_s[j][i]
 *   o[i]   = sum_j exp(z_j - max z) V_s[j][i] / sum_j exp(z_j - max z)
 * all in double precision, after widening the stored fp32/fp16/bf16 values
 * exactly to double (or taking already-decoded double values as they are, which is
 * how the FP8 cache's dequantised values come in).
 *
 * Pool layout of one layer: [num_blocks][num_kv_heads][block_size][head_dim].
 * Reading taken where the pages are silent: softmax scale is a parameter
 * (callers pass 1/sqrt(head_dim)); grouped-query heads map by contiguous groups.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F32 = 0, ORACLE_F16 = 1, ORACLE_BF16 = 2, ORACLE_F64 = 3 };

/* IEEE 754 binary16 -> double, from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int expo = (h >> 10) & 0x1F;
    int frac = h & 0x3FF;
    double mag;
    if (expo == 0)
        mag = ldexp((double)frac, -24);                 /* zero or subnormal: frac * 2^-24 */
    else if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + frac), expo - 25);  /* (1 + frac/1024) * 2^(expo-15) */
    return sign ? -mag : mag;
}

/* bfloat16 -> double: the 16 bits are the upper half of an IEEE binary32. */
double oracle_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elem(const void *base, int dtype, size_t idx)
{
    switch (dtype) {
    case ORACLE_F32: return (double)((const float *)base)[idx];
    case ORACLE_F16: return oracle_half_to_double(((const uint16_t *)base)[idx]);
    case ORACLE_F64: return ((const double *)base)[idx];   /* already-decoded values */
    default:         return oracle_bf16_to_double(((const uint16_t *)base)[idx]);
    }
}

/* Decode `count` stored elements to double (used by tests to pin the decoders). */
void oracle_widen(const void *src, int dtype, size_t count, double *dst)
{
    for (size_t i = 0; i < count; ++i)
        dst[i] = load_elem(src, dtype, i);
}

/*
 * Paged decode attention for every (sequence, query head).
 *   k_pool, v_pool : one layer, [num_blocks][num_kv_heads][block_size][head_dim], `dtype`
 *   tables         : [n_seqs][max_blocks] int32 physical block ids
 *   lens           : [n_seqs] int32 tokens per sequence (>= 1)
 *   q              : [n_seqs][num_q_heads][head_dim], `dtype`
 *   out            : [n_seqs][num_q_heads][head_dim] double
 * Returns 0, or -1 for an invalid argument (nothing written then).
 */
int oracle_paged_decode(const void *k_pool, const void *v_pool, int dtype,
                        int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                        const int32_t *tables, int max_blocks, const int32_t *lens, int n_seqs,
                        const void *q, int num_q_heads, double scale, double *out,
                        int n_threads)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || block_size <= 0 || head_dim <= 0)
        return -1;
    for (int s = 0; s < n_seqs; ++s) {
        int L = lens[s];
        if (L < 1 || (L + block_size - 1) / block_size > max_blocks)
            return -1;
        for (int b = 0; b < (L + block_size - 1) / block_size; ++b) {
            int32_t blk = tables[(size_t)s * max_blocks + b];
            if (blk < 0 || blk >= num_blocks)
                return -1;
        }
    }
    const int group = num_q_heads / num_kv_heads;
    const long total = (long)n_seqs * num_q_heads;
#ifdef _OPENMP
    const int nt = n_threads > 0 ? n_threads : omp_get_num_procs();
#else
    (void)n_threads;
#endif

#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (long sh = 0; sh < total; ++sh) {
        const int s = (int)(sh / num_q_heads);
        const int h = (int)(sh % num_q_heads);
        const int g = h / group;
        const int L = lens[s];
        double *K = malloc(sizeof(double) * (size_t)L * head_dim);
        double *V = malloc(sizeof(double) * (size_t)L * head_dim);
        double *z = malloc(sizeof(double) * (size_t)L);
        double *qh = malloc(sizeof(double) * (size_t)head_dim);

        /* gather: logical position j lives in block table[s][j / B] at row j % B */
        for (int j = 0; j < L; ++j) {
            int32_t blk = tables[(size_t)s * max_blocks + j / block_size];
            size_t row = (((size_t)blk * num_kv_heads + g) * block_size + j % block_size) * head_dim;
            for (int i = 0; i < head_dim; ++i) {
                K[(size_t)j * head_dim + i] = load_elem(k_pool, dtype, row + i);
                V[(size_t)j * head_dim + i] = load_elem(v_pool, dtype, row + i);
            }
        }
        for (int i = 0; i < head_dim; ++i)
            qh[i] = load_elem(q, dtype, ((size_t)s * num_q_heads + h) * head_dim + i);

        /* textbook softmax attention on the contiguous arrays */
        double zmax = -INFINITY;
        for (int j = 0; j < L; ++j) {
            double acc = 0.0;
            for (int i = 0; i < head_dim; ++i)
                acc += qh[i] * K[(size_t)j * head_dim + i];
            z[j] = scale * acc;
            if (z[j] > zmax)
                zmax = z[j];
        }
        double denom = 0.0;
        for (int j = 0; j < L; ++j) {
            z[j] = exp(z[j] - zmax);
            denom += z[j];
        }
        double *o = out + ((size_t)s * num_q_heads + h) * head_dim;
        for (int i = 0; i < head_dim; ++i) {
            double acc = 0.0;
            for (int j = 0; j < L; ++j)
                acc += z[j] * V[(size_t)j * head_dim + i];
            o[i] = acc / denom;
        }
        free(K);
        free(V);
        free(z);
        free(qh);
    }
    return 0;
}

/*
 * Paged chunked-prefill attention (causal), the same definition applied to every
 * query of a prompt chunk: "What problem does PagedAttention solve, and what is
 * continuous batching?", sections "Why the KV cache becomes the problem" (prefill
 * is the pass over the prompt) and "The prefill and decode phases need careful
 * scheduling" (chunked prefill breaks a long prompt into pieces).  Reading: the
 * chunk's keys and values are already in the cache, the chunk is the last C_s
 * tokens of sequence s, and the query at absolute position p attends to keys 0..p.
 *   q     : [total_q][num_q_heads][head_dim]; sequence s owns rows
 *           q_start[s] .. q_start[s+1]-1 (C_s rows, C_s <= lens[s])
 *   out   : same shape, double
 * Returns 0, or -1 for an invalid argument (nothing written then).
 */
int oracle_paged_prefill(const void *k_pool, const void *v_pool, int dtype,
                         int64_t num_blocks, int block_size, int num_kv_heads, int head_dim,
                         const int32_t *tables, int max_blocks, const int32_t *lens,
                         const int32_t *q_start, int n_seqs, const void *q, int num_q_heads,
                         double scale, double *out, int n_threads)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || block_size <= 0 || head_dim <= 0)
        return -1;
    for (int s = 0; s < n_seqs; ++s) {
        int L = lens[s], C = q_start[s + 1] - q_start[s];
        if (L < 1 || C < 0 || C > L || (L + block_size - 1) / block_size > max_blocks)
            return -1;
        for (int b = 0; b < (L + block_size - 1) / block_size; ++b) {
            int32_t blk = tables[(size_t)s * max_blocks + b];
            if (blk < 0 || blk >= num_blocks)
                return -1;
        }
    }
    const int group = num_q_heads / num_kv_heads;
    const long total_rows = q_start[n_seqs];
#ifdef _OPENMP
    const int nt = n_threads > 0 ? n_threads : omp_get_num_procs();
#else
    (void)n_threads;
#endif

#pragma omp parallel for schedule(dynamic, 1) num_threads(nt)
    for (long rh = 0; rh < total_rows * num_q_heads; ++rh) {
        const long row = rh / num_q_heads;
        const int h = (int)(rh % num_q_heads);
        const int g = h / group;
        int s = 0;
        while (q_start[s + 1] <= row)
            ++s;
        const int L = lens[s];
        const int C = q_start[s + 1] - q_start[s];
        const int p = L - C + (int)(row - q_start[s]);      /* absolute position of this query */
        const int nkeys = p + 1;                              /* causal: keys 0..p */
        double *z = malloc(sizeof(double) * (size_t)nkeys);
        double *qh = malloc(sizeof(double) * (size_t)head_dim);
        for (int i = 0; i < head_dim; ++i)
            qh[i] = load_elem(q, dtype, ((size_t)row * num_q_heads + h) * head_dim + i);
        double zmax = -INFINITY;
        for (int j = 0; j < nkeys; ++j) {
            int32_t blk = tables[(size_t)s * max_blocks + j / block_size];
            size_t base = (((size_t)blk * num_kv_heads + g) * block_size + j % block_size) * head_dim;
            double acc = 0.0;
            for (int i = 0; i < head_dim; ++i)
                acc += qh[i] * load_elem(k_pool, dtype, base + i);
            z[j] = scale * acc;
            if (z[j] > zmax)
                zmax = z[j];
        }
        double denom = 0.0;
        for (int j = 0; j < nkeys; ++j) {
            z[j] = exp(z[j] - zmax);
            denom += z[j];
        }
        double *o = out + ((size_t)row * num_q_heads + h) * head_dim;
        for (int i = 0; i < head_dim; ++i)
            o[i] = 0.0;
        for (int j = 0; j < nkeys; ++j) {
            int32_t blk = tables[(size_t)s * max_blocks + j / block_size];
            size_t base = (((size_t)blk * num_kv_heads + g) * block_size + j % block_size) * head_dim;
            for (int i = 0; i < head_dim; ++i)
                o[i] += z[j] * load_elem(v_pool, dtype, base + i);
        }
        for (int i = 0; i < head_dim; ++i)
            o[i] /= denom;
        free(z);
        free(qh);
    }
    return 0;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_num_procs();
#else
    return 1;
#endif
}
