/*
 * Plain C fp64 oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Independent second implementation of the NumPy oracle (oracle/reference.py);
 * it shares no code with the CUDA library and includes none of its headers.
 * Used by the tests (cross-check against the NumPy oracle and, through it,
 * the pins) and timed as the CPU baseline of the benchmark.
 *
 * What it computes, per sequence b and query head h (the pages' description:
 * "PagedAttention" digest, sections "PagedAttention in one picture" and
 * "Misconceptions" -- walk the block table, gather each token's K and V from
 * wherever its block lives, then ordinary attention, unchanged):
 *   kv head   g   = h / (Hq / Hkv)
 *   token i   of  [0, ctx_b) lives at block_tables[b][i / BS], offset i % BS
 *   s_i       = scale * sum_d q[b,h,d] * K_i[d]
 *   p_i       = exp(s_i - max s) / sum_j exp(s_j - max s)
 *   out[b,h]  = sum_i p_i V_i
 * Everything in double on exactly upcast stored values.  ctx_b = 0 gives a
 * zero row.
 *
 * Cache layout: [NB][Hkv][BS][D] row-major, element type by `dtype`
 * (0 = f32, 1 = f16, 2 = bf16).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC pa_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2 };

/* IEEE 754 binary16 -> double, from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
static double half_to_double(uint16_t h) {
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    } else if (e == 31) {
        v = f ? NAN : INFINITY;
    } else {
        v = ldexp((double)(1024 + f), e - 25);     /* (1 + f/1024) * 2^(e-15) */
    }
    return sign ? -v : v;
}

/* bfloat16 is the upper 16 bits of a binary32. */
static double bf16_to_double(uint16_t h) {
    uint32_t u = (uint32_t)h << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double load_elt(const void* base, size_t idx, int dtype) {
    switch (dtype) {
        case OR_F32: return (double)((const float*)base)[idx];
        case OR_F16: return half_to_double(((const uint16_t*)base)[idx]);
        default: return bf16_to_double(((const uint16_t*)base)[idx]);
    }
}

/* One output row: sequence b, query head h, KV head g.  Returns 0, or -2 if
 * the context needs a table entry past max_blocks_per_seq or a block id lies
 * outside [0, NB).  o[D] is zeroed first. */
static int decode_row(double* o, const void* q, const void* key_cache, const void* value_cache,
                      int dtype, const int32_t* block_tables, int max_blocks_per_seq, int ctx,
                      int b, int h, int g, int num_heads, int num_kv_heads, int D,
                      int block_size, int num_blocks, double scale) {
    for (int d = 0; d < D; ++d) o[d] = 0.0;
    if (ctx <= 0) return 0;
    if ((ctx + block_size - 1) / block_size > max_blocks_per_seq) return -2;

    double* qv = (double*)malloc(sizeof(double) * D);
    double* s = (double*)malloc(sizeof(double) * ctx);
    size_t* row = (size_t*)malloc(sizeof(size_t) * ctx);
    int rc = 0;
    for (int d = 0; d < D; ++d) qv[d] = load_elt(q, ((size_t)b * num_heads + h) * D + d, dtype);

    /* step 1: walk the block table -> element offset of each token's row */
    for (int i = 0; i < ctx; ++i) {
        const int blk = block_tables[(size_t)b * max_blocks_per_seq + i / block_size];
        if (blk < 0 || blk >= num_blocks) { rc = -2; break; }
        row[i] = (((size_t)blk * num_kv_heads + g) * block_size + (size_t)(i % block_size)) * D;
    }
    if (rc == 0) {
        /* step 2: logits */
        double m = -INFINITY;
        for (int i = 0; i < ctx; ++i) {
            double acc = 0.0;
            for (int d = 0; d < D; ++d) acc += qv[d] * load_elt(key_cache, row[i] + d, dtype);
            s[i] = scale * acc;
            if (s[i] > m) m = s[i];
        }
        /* step 3: softmax weights */
        double l = 0.0;
        for (int i = 0; i < ctx; ++i) { s[i] = exp(s[i] - m); l += s[i]; }
        /* step 4: weighted sum of V */
        for (int i = 0; i < ctx; ++i) {
            const double p = s[i] / l;
            for (int d = 0; d < D; ++d) o[d] += p * load_elt(value_cache, row[i] + d, dtype);
        }
    }
    free(qv); free(s); free(row);
    return rc;
}

/* Every (b, h).  out is [num_seqs][num_heads][head_dim].  Returns 0, -1 on bad
 * arguments, -2 if some needed block id is outside the pool or a context
 * exceeds the table (those rows are left zero). */
int oracle_decode(double* out, const void* q, const void* key_cache, const void* value_cache,
                  int dtype, const int32_t* block_tables, int max_blocks_per_seq,
                  const int32_t* context_lens, int num_seqs, int num_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, double scale, int num_threads) {
    if (!out || !q || !key_cache || !value_cache || !block_tables || !context_lens) return -1;
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0) return -1;
    const int group = num_heads / num_kv_heads;
    int status = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (long bh = 0; bh < (long)num_seqs * num_heads; ++bh) {
        const int b = (int)(bh / num_heads), h = (int)(bh % num_heads);
        const int rc = decode_row(out + (size_t)bh * head_dim, q, key_cache, value_cache, dtype,
                                  block_tables, max_blocks_per_seq, context_lens[b], b, h, h / group,
                                  num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale);
        if (rc < status) status = rc;
    }
    return status;
}

/* A chosen subset of (b, h): pairs[2k] = b, pairs[2k+1] = h; out is
 * [npairs][head_dim].  Same arithmetic as oracle_decode. */
int oracle_decode_pairs(double* out, const int32_t* pairs, int npairs, const void* q,
                        const void* key_cache, const void* value_cache, int dtype,
                        const int32_t* block_tables, int max_blocks_per_seq,
                        const int32_t* context_lens, int num_heads, int num_kv_heads,
                        int head_dim, int block_size, int num_blocks, double scale,
                        int num_threads) {
    if (!out || !pairs || !q || !key_cache || !value_cache || !block_tables || !context_lens) return -1;
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0) return -1;
    const int group = num_heads / num_kv_heads;
    int status = 0;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#else
    (void)num_threads;
#endif
#pragma omp parallel for schedule(dynamic) reduction(min : status)
    for (int k = 0; k < npairs; ++k) {
        const int b = pairs[2 * k], h = pairs[2 * k + 1];
        const int rc = decode_row(out + (size_t)k * head_dim, q, key_cache, value_cache, dtype,
                                  block_tables, max_blocks_per_seq, context_lens[b], b, h, h / group,
                                  num_heads, num_kv_heads, head_dim, block_size, num_blocks, scale);
        if (rc < status) status = rc;
    }
    return status;
}
