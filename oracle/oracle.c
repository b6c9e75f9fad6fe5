/*
 * oracle.c -- plain, slow, obviously correct CPU reference for the PagedAttention
 * hot path.  TEST INFRASTRUCTURE ONLY: nothing on the product path links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header, table or constant with the CUDA library.
 *
 * Sources (the three web pages this library follows):
 *   [Core Concepts]  "3、核心概念：LLM推理原理、KV Cache、PagedAttention、连续批处理" --
 *                    §3.1 (autoregressive decode with a KV cache), §3.2 (fixed-size blocks,
 *                    block table, "PagedAttention 如何工作": prefill writes prompt K/V into
 *                    blocks, each decode step writes the new token at the end of the current
 *                    block and takes a new physical block when it is full; the kernel reads
 *                    the non-contiguous KV through the block table).
 *   [vLLM overview]  uml.org.cn vLLM page, section 二 (PagedAttention: pages of 16 tokens,
 *                    per-request page table, pages stitched back together for attention;
 *                    Prefix Sharing: shared pages stay unchanged, a diverging request's new
 *                    token is written into a copied page -- copy-on-write).
 *   [KV Cache to vLLM] "从KV Cache到vLLM：大模型推理提速与显存优化实战" -- §1.2 (the new
 *                    token's query attends over all cached keys, the weighted sum of values),
 *                    §2.1 (KV size formula), §2.2 (1-byte KV storage, GQA head sharing).
 *
 * Conventions (the pages fix none of these; the readings are listed with the design notes):
 *   - block size bs = 16 or 32 tokens (Core Concepts §3.2: "usually 16 or 32");
 *     cache layout [num_blocks][num_kv_heads][bs][head_dim];
 *   - bf16 values are passed as their 16-bit patterns (uint16_t), fp8 as E4M3 bytes;
 *   - query head h uses KV head floor(h / (Hq / Hkv)) (contiguous GQA groups);
 *   - all attention arithmetic is fp64 on the exact values of the inputs.
 *
 * Every function returns 0 on success and a negative number on a malformed input
 * (-1: a size is invalid, -4: a block id or slot points outside the pool).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>


/* ---------------------------------------------------------------- value formats */

/* bf16 -> double: a bf16 pattern is the upper half of an IEEE binary32 pattern. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static float bf16_value_f(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/*
 * E4M3 (OCP 8-bit floating point, "FN" flavour) decode, written from the format's
 * definition: 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits.  Exponent
 * field 0 encodes subnormals m/8 * 2^-6; S.1111.111 is NaN; no infinities.
 */
double oracle_e4m3_decode(uint8_t code)
{
    int sign = (code >> 7) & 1;
    int e = (code >> 3) & 0xF;
    int m = code & 0x7;
    double v;
    if (e == 0xF && m == 0x7) return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

/* values of the 127 non-negative finite E4M3 codes 0x00 .. 0x7E, which ascend with the code */
static double e4m3_pos_value[127];

__attribute__((constructor)) static void e4m3_table_init(void)
{
    for (int c = 0; c < 127; ++c) e4m3_pos_value[c] = oracle_e4m3_decode((uint8_t)c);
}

/*
 * E4M3 encode of a binary32 value: round to nearest, ties to the code with an even mantissa,
 * saturating to +-448 (the largest finite magnitude).  |x| is bracketed between two consecutive
 * non-negative codes by bisection over their ascending values, then the nearer one is taken (on a tie
 * the even one: consecutive codes differ in the last mantissa bit).  NaN maps to the NaN code 0x7F
 * (sign kept).
 */
uint8_t oracle_e4m3_encode(float x)
{
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs((double)x);
    int lo = 0, hi = 126, best;
    double below, above;
    if (isnan(x)) return (uint8_t)(sign | 0x7F);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E); /* satfinite */
    while (hi - lo > 1) { /* invariant: value[lo] <= a < value[hi] */
        int mid = (lo + hi) / 2;
        if (e4m3_pos_value[mid] <= a) lo = mid; else hi = mid;
    }
    below = a - e4m3_pos_value[lo];
    above = e4m3_pos_value[hi] - a;
    best = (above < below || (above == below && (hi & 1) == 0)) ? hi : lo;
    return (uint8_t)(sign | best);
}

/*
 * INT8 KV element [KV Cache to vLLM §2.2: INT8 and FP8 KV caches store one byte per element]:
 * symmetric quantisation with one fp32 scale per KV head; code = clamp(round(x / scale), -127, 127),
 * rounding the binary32 quotient to the nearest integer, ties to even; value = code * scale.
 */
int8_t oracle_int8_encode(float x)
{
    float r = rintf(x); /* default rounding mode: to nearest, ties to even */
    if (isnan(x)) return 0;
    if (r > 127.0f) r = 127.0f;
    if (r < -127.0f) r = -127.0f;
    return (int8_t)r;
}

/*
 * KV size formula [KV Cache to vLLM §2.1]:
 *   bytes = 2 (K and V) x layers x kv_heads x head_dim x seq_len x batch x bytes/element.
 */
int64_t oracle_kv_cache_bytes(int64_t layers, int64_t kv_heads, int64_t head_dim,
                              int64_t seq_len, int64_t batch, int64_t elem_bytes)
{
    return 2 * layers * kv_heads * head_dim * seq_len * batch * elem_bytes;
}

/* ---------------------------------------------------------------- append */

/*
 * Append [Core Concepts §3.2, "PagedAttention 如何工作"]: each token n carries its
 * slot = physical_block * bs + offset; its K and V rows (all KV heads) are written at
 * cache[slot / bs][h][slot % bs][:].  slot < 0 marks a padding token: nothing written.
 * kv_dtype 0 = bf16 (bit copy), 1 = fp8 E4M3 (code of the binary32 quotient x / scale[h]),
 * 2 = int8 (rounded quotient, see oracle_int8_encode).
 */
int oracle_kv_append(void *k_cache, void *v_cache, const uint16_t *k, const uint16_t *v,
                     const int64_t *slot_mapping, int64_t num_tokens, int num_kv_heads,
                     int head_dim, int64_t num_blocks, int bs, int kv_dtype,
                     const float *k_scale, const float *v_scale)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || bs <= 0) return -1;
    if (kv_dtype < 0 || kv_dtype > 2) return -1;
    for (int64_t n = 0; n < num_tokens; ++n) {
        int64_t slot = slot_mapping[n];
        if (slot < 0) continue;
        if (slot >= num_blocks * bs) return -4;
    }
    /* KV heads are disjoint parts of the cache: one thread per head, tokens in order within it */
#pragma omp parallel for schedule(static)
    for (int h = 0; h < num_kv_heads; ++h) {
        for (int64_t n = 0; n < num_tokens; ++n) {
            int64_t slot = slot_mapping[n];
            int64_t blk, off;
            if (slot < 0) continue;
            blk = slot / bs;
            off = slot % bs;
            int64_t src = (n * num_kv_heads + h) * (int64_t)head_dim;
            int64_t dst = ((blk * num_kv_heads + h) * bs + off) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d) {
                if (kv_dtype == 0) {
                    ((uint16_t *)k_cache)[dst + d] = k[src + d];
                    ((uint16_t *)v_cache)[dst + d] = v[src + d];
                } else {
                    /* binary32 division: C float '/' is the IEEE correctly rounded divide */
                    float qk = bf16_value_f(k[src + d]) / k_scale[h];
                    float qv = bf16_value_f(v[src + d]) / v_scale[h];
                    if (kv_dtype == 1) {
                        ((uint8_t *)k_cache)[dst + d] = oracle_e4m3_encode(qk);
                        ((uint8_t *)v_cache)[dst + d] = oracle_e4m3_encode(qv);
                    } else {
                        ((int8_t *)k_cache)[dst + d] = oracle_int8_encode(qk);
                        ((int8_t *)v_cache)[dst + d] = oracle_int8_encode(qv);
                    }
                }
            }
        }
    }
    return 0;
}

/* ---------------------------------------------------------------- copy-on-write */

/*
 * Copy-on-write fork [vLLM overview, Prefix Sharing]: for each (src, dst) pair the whole
 * physical block (all KV heads, 16 slots, K and V) is copied, so the diverging request's
 * next token can be written into its private copy while the shared page stays unchanged.
 * Pairs are applied in order.
 */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int32_t *pairs, int64_t num_pairs,
                       int num_kv_heads, int head_dim, int64_t num_blocks, int bs, int elem_bytes)
{
    int64_t block_bytes = (int64_t)num_kv_heads * bs * head_dim * elem_bytes;
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || elem_bytes <= 0) return -1;
    for (int64_t p = 0; p < num_pairs; ++p) {
        int32_t s = pairs[2 * p], d = pairs[2 * p + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks) return -4;
    }
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
        memmove((char *)k_cache + d * block_bytes, (char *)k_cache + s * block_bytes, block_bytes);
        memmove((char *)v_cache + d * block_bytes, (char *)v_cache + s * block_bytes, block_bytes);
    }
    return 0;
}

/*
 * Swap [vLLM overview, section 三 (KV cache eviction): when GPU memory runs short, pages are moved
 * out to CPU memory, and brought back when needed]: for each (src, dst) pair the whole block of
 * the source pool (all KV heads, 16 slots, K and V) is copied into block dst of the destination
 * pool.  The two pools are distinct arrays with the same per-block geometry.
 */
int oracle_swap_blocks(void *dst_k, void *dst_v, int64_t dst_num_blocks, const void *src_k, const void *src_v,
                       int64_t src_num_blocks, const int32_t *pairs, int64_t num_pairs, int num_kv_heads,
                       int head_dim, int bs, int elem_bytes)
{
    int64_t block_bytes = (int64_t)num_kv_heads * bs * head_dim * elem_bytes;
    if (num_pairs < 0 || num_kv_heads <= 0 || head_dim <= 0 || elem_bytes <= 0) return -1;
    for (int64_t p = 0; p < num_pairs; ++p) {
        int32_t s = pairs[2 * p], d = pairs[2 * p + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks) return -4;
    }
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t s = pairs[2 * p], d = pairs[2 * p + 1];
        memcpy((char *)dst_k + d * block_bytes, (const char *)src_k + s * block_bytes, block_bytes);
        memcpy((char *)dst_v + d * block_bytes, (const char *)src_v + s * block_bytes, block_bytes);
    }
    return 0;
}

/* ---------------------------------------------------------------- attention */

/* value of element d of token t (logical position) of KV head g of one sequence, read
 * through that sequence's block table: physical block = table[t / bs], slot t % bs. */
static double cache_value(const void *cache, int kv_dtype, float scale, int64_t phys, int bs,
                          int num_kv_heads, int g, int64_t t, int head_dim, int d)
{
    int64_t idx = ((phys * num_kv_heads + g) * bs + (t % bs)) * (int64_t)head_dim + d;
    if (kv_dtype == 0) return bf16_value(((const uint16_t *)cache)[idx]);
    if (kv_dtype == 2) return (double)((const int8_t *)cache)[idx] * (double)scale;
    return oracle_e4m3_decode(((const uint8_t *)cache)[idx]) * (double)scale;
}

/*
 * Gather the first n_keys tokens of one sequence's paged K/V (one KV head) into contiguous [n_keys][D]
 * arrays: the block table "stitches the pages back together" (vLLM overview, section 二).
 */
static int gather_kv(double *K, double *V, const void *k_cache, const void *v_cache, int kv_dtype, float ks,
                     float vs, const int32_t *table, int64_t n_keys, int num_kv_heads, int g, int head_dim,
                     int64_t num_blocks, int bs)
{
    for (int64_t t = 0; t < n_keys; ++t) {
        int64_t phys = table[t / bs];
        if (phys < 0 || phys >= num_blocks) return -4;
        for (int d = 0; d < head_dim; ++d) {
            K[t * head_dim + d] = cache_value(k_cache, kv_dtype, ks, phys, bs, num_kv_heads, g, t, head_dim, d);
            V[t * head_dim + d] = cache_value(v_cache, kv_dtype, vs, phys, bs, num_kv_heads, g, t, head_dim, d);
        }
    }
    return 0;
}

/*
 * Attention of one query vector over the first n_keys rows of gathered K/V
 * [KV Cache to vLLM §1.2; Core Concepts §3.1]:
 *   s_t = scale * sum_d q_d K_td,  p = softmax(s),  o_d = sum_t p_t V_td.
 * n_keys == 0 gives o = 0.
 */
static void attend_gathered(double *out, const uint16_t *q, const double *K, const double *V, int64_t n_keys,
                            int head_dim, double scale, double *s)
{
    double mx, sum;
    for (int d = 0; d < head_dim; ++d) out[d] = 0.0;
    if (n_keys == 0) return;
    for (int64_t t = 0; t < n_keys; ++t) {
        double acc = 0.0;
        for (int d = 0; d < head_dim; ++d) acc += bf16_value(q[d]) * K[t * head_dim + d];
        s[t] = scale * acc;
    }
    mx = s[0];
    for (int64_t t = 1; t < n_keys; ++t) if (s[t] > mx) mx = s[t];
    sum = 0.0;
    for (int64_t t = 0; t < n_keys; ++t) { s[t] = exp(s[t] - mx); sum += s[t]; }
    for (int64_t t = 0; t < n_keys; ++t) {
        double p = s[t] / sum;
        for (int d = 0; d < head_dim; ++d) out[d] += p * V[t * head_dim + d];
    }
}

/*
 * Decode attention [Core Concepts §3.2; KV Cache to vLLM §1.2, §2.2]: for every sequence
 * b and query head h, the new token's query q[b][h] attends over all context_lens[b]
 * cached tokens (the just-appended one included) of KV head h / (Hq / Hkv).
 * q: [B][Hq][D] bf16; block_tables: [B][max_blocks_per_seq]; out: [B][Hq][D] fp64.
 */
int oracle_paged_decode(double *out, const uint16_t *q, const void *k_cache, const void *v_cache,
                        const int32_t *block_tables, int max_blocks_per_seq,
                        const int32_t *context_lens, int num_seqs, int num_q_heads,
                        int num_kv_heads, int head_dim, int64_t num_blocks, int bs, double scale,
                        int kv_dtype, const float *k_scale, const float *v_scale)
{
    int64_t max_len = 0;
    int status = 0;
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return -1;
    if (num_q_heads % num_kv_heads != 0) return -1;
    for (int b = 0; b < num_seqs; ++b) {
        if (context_lens[b] < 0) return -1;
        if ((context_lens[b] + bs - 1) / bs > max_blocks_per_seq) return -1;
        if (context_lens[b] > max_len) max_len = context_lens[b];
    }
#pragma omp parallel reduction(min : status)
    {
        double *K = (double *)malloc(sizeof(double) * (size_t)(max_len + 1) * head_dim);
        double *V = (double *)malloc(sizeof(double) * (size_t)(max_len + 1) * head_dim);
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_len + 1));
#pragma omp for schedule(dynamic)
        for (int64_t bh = 0; bh < (int64_t)num_seqs * num_q_heads; ++bh) {
            int b = (int)(bh / num_q_heads), h = (int)(bh % num_q_heads);
            int g = h / (num_q_heads / num_kv_heads);
            float ks = kv_dtype ? k_scale[g] : 1.0f, vs = kv_dtype ? v_scale[g] : 1.0f;
            int r = gather_kv(K, V, k_cache, v_cache, kv_dtype, ks, vs,
                              block_tables + (int64_t)b * max_blocks_per_seq, context_lens[b],
                              num_kv_heads, g, head_dim, num_blocks, bs);
            if (r < status) status = r;
            if (r == 0)
                attend_gathered(out + bh * head_dim, q + bh * head_dim, K, V, context_lens[b], head_dim, scale, s);
        }
        free(K);
        free(V);
        free(s);
    }
    return status;
}

/*
 * Prefill of a chunk over its paged history [vLLM overview, Continuous Batching: requests
 * in prefill run in the same batch as decoding ones; Core Concepts §3.2: prefill writes the
 * prompt's K/V into blocks].  Chunk c holds queries cu_q_lens[c] .. cu_q_lens[c+1]-1 (C_c of
 * them); context_lens[c] = H_c + C_c counts its history H_c plus the chunk.  Query i of the
 * chunk sits at absolute position H_c + i and attends, causally, to tokens t <= H_c + i.
 * q, out: [total_q][Hq][D].
 */
int oracle_paged_prefill(double *out, const uint16_t *q, const int32_t *cu_q_lens, int num_chunks,
                         const void *k_cache, const void *v_cache, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *context_lens, int num_q_heads,
                         int num_kv_heads, int head_dim, int64_t num_blocks, int bs, double scale,
                         int kv_dtype, const float *k_scale, const float *v_scale)
{
    int64_t max_len = 0;
    int status = 0;
    if (num_chunks < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0) return -1;
    if (num_q_heads % num_kv_heads != 0) return -1;
    for (int c = 0; c < num_chunks; ++c) {
        int32_t C = cu_q_lens[c + 1] - cu_q_lens[c];
        if (C < 0 || context_lens[c] < C) return -1;
        if ((context_lens[c] + bs - 1) / bs > max_blocks_per_seq) return -1;
        if (context_lens[c] > max_len) max_len = context_lens[c];
    }
#pragma omp parallel reduction(min : status)
    {
        double *K = (double *)malloc(sizeof(double) * (size_t)(max_len + 1) * head_dim);
        double *V = (double *)malloc(sizeof(double) * (size_t)(max_len + 1) * head_dim);
        double *s = (double *)malloc(sizeof(double) * (size_t)(max_len + 1));
        /* per (chunk, query head): the chunk's context is gathered once; row i then attends over its
         * first hist + i + 1 keys */
#pragma omp for schedule(dynamic)
        for (int64_t ch = 0; ch < (int64_t)num_chunks * num_q_heads; ++ch) {
            int c = (int)(ch / num_q_heads), h = (int)(ch % num_q_heads);
            int g = h / (num_q_heads / num_kv_heads);
            float ks = kv_dtype ? k_scale[g] : 1.0f, vs = kv_dtype ? v_scale[g] : 1.0f;
            int64_t C = cu_q_lens[c + 1] - cu_q_lens[c];
            int64_t hist = context_lens[c] - C;
            int r = gather_kv(K, V, k_cache, v_cache, kv_dtype, ks, vs,
                              block_tables + (int64_t)c * max_blocks_per_seq, context_lens[c],
                              num_kv_heads, g, head_dim, num_blocks, bs);
            if (r < status) status = r;
            for (int64_t i = 0; r == 0 && i < C; ++i) {
                int64_t ih = (cu_q_lens[c] + i) * num_q_heads + h;
                attend_gathered(out + ih * head_dim, q + ih * head_dim, K, V,
                                hist + i + 1, head_dim, scale, s);
            }
        }
        free(K);
        free(V);
        free(s);
    }
    return status;
}

/* number of OpenMP threads the oracle runs with (1 when built without OpenMP) */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* run the following calls on n OpenMP threads (for timing the oracle on one core and on all) */
void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    extern void omp_set_num_threads(int);
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
