/*
 * gqa_oracle.c -- plain fp64 CPU oracle for single-query (decode) grouped-query
 * attention over an optionally paged KV cache.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the bench's
 * CPU-baseline leg may load or call this file.  The product path (the CUDA
 * library) never does, and this file shares no code, header, table or helper
 * with it.
 *
 * What it computes, and where the pages fix it:
 *
 *   For request b and query head h, with G = Hq / Hkv query heads per KV head
 *   and kvh = floor(h / G) ("a group of G query heads shares one key/value
 *   head": Attention co-design for long-context inference, glossary entry
 *   "Group size (G)"; Essential LLM optimization techniques (2), section 1-1,
 *   the Llama 3 config with 32 attention heads over 8 KV heads):
 *
 *       s_t   = scale * sum_d q[b,h,d] * K[b,kvh,t,d]          0 <= t < L_b
 *       out   = sum_t softmax(s)_t * V[b,kvh,t,:]
 *
 *   One query token per head attends to every cached key of its request
 *   (Inference optimization: KV cache, MQA/GQA, batching..., section 1
 *   "Prefill and decode" and section 2 "KV cache"; LeanAttention decode tiles
 *   digest, section "Prefill and decode have different shapes").
 *
 *   Row t of (b, kvh) is found through the block table: logical block t / bs of
 *   request b names a physical block, and the row sits at offset t mod bs inside
 *   it (Essential LLM optimization techniques (2), section 3 "PagedAttention",
 *   Figure 6-13).  Cache layout (the pages do not fix one):
 *   [num_blocks, Hkv, block_size, D]; with no block table the cache is
 *   [B, Hkv, capacity, D] and block_size is the per-request capacity.
 *
 *   A partial softmax state over a key range is (m, l, acc) with
 *   m = max_t s_t, l = sum_t exp(s_t - m), acc = sum_t exp(s_t - m) V_t.  Partial
 *   states merge exactly after rescaling to a common maximum (LeanAttention
 *   decode tiles digest, section "Exact softmax that merges piece by piece").
 *
 * Everything is evaluated in double precision from the exactly upcast bf16
 * inputs, with a plain two-pass softmax (maximum first, then exponentials).
 * Slots past a request's length and unused block-table entries are never read.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_OK 0
#define ORACLE_BAD_ARG 1
#define ORACLE_BAD_BLOCK 2
#define ORACLE_NO_MEMORY 3

/* bf16 is the upper half of an IEEE binary32; widening it is exact. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_bf16_to_double(uint16_t bits) { return bf16_to_double(bits); }

/* FP8 E4M3 (the "fn" encoding: 1 sign bit, 4 exponent bits with bias 7, 3
 * mantissa bits, no infinities, S.1111.111 is NaN), widened exactly:
 * normal (-1)^s 2^(e-7) (1 + m/8), subnormal (e = 0) (-1)^s 2^-6 (m/8). */
static double e4m3_to_double(uint8_t bits)
{
    int s = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m / 8.0, -6);
    else
        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return s ? -v : v;
}

double oracle_e4m3_to_double(uint8_t bits) { return e4m3_to_double(bits); }

/* One cache holds bf16 rows, or FP8 E4M3 rows with one scale per tensor (the
 * value is the E4M3 number times k_scale or v_scale): FP8 caches halve the bytes
 * a decode step reads (Attention co-design for long-context inference, the
 * FP8 KV cache in its list of techniques). */
typedef struct {
    const uint16_t *k, *v;
    const uint8_t *k8, *v8;     /* non-NULL: FP8 cache (k, v unused) */
    double k_scale, v_scale;
    const int32_t *block_table; /* NULL: contiguous cache */
    int Hkv, D, block_size, max_blocks, num_blocks;
} kv_cache;

static double key_at(const kv_cache *c, int64_t i)
{
    return c->k8 ? e4m3_to_double(c->k8[i]) * c->k_scale : bf16_to_double(c->k[i]);
}

static double value_at(const kv_cache *c, int64_t i)
{
    return c->v8 ? e4m3_to_double(c->v8[i]) * c->v_scale : bf16_to_double(c->v[i]);
}

/* Element offset of key/value row t of (request b, kv head kvh); -1 when the
 * block table names a block outside the pool. */
static int64_t kv_row(const kv_cache *c, int b, int kvh, int64_t t)
{
    int64_t block, offset;
    if (c->block_table) {
        block = c->block_table[(int64_t)b * c->max_blocks + t / c->block_size];
        offset = t % c->block_size;
        if (block < 0 || block >= c->num_blocks)
            return -1;
    } else {
        block = b;
        offset = t;
    }
    return ((block * c->Hkv + kvh) * (int64_t)c->block_size + offset) * c->D;
}

/* Partial softmax state of query vector qrow against key rows [t0, t1) of
 * (b, kvh).  acc has D entries.  An empty range gives m = -inf, l = 0, acc = 0. */
static int attention_state(const kv_cache *c, const uint16_t *qrow, double scale,
                           int b, int kvh, int64_t t0, int64_t t1,
                           double *acc, double *m_out, double *l_out)
{
    const int D = c->D;
    int64_t n = t1 > t0 ? t1 - t0 : 0;
    for (int d = 0; d < D; ++d)
        acc[d] = 0.0;
    *m_out = -INFINITY;
    *l_out = 0.0;
    if (n == 0)
        return ORACLE_OK;

    double *s = (double *)malloc((size_t)n * sizeof(double));
    int64_t *rows = (int64_t *)malloc((size_t)n * sizeof(int64_t));
    if (!s || !rows) {
        free(s);
        free(rows);
        return ORACLE_NO_MEMORY;
    }

    /* Scores: s_t = scale * <q, k_t>. */
    for (int64_t i = 0; i < n; ++i) {
        int64_t row = kv_row(c, b, kvh, t0 + i);
        if (row < 0) {
            free(s);
            free(rows);
            return ORACLE_BAD_BLOCK;
        }
        rows[i] = row;
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_double(qrow[d]) * key_at(c, row + d);
        s[i] = scale * dot;
    }

    /* Pass 1: the maximum score. */
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i)
        if (s[i] > m)
            m = s[i];

    /* Pass 2: exponentials relative to the maximum, their sum, and the
     * exponential-weighted sum of value rows. */
    double l = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(s[i] - m);
        l += w;
        for (int d = 0; d < D; ++d)
            acc[d] += w * value_at(c, rows[i] + d);
    }

    *m_out = m;
    *l_out = l;
    free(s);
    free(rows);
    return ORACLE_OK;
}

static int check_shape(int B, int Hq, int Hkv, int D, int block_size,
                       const int32_t *block_table, int max_blocks, int num_blocks)
{
    if (B < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || block_size <= 0)
        return ORACLE_BAD_ARG;
    if (Hq % Hkv != 0)
        return ORACLE_BAD_ARG;
    if (block_table && (max_blocks <= 0 || num_blocks <= 0))
        return ORACLE_BAD_ARG;
    return ORACLE_OK;
}

/*
 * Normalised attention output, in double, for query rows
 * r in [row_begin, row_end) of the flattened [B, Hq] grid (r = b * Hq + h).
 * out holds (row_end - row_begin) * D doubles.  A request of length 0 yields a
 * zero row (the pages define no output for an empty context; zero is the
 * convention used here).
 */
int oracle_gqa_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                      const int32_t *block_table, const int32_t *seq_lens,
                      int B, int Hq, int Hkv, int D, int block_size,
                      int max_blocks, int num_blocks, double scale,
                      int64_t row_begin, int64_t row_end, double *out)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks, num_blocks);
    if (rc)
        return rc;
    if (row_begin < 0 || row_end > (int64_t)B * Hq || row_begin > row_end)
        return ORACLE_BAD_ARG;
    kv_cache c = {k_cache, v_cache, NULL, NULL, 1.0, 1.0, block_table, Hkv, D, block_size, max_blocks, num_blocks};
    const int G = Hq / Hkv;
    int64_t capacity = block_table ? (int64_t)max_blocks * block_size : block_size;

    for (int64_t r = row_begin; r < row_end; ++r) {
        int b = (int)(r / Hq), h = (int)(r % Hq);
        int kvh = h / G;
        int64_t L = seq_lens[b];
        if (L < 0 || L > capacity)
            return ORACLE_BAD_ARG;
        double m, l;
        double *o = out + (r - row_begin) * D;
        rc = attention_state(&c, q + r * D, scale, b, kvh, 0, L, o, &m, &l);
        if (rc)
            return rc;
        for (int d = 0; d < D; ++d)
            o[d] = l > 0.0 ? o[d] / l : 0.0;
    }
    return ORACLE_OK;
}

/*
 * oracle_gqa_decode over an FP8 E4M3 cache: k8, v8 hold one byte per element
 * (same layouts as the bf16 caches), their values are e4m3(byte) * k_scale and
 * e4m3(byte) * v_scale.  q stays bf16.
 */
int oracle_gqa_decode_fp8(const uint16_t *q, const uint8_t *k8, const uint8_t *v8,
                          double k_scale, double v_scale, const int32_t *block_table,
                          const int32_t *seq_lens, int B, int Hq, int Hkv, int D,
                          int block_size, int max_blocks, int num_blocks, double scale,
                          int64_t row_begin, int64_t row_end, double *out)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks, num_blocks);
    if (rc)
        return rc;
    if (row_begin < 0 || row_end > (int64_t)B * Hq || row_begin > row_end)
        return ORACLE_BAD_ARG;
    kv_cache c = {NULL, NULL, k8, v8, k_scale, v_scale, block_table, Hkv, D, block_size,
                  max_blocks, num_blocks};
    const int G = Hq / Hkv;
    int64_t capacity = block_table ? (int64_t)max_blocks * block_size : block_size;

    for (int64_t r = row_begin; r < row_end; ++r) {
        int b = (int)(r / Hq), kvh = (int)(r % Hq) / G;
        int64_t L = seq_lens[b];
        if (L < 0 || L > capacity)
            return ORACLE_BAD_ARG;
        double m, l;
        double *o = out + (r - row_begin) * D;
        const uint16_t *qrow = q + r * D;
        rc = attention_state(&c, qrow, scale, b, kvh, 0, L, o, &m, &l);
        if (rc)
            return rc;
        for (int d = 0; d < D; ++d)
            o[d] = l > 0.0 ? o[d] / l : 0.0;
    }
    return ORACLE_OK;
}

/*
 * Several query tokens per request (the verification pass of speculative
 * decoding: the large model scores the gamma drafted positions together in one
 * pass; Inference optimization: KV cache, MQA/GQA, batching..., section 5
 * "Speculative decoding").  The drafted tokens' keys and values are already in
 * the cache, so request b holds L_b >= Q tokens and query token i (0 <= i < Q)
 * sits at position L_b - Q + i.  Reading of the pages: each position sees the
 * keys up to and including its own, t <= L_b - Q + i (causal inside the Q new
 * tokens), as in a prefill pass over them.
 *
 * q and out are [B, Q, Hq, D]; rows r in [row_begin, row_end) of the flattened
 * [B, Q, Hq] grid (r = (b * Q + i) * Hq + h).  With Q = 1 this is
 * oracle_gqa_decode.  L_b < Q is an error (ORACLE_BAD_ARG).
 */
int oracle_gqa_decode_multi(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                            const int32_t *block_table, const int32_t *seq_lens,
                            int B, int Q, int Hq, int Hkv, int D, int block_size,
                            int max_blocks, int num_blocks, double scale,
                            int64_t row_begin, int64_t row_end, double *out)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks, num_blocks);
    if (rc)
        return rc;
    if (Q <= 0 || row_begin < 0 || row_end > (int64_t)B * Q * Hq || row_begin > row_end)
        return ORACLE_BAD_ARG;
    kv_cache c = {k_cache, v_cache, NULL, NULL, 1.0, 1.0, block_table, Hkv, D, block_size, max_blocks, num_blocks};
    const int G = Hq / Hkv;
    int64_t capacity = block_table ? (int64_t)max_blocks * block_size : block_size;

    for (int64_t r = row_begin; r < row_end; ++r) {
        int h = (int)(r % Hq);
        int64_t bi = r / Hq;
        int b = (int)(bi / Q), i = (int)(bi % Q);
        int kvh = h / G;
        int64_t L = seq_lens[b];
        if (L < Q || L > capacity)
            return ORACLE_BAD_ARG;
        double m, l;
        double *o = out + (r - row_begin) * D;
        rc = attention_state(&c, q + r * D, scale, b, kvh, 0, L - Q + i + 1, o, &m, &l);
        if (rc)
            return rc;
        for (int d = 0; d < D; ++d)
            o[d] = l > 0.0 ? o[d] / l : 0.0;
    }
    return ORACLE_OK;
}

/*
 * Partial softmax states (acc unnormalised, m, l; natural-log units) for query
 * rows [row_begin, row_end) over the per-request key range
 * [kv_begin[b], kv_end[b]).  acc holds (row_end - row_begin) * D doubles; m and
 * l hold row_end - row_begin doubles each.
 */
int oracle_gqa_decode_states(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                             const int32_t *block_table, const int32_t *kv_begin,
                             const int32_t *kv_end, int B, int Hq, int Hkv, int D,
                             int block_size, int max_blocks, int num_blocks, double scale,
                             int64_t row_begin, int64_t row_end,
                             double *acc, double *m, double *l)
{
    int rc = check_shape(B, Hq, Hkv, D, block_size, block_table, max_blocks, num_blocks);
    if (rc)
        return rc;
    if (row_begin < 0 || row_end > (int64_t)B * Hq || row_begin > row_end)
        return ORACLE_BAD_ARG;
    kv_cache c = {k_cache, v_cache, NULL, NULL, 1.0, 1.0, block_table, Hkv, D, block_size, max_blocks, num_blocks};
    const int G = Hq / Hkv;
    int64_t capacity = block_table ? (int64_t)max_blocks * block_size : block_size;

    for (int64_t r = row_begin; r < row_end; ++r) {
        int b = (int)(r / Hq), h = (int)(r % Hq);
        int64_t t0 = kv_begin[b], t1 = kv_end[b];
        if (t0 < 0 || t1 > capacity)
            return ORACLE_BAD_ARG;
        int64_t i = r - row_begin;
        rc = attention_state(&c, q + r * D, scale, b, h / G, t0, t1, acc + i * D, m + i, l + i);
        if (rc)
            return rc;
    }
    return ORACLE_OK;
}

/*
 * Exact merge of S partial states per row (LeanAttention decode tiles digest,
 * section "Exact softmax that merges piece by piece": every piece carries its
 * own maximum, normaliser and weighted values; rescaling all of them to the
 * common maximum and adding gives the unsplit result, in any order).
 *
 *   m* = max_i m_i,  w_i = exp(m_i - m*)  (0 for an empty piece, m_i = -inf)
 *   l* = sum_i w_i l_i,  out = sum_i w_i acc_i / l*,  lse = m* + log(l*)
 *
 * acc is [S, N, D], m and l are [S, N]; out is [N, D]; lse ([N]) may be NULL.
 * A row whose pieces are all empty gives out = 0 and lse = -inf.
 */
int oracle_merge_states(const double *acc, const double *m, const double *l,
                        int S, int N, int D, double *out, double *lse)
{
    if (S < 0 || N < 0 || D <= 0)
        return ORACLE_BAD_ARG;
    for (int n = 0; n < N; ++n) {
        double mstar = -INFINITY;
        for (int i = 0; i < S; ++i)
            if (m[(int64_t)i * N + n] > mstar)
                mstar = m[(int64_t)i * N + n];
        double lstar = 0.0;
        double *o = out + (int64_t)n * D;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        for (int i = 0; i < S; ++i) {
            double mi = m[(int64_t)i * N + n];
            double w = (mi == -INFINITY) ? 0.0 : exp(mi - mstar);
            lstar += w * l[(int64_t)i * N + n];
            const double *a = acc + ((int64_t)i * N + n) * D;
            for (int d = 0; d < D; ++d)
                o[d] += w * a[d];
        }
        for (int d = 0; d < D; ++d)
            o[d] = lstar > 0.0 ? o[d] / lstar : 0.0;
        if (lse)
            lse[n] = lstar > 0.0 ? mstar + log(lstar) : -INFINITY;
    }
    return ORACLE_OK;
}
