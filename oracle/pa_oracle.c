/*
 * pa_oracle.c -- the oracle: a plain, slow, obviously-correct CPU statement of
 * paged decode attention and of the paged KV-cache write.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may call, link or
 * load this file: only the tests, the smoke check of the entry module and the
 * bench's CPU-baseline leg use it.  It shares no code, header, table or helper
 * with the CUDA library; the two meet only through seeded inputs.
 *
 * Arithmetic is IEEE binary64 throughout, except the one place where a float
 * decides an integer (the INT8 / FP8 quantisation code): there the division
 * x / s is done in binary32 round-to-nearest-even, the kernel's precision, so
 * that both sides take the same decision.
 *
 * Pages cited (by title, then section):
 *   [vllm-musa]  "KV Cache 与 PagedAttention（vllm-musa 实战）" (7yue.com,
 *                MUSA learning center m8-l2)
 *   [KV量化]      "大模型推理优化实战：KV Cache量化与PagedAttention显存管理配置"
 *                (yunthe.com)
 *   [深度解析]     "LLM推理优化：vLLM PagedAttention深度解析与工程实践" (jsqmd.com)
 *   [KVcache-learning] "KVcache-learning" (fairy2021.github.io), chapters s00-s13
 *
 * Readings of points the pages leave open:
 *   R1  attention is ONE softmax over all cached tokens of the sequence
 *       ([深度解析] §二 formula; [KVcache-learning] s05 "传统 Attention 计算");
 *       the per-block "attn += softmax(...)" line of s05 is read as shorthand
 *       for the same result, since paging "does not change the computation"
 *       ([深度解析] §九).
 *   R2  GQA: query head h reads kv head h / (H / H_kv) (contiguous groups).
 *   R3  cache layout [num_blocks, block_size, H_kv, D] for K and for V
 *       ([深度解析] §4.1 comment), scales [num_blocks, H_kv, block_size].
 *   R4  a v2 partition p covers tokens [p*P, min((p+1)*P, len)); an empty
 *       partition has m = -inf, l = 0 and is skipped by the merge.
 *   R5  INT8: symmetric, per token per head, s = absmax / 127, code =
 *       clamp(rne(x / s), -127, 127); all-zero rows have s = 0, codes 0.
 *   R6  FP8: OCP E4M3 (1-4-3, bias 7, max 448, S.1111.111 = NaN),
 *       s = absmax / 448, code = e4m3(x / s) with round-to-nearest-even and
 *       saturation to +-448 ([KVcache-learning] s09 gives E4M3 and +-448);
 *       an all-zero row has s = 0 and codes 0.
 *   R7  a slot < 0 in slot_mapping means "no write".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ORC_F64 exists only so tests can hand the oracle already-dequantised caches. */
enum { ORC_F32 = 0, ORC_F16 = 1, ORC_BF16 = 2, ORC_INT8 = 3, ORC_FP8E4M3 = 4, ORC_F64 = 5 };
enum { ORC_OK = 0, ORC_ERR_ARG = 1, ORC_ERR_RANGE = 2, ORC_ERR_NOMEM = 3 };

/* ------------------------------------------------------------------------ */
/* Storage formats -> value.  Written from the format definitions.           */
/* ------------------------------------------------------------------------ */

/* IEEE 754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits. */
double orc_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);               /* subnormal: f * 2^-24 */
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);   /* (1.f) * 2^(e-15) */
    return sign ? -v : v;
}

/* bfloat16 is the upper half of an IEEE binary32. */
double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP 8-bit floating point, E4M3: 1 sign, 4 exponent (bias 7), 3 mantissa.
 * No infinities; S.1111.111 is NaN; largest finite 1.75 * 2^8 = 448. */
double orc_e4m3_to_double(uint8_t c)
{
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 0xf;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);                /* subnormal: m/8 * 2^-6 */
    else
        v = ldexp((double)(8 + m), e - 10);      /* (1.m) * 2^(e-7) */
    return sign ? -v : v;
}

/* Round a non-negative double to the nearest integer, ties to even. */
static double round_half_even(double y)
{
    double r = floor(y);
    double frac = y - r;
    if (frac > 0.5)
        return r + 1.0;
    if (frac < 0.5)
        return r;
    return (fmod(r, 2.0) == 0.0) ? r : r + 1.0;
}

/* binary32 -> E4M3, round-to-nearest-even, saturating to +-448 (R6).
 * NaN maps to the NaN code with the input's sign. */
uint8_t orc_e4m3_from_float(float v)
{
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (isnan(v))
        return (uint8_t)(sign | 0x7f);
    if (a >= 448.0)
        return (uint8_t)(sign | 0x7e);           /* satfinite */
    /* Values below 2^-6 use the subnormal quantum 2^-9; a value in
     * [2^E, 2^(E+1)) with E >= -6 uses the quantum 2^(E-3). */
    int E = -6;
    while (E < 8 && a >= ldexp(1.0, E + 1))
        E++;
    double quantum = (a < ldexp(1.0, -6)) ? ldexp(1.0, -9) : ldexp(1.0, E - 3);
    double n = round_half_even(a / quantum);     /* exact power-of-2 scaling */
    double r = n * quantum;                      /* rounded magnitude */
    if (r >= 448.0)
        return (uint8_t)(sign | 0x7e);
    if (r < ldexp(1.0, -6)) {                    /* subnormal (or zero) */
        return (uint8_t)(sign | (uint8_t)(r / ldexp(1.0, -9)));
    }
    /* normal: find the exponent of the rounded value (rounding may carry) */
    int Er = -6;
    while (Er < 8 && r >= ldexp(1.0, Er + 1))
        Er++;
    int mant = (int)(r / ldexp(1.0, Er - 3)) - 8;
    return (uint8_t)(sign | ((Er + 7) << 3) | mant);
}

/* ------------------------------------------------------------------------ */
/* Per-token-per-head quantisation (R5, R6).                                 */
/* ------------------------------------------------------------------------ */

/* binary32 round-to-nearest-even of a float of modest magnitude. */
static float rne_f32(float y)
{
    float r = floorf(y);
    float frac = y - r;                          /* exact for |y| < 2^23 */
    if (frac > 0.5f)
        return r + 1.0f;
    if (frac < 0.5f)
        return r;
    return (fmodf(r, 2.0f) == 0.0f) ? r : r + 1.0f;
}

static float absmax_f32(const float* x, int n)
{
    float a = 0.0f;
    for (int i = 0; i < n; ++i) {
        float v = fabsf(x[i]);
        if (v > a)
            a = v;
    }
    return a;
}

/* INT8 row: returns the scale, writes n codes. */
float orc_quant_int8_row(const float* x, int n, int8_t* codes)
{
    float s = absmax_f32(x, n) / 127.0f;         /* binary32 division */
    for (int i = 0; i < n; ++i) {
        if (s == 0.0f) {
            codes[i] = 0;
            continue;
        }
        float y = x[i] / s;                      /* binary32 division */
        float r = (y < 0.0f) ? -rne_f32(-y) : rne_f32(y);
        if (r > 127.0f)
            r = 127.0f;
        if (r < -127.0f)
            r = -127.0f;
        codes[i] = (int8_t)r;
    }
    return s;
}

/* FP8 E4M3 row: returns the scale, writes n codes. */
float orc_quant_fp8_row(const float* x, int n, uint8_t* codes)
{
    float s = absmax_f32(x, n) / 448.0f;         /* binary32 division */
    for (int i = 0; i < n; ++i) {
        if (s == 0.0f) {
            codes[i] = 0;                        /* all-zero row (R6) */
            continue;
        }
        codes[i] = orc_e4m3_from_float(x[i] / s);  /* binary32 division */
    }
    return s;
}

/* ------------------------------------------------------------------------ */
/* Element access.                                                           */
/* ------------------------------------------------------------------------ */

static double load_value(const void* base, int dtype, size_t i)
{
    switch (dtype) {
    case ORC_F32: return (double)((const float*)base)[i];
    case ORC_F16: return orc_f16_to_double(((const uint16_t*)base)[i]);
    case ORC_BF16: return orc_bf16_to_double(((const uint16_t*)base)[i]);
    case ORC_INT8: return (double)((const int8_t*)base)[i];
    case ORC_FP8E4M3: return orc_e4m3_to_double(((const uint8_t*)base)[i]);
    case ORC_F64: return ((const double*)base)[i];
    }
    return NAN;
}

static int elem_bytes(int dtype)
{
    return (dtype == ORC_F64) ? 8 : (dtype == ORC_F32) ? 4
         : (dtype == ORC_F16 || dtype == ORC_BF16) ? 2 : 1;
}

static int is_quantised(int dtype) { return dtype == ORC_INT8 || dtype == ORC_FP8E4M3; }

/* The value of cache element (block, offset, head, d): a stored float, or for
 * a quantised cache the code times its per-token-per-head scale (R3, R5, R6). */
static double cache_value(const void* cache, const float* scales, int dtype,
                          int64_t block, int offset, int head, int d,
                          int bs, int Hkv, int D)
{
    size_t idx = (((size_t)block * bs + offset) * Hkv + head) * D + d;
    double v = load_value(cache, dtype, idx);
    if (is_quantised(dtype)) {
        size_t sidx = ((size_t)block * Hkv + head) * bs + offset;
        v *= (double)scales[sidx];
    }
    return v;
}

/* ------------------------------------------------------------------------ */
/* KV-size arithmetic ([vllm-musa] §一; [深度解析] §二; [KVcache-learning] s11). */
/* ------------------------------------------------------------------------ */

/* Bytes of K and V one token occupies over all layers: 2 * L * H_kv * D * b. */
double orc_kv_bytes_per_token(int num_layers, int num_kv_heads, int head_dim,
                              int dtype_bytes)
{
    return 2.0 * num_layers * num_kv_heads * head_dim * dtype_bytes;
}

/* ------------------------------------------------------------------------ */
/* Contiguous attention for one sequence ([深度解析] §二; [KVcache-learning] s01, */
/* s05 "传统 Attention 计算").  k, v: [T, H_kv, D]; q, out: [H, D].            */
/* ------------------------------------------------------------------------ */
int orc_attention_contiguous(double* out, const double* q, const double* k,
                             const double* v, int T, int H, int Hkv, int D,
                             double scale)
{
    if (H <= 0 || Hkv <= 0 || D <= 0 || T < 0 || H % Hkv != 0)
        return ORC_ERR_ARG;
    int G = H / Hkv;
    double* x = (double*)malloc(sizeof(double) * (T > 0 ? T : 1));
    if (!x)
        return ORC_ERR_NOMEM;
    for (int h = 0; h < H; ++h) {
        int kvh = h / G;                         /* R2 */
        double* o = out + (size_t)h * D;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        if (T == 0)
            continue;
        double m = -INFINITY;
        for (int t = 0; t < T; ++t) {
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += q[(size_t)h * D + d] * k[((size_t)t * Hkv + kvh) * D + d];
            x[t] = scale * dot;
            if (x[t] > m)
                m = x[t];
        }
        double denom = 0.0;
        for (int t = 0; t < T; ++t) {
            double w = exp(x[t] - m);
            denom += w;
            for (int d = 0; d < D; ++d)
                o[d] += w * v[((size_t)t * Hkv + kvh) * D + d];
        }
        for (int d = 0; d < D; ++d)
            o[d] /= denom;
    }
    free(x);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Paged decode attention ([vllm-musa] §五 kernel entry: out, q, k_cache,    */
/* v_cache, block_tables, seq_lens, block_size, num_kv_heads, scale; token t */
/* of sequence s lives in physical block block_tables[s][t / bs] at offset   */
/* t % bs -- [vllm-musa] §五, [深度解析] §3.1 Block Table).                   */
/* q: storage dtype q_dtype, [S, H, D]; out: binary64 [S, H, D].             */
/* ------------------------------------------------------------------------ */

static int check_tables(const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                        int num_seqs, int bs, int num_blocks)
{
    for (int s = 0; s < num_seqs; ++s) {
        int len = seq_lens[s];
        if (len < 0 || (int64_t)len > (int64_t)max_blocks * bs)
            return ORC_ERR_RANGE;
        int nb = (len + bs - 1) / bs;
        for (int i = 0; i < nb; ++i) {
            int32_t b = block_tables[(size_t)s * max_blocks + i];
            if (b < 0 || b >= num_blocks)
                return ORC_ERR_RANGE;
        }
    }
    return ORC_OK;
}

/* Logits x_t = scale * q[s,h,:] . K_t for t in [t0, t1).  */
static void paged_logits(double* x, const void* q, int q_dtype, const void* k_cache,
                         const float* k_scale, int cache_dtype, const int32_t* table,
                         int s, int h, int kvh, int t0, int t1, int H, int Hkv, int D,
                         int bs, double scale)
{
    for (int t = t0; t < t1; ++t) {
        int64_t block = table[t / bs];
        int off = t % bs;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) {
            double qv = load_value(q, q_dtype, ((size_t)s * H + h) * D + d);
            double kv = cache_value(k_cache, k_scale, cache_dtype, block, off, kvh, d, bs, Hkv, D);
            dot += qv * kv;
        }
        x[t - t0] = scale * dot;
    }
}

int orc_paged_decode(double* out, const void* q, int q_dtype,
                     const void* k_cache, const void* v_cache, int cache_dtype,
                     const float* k_scale, const float* v_scale,
                     const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                     int num_seqs, int H, int Hkv, int D, int bs, int num_blocks,
                     double scale)
{
    if (H <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || H % Hkv != 0)
        return ORC_ERR_ARG;
    if (is_quantised(cache_dtype) && (!k_scale || !v_scale))
        return ORC_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, seq_lens, num_seqs, bs, num_blocks);
    if (rc != ORC_OK)
        return rc;
    int G = H / Hkv;
    for (int s = 0; s < num_seqs; ++s) {
        int len = seq_lens[s];
        const int32_t* table = block_tables + (size_t)s * max_blocks;
        double* x = (double*)malloc(sizeof(double) * (len > 0 ? len : 1));
        if (!x)
            return ORC_ERR_NOMEM;
        for (int h = 0; h < H; ++h) {
            int kvh = h / G;                     /* R2 */
            double* o = out + ((size_t)s * H + h) * D;
            for (int d = 0; d < D; ++d)
                o[d] = 0.0;
            if (len == 0)
                continue;                        /* empty context: output 0 */
            paged_logits(x, q, q_dtype, k_cache, k_scale, cache_dtype, table,
                         s, h, kvh, 0, len, H, Hkv, D, bs, scale);
            double m = -INFINITY;
            for (int t = 0; t < len; ++t)
                if (x[t] > m)
                    m = x[t];
            double denom = 0.0;
            for (int t = 0; t < len; ++t) {
                double w = exp(x[t] - m);
                denom += w;
                int64_t block = table[t / bs];
                for (int d = 0; d < D; ++d)
                    o[d] += w * cache_value(v_cache, v_scale, cache_dtype, block, t % bs,
                                            kvh, d, bs, Hkv, D);
            }
            for (int d = 0; d < D; ++d)
                o[d] /= denom;
        }
        free(x);
    }
    return ORC_OK;
}

/* The same attention for chosen (sequence, head) pairs only, so full-size
 * problems can be checked on sampled outputs.  pairs: int32 [n, 2] = (s, h);
 * out: binary64 [n, D]. */
int orc_paged_decode_pairs(double* out, const int32_t* pairs, int npairs,
                           const void* q, int q_dtype,
                           const void* k_cache, const void* v_cache, int cache_dtype,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                           int num_seqs, int H, int Hkv, int D, int bs, int num_blocks,
                           double scale)
{
    if (H <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || H % Hkv != 0)
        return ORC_ERR_ARG;
    if (is_quantised(cache_dtype) && (!k_scale || !v_scale))
        return ORC_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, seq_lens, num_seqs, bs, num_blocks);
    if (rc != ORC_OK)
        return rc;
    int G = H / Hkv;
    for (int i = 0; i < npairs; ++i) {
        int s = pairs[2 * i], h = pairs[2 * i + 1];
        if (s < 0 || s >= num_seqs || h < 0 || h >= H)
            return ORC_ERR_ARG;
        int len = seq_lens[s];
        const int32_t* table = block_tables + (size_t)s * max_blocks;
        int kvh = h / G;
        double* o = out + (size_t)i * D;
        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        if (len == 0)
            continue;
        double* x = (double*)malloc(sizeof(double) * len);
        if (!x)
            return ORC_ERR_NOMEM;
        paged_logits(x, q, q_dtype, k_cache, k_scale, cache_dtype, table,
                     s, h, kvh, 0, len, H, Hkv, D, bs, scale);
        double m = -INFINITY;
        for (int t = 0; t < len; ++t)
            if (x[t] > m)
                m = x[t];
        double denom = 0.0;
        for (int t = 0; t < len; ++t) {
            double w = exp(x[t] - m);
            denom += w;
            int64_t block = table[t / bs];
            for (int d = 0; d < D; ++d)
                o[d] += w * cache_value(v_cache, v_scale, cache_dtype, block, t % bs,
                                        kvh, d, bs, Hkv, D);
        }
        for (int d = 0; d < D; ++d)
            o[d] /= denom;
        free(x);
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* v2: split-K partitions, then a log-sum-exp merge ([深度解析] §4.1,         */
/* paged_attention_v2 "先 partial accumulate，再 merge"; R4).                 */
/* tmp_out [S, H, maxp, D] = o_p (already divided by l_p); max_logits and     */
/* exp_sums [S, H, maxp] = m_p, l_p = sum exp(x - m_p).                      */
/* ------------------------------------------------------------------------ */
int orc_paged_decode_partition(double* tmp_out, double* max_logits, double* exp_sums,
                               const void* q, int q_dtype,
                               const void* k_cache, const void* v_cache, int cache_dtype,
                               const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, int max_blocks,
                               const int32_t* seq_lens, int num_seqs, int H, int Hkv, int D,
                               int bs, int num_blocks, double scale,
                               int partition_size, int max_parts)
{
    if (H <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || H % Hkv != 0 || partition_size <= 0)
        return ORC_ERR_ARG;
    if (is_quantised(cache_dtype) && (!k_scale || !v_scale))
        return ORC_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, seq_lens, num_seqs, bs, num_blocks);
    if (rc != ORC_OK)
        return rc;
    int G = H / Hkv;
    double* x = (double*)malloc(sizeof(double) * partition_size);
    if (!x)
        return ORC_ERR_NOMEM;
    for (int s = 0; s < num_seqs; ++s) {
        int len = seq_lens[s];
        if ((len + partition_size - 1) / partition_size > max_parts) {
            free(x);
            return ORC_ERR_RANGE;
        }
        const int32_t* table = block_tables + (size_t)s * max_blocks;
        for (int h = 0; h < H; ++h) {
            int kvh = h / G;
            for (int p = 0; p < max_parts; ++p) {
                size_t ml = ((size_t)s * H + h) * max_parts + p;
                double* o = tmp_out + ml * D;
                int t0 = p * partition_size;
                int t1 = t0 + partition_size < len ? t0 + partition_size : len;
                for (int d = 0; d < D; ++d)
                    o[d] = 0.0;
                if (t0 >= t1) {                  /* empty partition (R4) */
                    max_logits[ml] = -INFINITY;
                    exp_sums[ml] = 0.0;
                    continue;
                }
                paged_logits(x, q, q_dtype, k_cache, k_scale, cache_dtype, table,
                             s, h, kvh, t0, t1, H, Hkv, D, bs, scale);
                double m = -INFINITY;
                for (int t = t0; t < t1; ++t)
                    if (x[t - t0] > m)
                        m = x[t - t0];
                double l = 0.0;
                for (int t = t0; t < t1; ++t) {
                    double w = exp(x[t - t0] - m);
                    l += w;
                    int64_t block = table[t / bs];
                    for (int d = 0; d < D; ++d)
                        o[d] += w * cache_value(v_cache, v_scale, cache_dtype, block, t % bs,
                                                kvh, d, bs, Hkv, D);
                }
                for (int d = 0; d < D; ++d)
                    o[d] /= l;
                max_logits[ml] = m;
                exp_sums[ml] = l;
            }
        }
    }
    free(x);
    return ORC_OK;
}

/* Merge: M = max_p m_p over non-empty partitions, w_p = l_p * exp(m_p - M),
 * out = sum_p w_p o_p / sum_p w_p.  A sequence with no tokens gives 0. */
int orc_merge(double* out, const double* tmp_out, const double* max_logits,
              const double* exp_sums, const int32_t* seq_lens, int num_seqs, int H, int D,
              int partition_size, int max_parts)
{
    if (H <= 0 || D <= 0 || partition_size <= 0)
        return ORC_ERR_ARG;
    for (int s = 0; s < num_seqs; ++s) {
        int len = seq_lens[s];
        int np = (len + partition_size - 1) / partition_size;
        if (np > max_parts)
            return ORC_ERR_RANGE;
        for (int h = 0; h < H; ++h) {
            size_t base = ((size_t)s * H + h) * max_parts;
            double* o = out + ((size_t)s * H + h) * D;
            for (int d = 0; d < D; ++d)
                o[d] = 0.0;
            double M = -INFINITY;
            for (int p = 0; p < np; ++p)
                if (exp_sums[base + p] > 0.0 && max_logits[base + p] > M)
                    M = max_logits[base + p];
            if (M == -INFINITY)
                continue;
            double W = 0.0;
            for (int p = 0; p < np; ++p) {
                if (exp_sums[base + p] <= 0.0)
                    continue;
                double w = exp_sums[base + p] * exp(max_logits[base + p] - M);
                W += w;
                for (int d = 0; d < D; ++d)
                    o[d] += w * tmp_out[(base + p) * D + d];
            }
            for (int d = 0; d < D; ++d)
                o[d] /= W;
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Cache write: each new token's K and V row goes to slot                    */
/* slot_mapping[i] = block * bs + offset ([KV量化] BlockManager.append_token; */
/* [KVcache-learning] s06 allocate_token_block), optionally quantised.       */
/* key, value: storage dtype src_dtype, [num_tokens, H_kv, D].               */
/* ------------------------------------------------------------------------ */
int orc_reshape_and_cache(const void* key, const void* value, int src_dtype,
                          void* k_cache, void* v_cache, int cache_dtype,
                          float* k_scale, float* v_scale, const int64_t* slot_mapping,
                          int num_tokens, int Hkv, int D, int bs, int num_blocks)
{
    if (Hkv <= 0 || D <= 0 || bs <= 0 || num_tokens < 0)
        return ORC_ERR_ARG;
    int quant = is_quantised(cache_dtype);
    if (!quant && cache_dtype != src_dtype)
        return ORC_ERR_ARG;
    if (quant && (src_dtype == ORC_INT8 || src_dtype == ORC_FP8E4M3 || !k_scale || !v_scale))
        return ORC_ERR_ARG;
    for (int i = 0; i < num_tokens; ++i)
        if (slot_mapping[i] >= (int64_t)num_blocks * bs)
            return ORC_ERR_RANGE;
    int eb = elem_bytes(src_dtype);
    float* row = (float*)malloc(sizeof(float) * D);
    if (!row)
        return ORC_ERR_NOMEM;
    for (int i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;                            /* R7 */
        int64_t block = slot / bs;
        int off = (int)(slot % bs);
        for (int h = 0; h < Hkv; ++h) {
            for (int kv = 0; kv < 2; ++kv) {
                const void* src = kv == 0 ? key : value;
                void* dst = kv == 0 ? k_cache : v_cache;
                float* sc = kv == 0 ? k_scale : v_scale;
                size_t src_row = ((size_t)i * Hkv + h) * D;
                size_t dst_row = (((size_t)block * bs + off) * Hkv + h) * D;
                if (!quant) {
                    memcpy((char*)dst + dst_row * eb, (const char*)src + src_row * eb,
                           (size_t)D * eb);
                    continue;
                }
                for (int d = 0; d < D; ++d)      /* exact: every source value is a float */
                    row[d] = (float)load_value(src, src_dtype, src_row + d);
                size_t sidx = ((size_t)block * Hkv + h) * bs + off;
                if (cache_dtype == ORC_INT8)
                    sc[sidx] = orc_quant_int8_row(row, D, (int8_t*)dst + dst_row);
                else
                    sc[sidx] = orc_quant_fp8_row(row, D, (uint8_t*)dst + dst_row);
            }
        }
    }
    free(row);
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Block copy: copy-on-write of a shared block ([KVcache-learning] s05,      */
/* "写时复制": the writer gets its own copy of the block and its table is    */
/* repointed) and swap between GPU and CPU block pools ([KVcache-learning]   */
/* s06 swap_out / swap_in; [KV量化] swap_space).  For each pair p of         */
/* block_mapping ([num_pairs, 2] = (src id, dst id)), every token row of the */
/* source block (K and V, and the K/V scales of a quantised cache) is copied */
/* to the destination block.  Source and destination pools may be the same   */
/* arrays (copy-on-write) or different ones (swap).  Readings: destination   */
/* ids are distinct, and when the pools are the same arrays no destination   */
/* is also a source in the same call, so the result does not depend on the  */
/* order of the pairs; a call that breaks this is rejected.                  */
/* ------------------------------------------------------------------------ */
int orc_copy_blocks(const void* src_k, const void* src_v, const float* src_ks,
                    const float* src_vs, int src_num_blocks,
                    void* dst_k, void* dst_v, float* dst_ks, float* dst_vs, int dst_num_blocks,
                    int cache_dtype, const int64_t* block_mapping, int num_pairs,
                    int Hkv, int D, int bs)
{
    if (Hkv <= 0 || D <= 0 || bs <= 0 || num_pairs < 0 || cache_dtype == ORC_F64)
        return ORC_ERR_ARG;
    int quant = is_quantised(cache_dtype);
    if (quant && (!src_ks || !src_vs || !dst_ks || !dst_vs))
        return ORC_ERR_ARG;
    int same_pool = (const void*)dst_k == src_k;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t s = block_mapping[2 * p], d = block_mapping[2 * p + 1];
        if (s < 0 || s >= src_num_blocks || d < 0 || d >= dst_num_blocks)
            return ORC_ERR_RANGE;
        for (int q = 0; q < num_pairs; ++q) {
            if (q != p && block_mapping[2 * q + 1] == d)
                return ORC_ERR_ARG;              /* two writes to one block */
            if (same_pool && block_mapping[2 * q] == d)
                return ORC_ERR_ARG;              /* a destination that is also read */
        }
    }
    size_t eb = (size_t)elem_bytes(cache_dtype);
    for (int p = 0; p < num_pairs; ++p) {
        int64_t s = block_mapping[2 * p], d = block_mapping[2 * p + 1];
        for (int t = 0; t < bs; ++t) {
            for (int h = 0; h < Hkv; ++h) {
                size_t srow = (((size_t)s * bs + t) * Hkv + h) * D;
                size_t drow = (((size_t)d * bs + t) * Hkv + h) * D;
                memcpy((char*)dst_k + drow * eb, (const char*)src_k + srow * eb, D * eb);
                memcpy((char*)dst_v + drow * eb, (const char*)src_v + srow * eb, D * eb);
                if (quant) {
                    dst_ks[((size_t)d * Hkv + h) * bs + t] = src_ks[((size_t)s * Hkv + h) * bs + t];
                    dst_vs[((size_t)d * Hkv + h) * bs + t] = src_vs[((size_t)s * Hkv + h) * bs + t];
                }
            }
        }
    }
    return ORC_OK;
}

/* ------------------------------------------------------------------------ */
/* Multi-token query over the paged cache: a chunk of new tokens per          */
/* sequence attends to the cached prefix and, causally, to itself.  With      */
/* prefix caching a sequence whose first blocks are shared only computes its  */
/* remaining tokens ([深度解析] §4.2; [KVcache-learning] s08: the second     */
/* request only computes its few new tokens).  The chunk's K/V are in the     */
/* cache already (written by the cache write), so query row r of sequence s,  */
/* at absolute position pos = seq_len - q_len + r, is the decode of one query */
/* over the first pos + 1 cached tokens.                                      */
/*   q, out: [total_q, H, D], rows of sequence s at                           */
/*   [query_start[s], query_start[s + 1]);  0 <= q_len <= seq_len.            */
/* ------------------------------------------------------------------------ */
static int attend_row(double* o, const void* q, int q_dtype, size_t q_row,
                      const void* k_cache, const void* v_cache, int cache_dtype,
                      const float* k_scale, const float* v_scale, const int32_t* table,
                      int n, int h, int kvh, int H, int Hkv, int D, int bs, double scale)
{
    for (int d = 0; d < D; ++d)
        o[d] = 0.0;
    if (n == 0)
        return ORC_OK;
    double* x = (double*)malloc(sizeof(double) * n);
    if (!x)
        return ORC_ERR_NOMEM;
    for (int t = 0; t < n; ++t) {
        int64_t block = table[t / bs];
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += load_value(q, q_dtype, (q_row * H + h) * D + d) *
                   cache_value(k_cache, k_scale, cache_dtype, block, t % bs, kvh, d, bs, Hkv, D);
        x[t] = scale * dot;
    }
    double m = -INFINITY;
    for (int t = 0; t < n; ++t)
        if (x[t] > m)
            m = x[t];
    double denom = 0.0;
    for (int t = 0; t < n; ++t) {
        double w = exp(x[t] - m);
        denom += w;
        int64_t block = table[t / bs];
        for (int d = 0; d < D; ++d)
            o[d] += w * cache_value(v_cache, v_scale, cache_dtype, block, t % bs, kvh, d, bs,
                                    Hkv, D);
    }
    for (int d = 0; d < D; ++d)
        o[d] /= denom;
    free(x);
    return ORC_OK;
}

int orc_paged_prefill(double* out, const void* q, int q_dtype, const int32_t* query_start,
                      const void* k_cache, const void* v_cache, int cache_dtype,
                      const float* k_scale, const float* v_scale,
                      const int32_t* block_tables, int max_blocks, const int32_t* seq_lens,
                      int num_seqs, int H, int Hkv, int D, int bs, int num_blocks,
                      double scale)
{
    if (H <= 0 || Hkv <= 0 || D <= 0 || bs <= 0 || H % Hkv != 0 || query_start[0] != 0)
        return ORC_ERR_ARG;
    if (is_quantised(cache_dtype) && (!k_scale || !v_scale))
        return ORC_ERR_ARG;
    int rc = check_tables(block_tables, max_blocks, seq_lens, num_seqs, bs, num_blocks);
    if (rc != ORC_OK)
        return rc;
    int G = H / Hkv;
    for (int s = 0; s < num_seqs; ++s) {
        int qlen = query_start[s + 1] - query_start[s];
        if (qlen < 0 || qlen > seq_lens[s])
            return ORC_ERR_ARG;
        const int32_t* table = block_tables + (size_t)s * max_blocks;
        for (int r = 0; r < qlen; ++r) {
            size_t row = (size_t)query_start[s] + r;
            int pos = seq_lens[s] - qlen + r;    /* absolute position of this query */
            for (int h = 0; h < H; ++h) {
                rc = attend_row(out + (row * H + h) * D, q, q_dtype, row, k_cache, v_cache,
                                cache_dtype, k_scale, v_scale, table, pos + 1, h, h / G, H,
                                Hkv, D, bs, scale);
                if (rc != ORC_OK)
                    return rc;
            }
        }
    }
    return ORC_OK;
}
