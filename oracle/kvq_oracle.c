/*
 * kvq_oracle.c -- plain, slow, obviously correct CPU oracle for attention over
 * a block-quantized KV cache (Q8_0 keys, Q4_0 values).
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark load this library.  It shares no code, header,
 * table or helper with the CUDA library; the two are written independently
 * from the same definitions.
 *
 * Sources (web pages on quantized KV caches at long context):
 *  [OSCAR2]  "OSCAR2 KV Cache benchmark" (molayo1419.me), "Compression Ratios"
 *            table: q8_0 costs 136 bytes per 128 elements (8.5 bits/elem);
 *            "Known Issues Fixed": the softmax max must be taken over the
 *            complete KQ scores, not over partial sums.
 *  [ROCM]    "Adaptive KV streaming lands on ROCm: Qwen3.8-27B at full 262k
 *            context ..." (richland.au), "Why it matters": Q8_0 K / Q4_0 V
 *            costs 26,624 bytes per token over 16 attention layers.
 *  [RX9070]  "Qwen 27B (IQ4_XS, Q8/Q4 KV) ... 262k context" (molayo1419.me),
 *            list of improvements, "Online Log-Sum-Exp prefill & pipelined
 *            prefetch": chunked prefill over streamed pages with online LSE
 *            accumulation; speculative-decoding paragraph: paged decode
 *            attention extended to the verify batch.
 *  [GUIDE]   "Context window and KV cache" (localaiforum.com), "Formula" and
 *            "GQA" sections: bytes/token = 2 x layers x kv_heads x head_dim x
 *            bytes/elem; a few KV heads serve many query heads.
 *
 * The pages print no bit layout and no formula for the quantizers or the
 * merge.  The readings taken here (all llama.cpp-style, the plainest ones the
 * pages support):
 *  - Q8_0 block (34 B): fp16 d (little-endian) then 32 int8 q.  In fp32, with
 *    no fused multiply-add: amax = max|x|; d = amax/127; id = d ? 1/d : 0;
 *    q = roundf(x*id) (ties away from zero).  Only fp16(d) is stored.
 *  - Q4_0 block (18 B): fp16 d then 16 bytes; byte j holds element j in the
 *    low nibble and element j+16 in the high nibble.  m = the signed value of
 *    the first element of largest |x|; d = m/-8; id = d ? 1/d : 0;
 *    u = min(15, trunc(x*id + 8.5)) with the product and the sum each rounded
 *    to fp32.  Dequant: d*(u-8).
 *  - OSCAR2 block (36 B per 128 elements; [OSCAR2] Compression Ratios table:
 *    2.25 bits per element, INT2 codes with fp16 zero-point metadata): fp16 d,
 *    fp16 m (the zero-point: the value code 0 decodes to), then 32 bytes;
 *    byte j holds the 2-bit codes of elements j, j+32, j+64, j+96 in bits
 *    0-1, 2-3, 4-5, 6-7.  In fp32, no fused multiply-add: mn = min x,
 *    mx = max x; d = (mx - mn)/3; id = d ? 1/d : 0;
 *    u = min(3, trunc((x - mn)*id + 0.5)), each operation rounded to fp32.
 *    fp16(d) and fp16(mn) are stored.  Dequant: d*u + m.  The page's Hadamard
 *    rotation is baked into the model weights offline ("Rotation Model
 *    Conversion"), so rows arrive rotated and nothing here rotates them.
 *  - fp32 -> fp16 is IEEE round-to-nearest-even with subnormals.
 *  - Attention (fp64): s_j = scale * sum_i q_i * k^_ij; m = max_j s_j;
 *    l = sum_j exp(s_j - m); o = sum_j exp(s_j - m) v^_j / l; lse = m + ln l.
 *    An empty key set gives o = 0, lse = -inf.  Query head g reads KV head
 *    g / (n_q_heads / n_kv_heads) (contiguous groups).
 *  - Decode causality: with n_kv keys after the T new rows are appended,
 *    query token t sees keys j <= n_kv - T + t.
 *  - Prefill causality: query token t sees keys j <= n_cached + t.
 *  - Merge of partials: lse = M + ln sum_c exp(lse_c - M), M = max_c lse_c;
 *    o = sum_c exp(lse_c - lse) o_c; partials with lse = -inf are skipped.
 *
 * Cache layout of one layer (the interface both sides implement):
 *   K: [n_kv_heads][capacity][head_dim/32] Q8_0 blocks (34 B each)
 *   V: [n_kv_heads][capacity][head_dim/32] Q4_0 blocks (18 B each)
 * The pages' main configuration.  Each tensor may also use another format
 * (q8_0/q8_0 and q4_0/q4_0 caches are the other choices of the KV-cache
 * guide's levers section; oscar2 is [OSCAR2]'s INT2 format): the cache
 * functions take the block format of K and of V (FMT_Q8_0, FMT_Q4_0 or
 * FMT_OSCAR2), and a head-row is head_dim / (elements per block) blocks of it.
 *
 * Build: gcc -std=c11 -O2 -fopenmp -ffp-contract=off -fPIC -shared.
 * Floating-point contraction must stay off: the quantizers are defined as a
 * sequence of separately rounded fp32 operations.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define QK 32
#define Q8_0_BYTES 34
#define Q4_0_BYTES 18
#define QK_OSCAR2 128
#define OSCAR2_BYTES 36
#define FMT_Q8_0 1
#define FMT_Q4_0 2
#define FMT_OSCAR2 3

/* ------------------------------------------------------------------------ */
/* fp16 <-> fp32, written from the IEEE 754 binary16 definition.            */
/* ------------------------------------------------------------------------ */

static uint16_t f32_to_f16(float f)
{
    uint32_t x;
    memcpy(&x, &f, 4);
    uint32_t sign = (x >> 16) & 0x8000u;
    uint32_t exp = (x >> 23) & 0xffu;
    uint32_t man = x & 0x7fffffu;
    if (exp == 0xffu) /* inf stays inf, NaN becomes the canonical quiet NaN */
        return (uint16_t)(sign | (man ? 0x7e00u : 0x7c00u));
    int e = (int)exp - 127 + 15; /* binary16 biased exponent */
    if (e >= 31)
        return (uint16_t)(sign | 0x7c00u);
    if (e >= 1) {
        /* normal: keep 10 mantissa bits, round the 13 dropped ones to even */
        uint32_t h = sign | ((uint32_t)e << 10) | (man >> 13);
        uint32_t rem = man & 0x1fffu;
        if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))
            h += 1u; /* a carry into the exponent is the correct result */
        return (uint16_t)h;
    }
    if (exp == 0)
        return (uint16_t)sign; /* fp32 zero or subnormal: far below 2^-25 */
    /* binary16 subnormal: value = m * 2^(exp-150) in units of 2^-24 */
    uint32_t m = man | 0x800000u;
    int shift = 14 - e; /* 14 .. */
    if (shift >= 25)
        return (uint16_t)sign; /* below half of the smallest subnormal */
    uint32_t q = m >> shift;
    uint32_t rem = m & ((1u << shift) - 1u);
    uint32_t half = 1u << (shift - 1);
    if (rem > half || (rem == half && (q & 1u)))
        q += 1u;
    return (uint16_t)(sign | q);
}

static double f16_to_f64(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (exp == 0)
        v = ldexp((double)man, -24);
    else if (exp == 31)
        v = man ? NAN : INFINITY;
    else
        v = ldexp((double)(man | 0x400), exp - 25);
    return sign ? -v : v;
}

void orc_f32_to_f16(const float *x, uint16_t *h, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        h[i] = f32_to_f16(x[i]);
}

void orc_f16_to_f64(const uint16_t *h, double *x, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        x[i] = f16_to_f64(h[i]);
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* Quantizers: one 32-element block at a time, separately rounded fp32 ops. */
/* ------------------------------------------------------------------------ */

static void quant_block_q8_0(const float *x, uint8_t *b)
{
    float amax = 0.0f;
    for (int i = 0; i < QK; ++i) {
        float a = fabsf(x[i]);
        if (a > amax)
            amax = a;
    }
    float d = amax / 127.0f;
    float id = (d != 0.0f) ? 1.0f / d : 0.0f;
    uint16_t dh = f32_to_f16(d);
    b[0] = (uint8_t)(dh & 0xff);
    b[1] = (uint8_t)(dh >> 8);
    for (int i = 0; i < QK; ++i) {
        float p = x[i] * id;
        b[2 + i] = (uint8_t)(int8_t)roundf(p);
    }
}

static void quant_block_q4_0(const float *x, uint8_t *b)
{
    float amax = 0.0f, m = 0.0f;
    for (int i = 0; i < QK; ++i) {
        float a = fabsf(x[i]);
        if (a > amax) { /* strict: the first largest element wins */
            amax = a;
            m = x[i];
        }
    }
    float d = m / -8.0f;
    float id = (d != 0.0f) ? 1.0f / d : 0.0f;
    uint16_t dh = f32_to_f16(d);
    b[0] = (uint8_t)(dh & 0xff);
    b[1] = (uint8_t)(dh >> 8);
    for (int j = 0; j < QK / 2; ++j) {
        float p0 = x[j] * id;
        float p1 = x[j + QK / 2] * id;
        float s0 = p0 + 8.5f;
        float s1 = p1 + 8.5f;
        int u0 = (int)truncf(s0);
        int u1 = (int)truncf(s1);
        if (u0 > 15) u0 = 15;
        if (u1 > 15) u1 = 15;
        b[2 + j] = (uint8_t)(u0 | (u1 << 4));
    }
}

static void quant_block_oscar2(const float *x, uint8_t *b)
{
    float mn = x[0], mx = x[0];
    for (int i = 1; i < QK_OSCAR2; ++i) {
        if (x[i] < mn)
            mn = x[i];
        if (x[i] > mx)
            mx = x[i];
    }
    float range = mx - mn;
    float d = range / 3.0f;
    float id = (d != 0.0f) ? 1.0f / d : 0.0f;
    uint16_t dh = f32_to_f16(d), mh = f32_to_f16(mn);
    b[0] = (uint8_t)(dh & 0xff);
    b[1] = (uint8_t)(dh >> 8);
    b[2] = (uint8_t)(mh & 0xff);
    b[3] = (uint8_t)(mh >> 8);
    for (int j = 0; j < 32; ++j) {
        int byte = 0;
        for (int k = 0; k < 4; ++k) {
            float diff = x[j + 32 * k] - mn;
            float p = diff * id;
            float s = p + 0.5f;
            int u = (int)truncf(s);
            if (u > 3)
                u = 3;
            byte |= u << (2 * k);
        }
        b[4 + j] = (uint8_t)byte;
    }
}

void orc_quantize_q8_0(const float *x, uint8_t *blocks, int64_t n)
{
    int64_t nb = n / QK;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i)
        quant_block_q8_0(x + i * QK, blocks + i * Q8_0_BYTES);
}

void orc_quantize_q4_0(const float *x, uint8_t *blocks, int64_t n)
{
    int64_t nb = n / QK;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i)
        quant_block_q4_0(x + i * QK, blocks + i * Q4_0_BYTES);
}

void orc_quantize_oscar2(const float *x, uint8_t *blocks, int64_t n)
{
    int64_t nb = n / QK_OSCAR2;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < nb; ++i)
        quant_block_oscar2(x + i * QK_OSCAR2, blocks + i * OSCAR2_BYTES);
}

/* Dequantization is exact in fp64 (and in fp32): an fp16 times a small int. */
static void dequant_block_q8_0(const uint8_t *b, double *y)
{
    double d = f16_to_f64((uint16_t)(b[0] | (b[1] << 8)));
    for (int i = 0; i < QK; ++i)
        y[i] = d * (double)(int8_t)b[2 + i];
}

static void dequant_block_q4_0(const uint8_t *b, double *y)
{
    double d = f16_to_f64((uint16_t)(b[0] | (b[1] << 8)));
    for (int j = 0; j < QK / 2; ++j) {
        y[j] = d * (double)((int)(b[2 + j] & 0x0f) - 8);
        y[j + QK / 2] = d * (double)((int)(b[2 + j] >> 4) - 8);
    }
}

/* d*u + m is exact in fp64: every finite fp16 is a multiple of 2^-24 below
 * 2^16, so d*u + m is a multiple of 2^-24 below 2^18 (42 significant bits). */
static void dequant_block_oscar2(const uint8_t *b, double *y)
{
    double d = f16_to_f64((uint16_t)(b[0] | (b[1] << 8)));
    double m = f16_to_f64((uint16_t)(b[2] | (b[3] << 8)));
    for (int j = 0; j < 32; ++j)
        for (int k = 0; k < 4; ++k)
            y[j + 32 * k] = d * (double)((b[4 + j] >> (2 * k)) & 3) + m;
}

void orc_dequant_q8_0(const uint8_t *blocks, double *x, int64_t n)
{
    for (int64_t i = 0; i < n / QK; ++i)
        dequant_block_q8_0(blocks + i * Q8_0_BYTES, x + i * QK);
}

void orc_dequant_q4_0(const uint8_t *blocks, double *x, int64_t n)
{
    for (int64_t i = 0; i < n / QK; ++i)
        dequant_block_q4_0(blocks + i * Q4_0_BYTES, x + i * QK);
}

void orc_dequant_oscar2(const uint8_t *blocks, double *x, int64_t n)
{
    for (int64_t i = 0; i < n / QK_OSCAR2; ++i)
        dequant_block_oscar2(blocks + i * OSCAR2_BYTES, x + i * QK_OSCAR2);
}

/* ------------------------------------------------------------------------ */
/* Cache layout helpers: a block format is FMT_Q8_0, FMT_Q4_0 or FMT_OSCAR2 */
/* ------------------------------------------------------------------------ */

static int block_elems(int fmt) { return fmt == FMT_OSCAR2 ? QK_OSCAR2 : QK; }

static size_t block_bytes(int fmt)
{
    return fmt == FMT_Q8_0 ? Q8_0_BYTES : fmt == FMT_Q4_0 ? Q4_0_BYTES : OSCAR2_BYTES;
}

static size_t row_bytes(int fmt, int head_dim)
{
    return (size_t)(head_dim / block_elems(fmt)) * block_bytes(fmt);
}

static void quant_block(int fmt, const float *x, uint8_t *b)
{
    if (fmt == FMT_Q8_0)
        quant_block_q8_0(x, b);
    else if (fmt == FMT_Q4_0)
        quant_block_q4_0(x, b);
    else
        quant_block_oscar2(x, b);
}

static void dequant_block(int fmt, const uint8_t *b, double *y)
{
    if (fmt == FMT_Q8_0)
        dequant_block_q8_0(b, y);
    else if (fmt == FMT_Q4_0)
        dequant_block_q4_0(b, y);
    else
        dequant_block_oscar2(b, y);
}

/* Head-row j of KV head h, dequantized into y[0..head_dim). */
static void dequant_row(const uint8_t *cache, int fmt, int head_dim, int64_t capacity, int h,
                        int64_t j, double *y)
{
    const uint8_t *r = cache + ((size_t)h * (size_t)capacity + (size_t)j) * row_bytes(fmt, head_dim);
    const int e = block_elems(fmt);
    for (int b = 0; b < head_dim / e; ++b)
        dequant_block(fmt, r + b * block_bytes(fmt), y + b * e);
}

/* Quantize-on-append: rows [pos, pos+n_tok) of every KV head.  k_new and
 * v_new are fp32 [n_tok][n_kv_heads][head_dim]; K blocks in format k_fmt, V
 * blocks in format v_fmt. */
void orc_append(uint8_t *k_cache, uint8_t *v_cache, int n_kv_heads, int head_dim,
                int64_t capacity, const float *k_new, const float *v_new, int64_t pos,
                int64_t n_tok, int k_fmt, int v_fmt)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int64_t t = 0; t < n_tok; ++t)
        for (int h = 0; h < n_kv_heads; ++h) {
            const float *ks = k_new + ((size_t)t * n_kv_heads + h) * head_dim;
            const float *vs = v_new + ((size_t)t * n_kv_heads + h) * head_dim;
            const size_t row = (size_t)h * capacity + (size_t)(pos + t);
            uint8_t *kd = k_cache + row * row_bytes(k_fmt, head_dim);
            uint8_t *vd = v_cache + row * row_bytes(v_fmt, head_dim);
            const int ek = block_elems(k_fmt), ev = block_elems(v_fmt);
            for (int b = 0; b < head_dim / ek; ++b)
                quant_block(k_fmt, ks + b * ek, kd + b * block_bytes(k_fmt));
            for (int b = 0; b < head_dim / ev; ++b)
                quant_block(v_fmt, vs + b * ev, vd + b * block_bytes(v_fmt));
        }
}

/* ------------------------------------------------------------------------ */
/* Attention, fp64                                                          */
/* ------------------------------------------------------------------------ */

/* Softmax attention of n_rows query vectors (fp64, [n_rows][head_dim]) that
 * all read KV head h, each over its own key range [k0[r], k1[r]).  Scores
 * for every visible key are computed first; the max is taken over those
 * complete scores, then the weights, their sum, the output and the lse.
 * Results: out [n_rows][head_dim], lse [n_rows]. */
static void attend(const uint8_t *k_cache, const uint8_t *v_cache, int k_fmt, int v_fmt,
                   int head_dim, int64_t capacity, int h, const double *q, int n_rows,
                   const int64_t *k0, const int64_t *k1, double scale, double *out, double *lse)
{
    int64_t lo = INT64_MAX, hi = INT64_MIN;
    for (int r = 0; r < n_rows; ++r) {
        if (k1[r] > k0[r]) {
            if (k0[r] < lo) lo = k0[r];
            if (k1[r] > hi) hi = k1[r];
        }
    }
    for (int r = 0; r < n_rows; ++r) {
        memset(out + (size_t)r * head_dim, 0, sizeof(double) * head_dim);
        lse[r] = -INFINITY;
    }
    if (hi <= lo)
        return;
    int64_t n = hi - lo;
    double *s = (double *)malloc(sizeof(double) * (size_t)n * n_rows);
    double *kh = (double *)malloc(sizeof(double) * head_dim);
    double *vh = (double *)malloc(sizeof(double) * head_dim);
    double *m = (double *)malloc(sizeof(double) * n_rows);
    double *l = (double *)malloc(sizeof(double) * n_rows);

    /* 1. complete scores */
    for (int64_t j = lo; j < hi; ++j) {
        dequant_row(k_cache, k_fmt, head_dim, capacity, h, j, kh);
        for (int r = 0; r < n_rows; ++r) {
            double acc = 0.0;
            const double *qr = q + (size_t)r * head_dim;
            for (int i = 0; i < head_dim; ++i)
                acc += qr[i] * kh[i];
            s[(size_t)r * n + (j - lo)] = scale * acc;
        }
    }
    /* 2. max over the complete visible scores */
    for (int r = 0; r < n_rows; ++r) {
        m[r] = -INFINITY;
        for (int64_t j = k0[r]; j < k1[r]; ++j) {
            double v = s[(size_t)r * n + (j - lo)];
            if (v > m[r])
                m[r] = v;
        }
        l[r] = 0.0;
    }
    /* 3. weights, their sum and the weighted V sum */
    for (int64_t j = lo; j < hi; ++j) {
        dequant_row(v_cache, v_fmt, head_dim, capacity, h, j, vh);
        for (int r = 0; r < n_rows; ++r) {
            if (j < k0[r] || j >= k1[r])
                continue;
            double p = exp(s[(size_t)r * n + (j - lo)] - m[r]);
            l[r] += p;
            double *o = out + (size_t)r * head_dim;
            for (int i = 0; i < head_dim; ++i)
                o[i] += p * vh[i];
        }
    }
    /* 4. normalise; lse in natural log */
    for (int r = 0; r < n_rows; ++r) {
        if (k1[r] <= k0[r])
            continue;
        double *o = out + (size_t)r * head_dim;
        for (int i = 0; i < head_dim; ++i)
            o[i] /= l[r];
        lse[r] = m[r] + log(l[r]);
    }
    free(s);
    free(kh);
    free(vh);
    free(m);
    free(l);
}

static void load_q(const uint16_t *q16, double *q, int64_t n)
{
    for (int64_t i = 0; i < n; ++i)
        q[i] = f16_to_f64(q16[i]);
}

/* Split-KV decode attention: per chunk c = keys [c*chunk, (c+1)*chunk) cut
 * to [0, n_kv), the partial (out, lse) of every query row over the visible
 * keys of that chunk.
 *   q        fp16 bits [T][n_q_heads][head_dim]
 *   out_part [T][n_q_heads][n_chunks][head_dim], lse_part [T][n_q_heads][n_chunks]
 * n_chunks = ceil(n_kv / chunk).  Query token t sees keys j <= n_kv - T + t. */
void orc_decode_attn(const uint8_t *k_cache, const uint8_t *v_cache, int n_kv_heads,
                     int head_dim, int64_t capacity, const uint16_t *q, int n_q_heads, int T,
                     int64_t n_kv, int64_t chunk, double scale, double *out_part,
                     double *lse_part, int k_fmt, int v_fmt)
{
    int G = n_q_heads / n_kv_heads;
    int64_t n_chunks = (n_kv + chunk - 1) / chunk;
    int rows = G * T;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int h = 0; h < n_kv_heads; ++h)
        for (int64_t c = 0; c < n_chunks; ++c) {
            double *qd = (double *)malloc(sizeof(double) * rows * head_dim);
            double *o = (double *)malloc(sizeof(double) * rows * head_dim);
            double *ls = (double *)malloc(sizeof(double) * rows);
            int64_t *k0 = (int64_t *)malloc(sizeof(int64_t) * rows);
            int64_t *k1 = (int64_t *)malloc(sizeof(int64_t) * rows);
            int64_t c0 = c * chunk, c1 = c0 + chunk < n_kv ? c0 + chunk : n_kv;
            for (int t = 0; t < T; ++t)
                for (int g = 0; g < G; ++g) {
                    int r = t * G + g, qh = h * G + g;
                    load_q(q + ((size_t)t * n_q_heads + qh) * head_dim, qd + (size_t)r * head_dim,
                           head_dim);
                    int64_t last = n_kv - T + t; /* last visible key */
                    k0[r] = c0;
                    k1[r] = (last + 1 < c1) ? last + 1 : c1;
                }
            attend(k_cache, v_cache, k_fmt, v_fmt, head_dim, capacity, h, qd, rows, k0, k1,
                   scale, o, ls);
            for (int t = 0; t < T; ++t)
                for (int g = 0; g < G; ++g) {
                    int r = t * G + g, qh = h * G + g;
                    size_t row = ((size_t)t * n_q_heads + qh) * (size_t)n_chunks + (size_t)c;
                    memcpy(out_part + row * head_dim, o + (size_t)r * head_dim,
                           sizeof(double) * head_dim);
                    lse_part[row] = ls[r];
                }
            free(qd);
            free(o);
            free(ls);
            free(k0);
            free(k1);
        }
}

/* Merge of partials: out_part [rows][n_chunks][head_dim], lse_part [rows][n_chunks]
 * -> out [rows][head_dim], lse [rows]. */
void orc_merge_lse(const double *out_part, const double *lse_part, int64_t rows, int n_chunks,
                   int head_dim, double *out, double *lse)
{
#pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        const double *lp = lse_part + (size_t)r * n_chunks;
        double M = -INFINITY;
        for (int c = 0; c < n_chunks; ++c)
            if (lp[c] > M)
                M = lp[c];
        double *o = out + (size_t)r * head_dim;
        memset(o, 0, sizeof(double) * head_dim);
        if (M == -INFINITY) {
            lse[r] = -INFINITY;
            continue;
        }
        double sum = 0.0;
        for (int c = 0; c < n_chunks; ++c)
            if (lp[c] != -INFINITY)
                sum += exp(lp[c] - M);
        double L = M + log(sum);
        for (int c = 0; c < n_chunks; ++c) {
            if (lp[c] == -INFINITY)
                continue;
            double w = exp(lp[c] - L);
            const double *oc = out_part + ((size_t)r * n_chunks + c) * head_dim;
            for (int i = 0; i < head_dim; ++i)
                o[i] += w * oc[i];
        }
        lse[r] = L;
    }
}

/* One-pass attention of arbitrary rows: row r is the fp16 query q_rows[r]
 * of query head q_head[r], over keys [key_begin[r], key_end[r]) of its KV
 * head.  Used for sampled checks at full context and for prefill rows. */
void orc_attn_rows(const uint8_t *k_cache, const uint8_t *v_cache, int n_kv_heads,
                   int head_dim, int64_t capacity, const uint16_t *q_rows,
                   const int32_t *q_head, int n_q_heads, const int64_t *key_begin,
                   const int64_t *key_end, int64_t n_rows, double scale, double *out,
                   double *lse, int k_fmt, int v_fmt)
{
    int G = n_q_heads / n_kv_heads;
#pragma omp parallel for schedule(dynamic)
    for (int64_t r = 0; r < n_rows; ++r) {
        double *qd = (double *)malloc(sizeof(double) * head_dim);
        load_q(q_rows + (size_t)r * head_dim, qd, head_dim);
        attend(k_cache, v_cache, k_fmt, v_fmt, head_dim, capacity, q_head[r] / G, qd, 1,
               key_begin + r, key_end + r, scale, out + (size_t)r * head_dim, lse + r);
        free(qd);
    }
}

/* Chunked prefill: T new query tokens over n_cached + T keys; token t sees
 * keys j <= n_cached + t.  out [T][n_q_heads][head_dim] and lse [T][n_q_heads]
 * are the one-pass result.  If page_out is not NULL, the per-page partials
 * (page p = keys [p*page, (p+1)*page)) are written to
 * page_out [T][n_q_heads][n_pages][head_dim] and page_lse [T][n_q_heads][n_pages],
 * n_pages = ceil((n_cached + T) / page). */
void orc_prefill_attn(const uint8_t *k_cache, const uint8_t *v_cache, int n_kv_heads,
                      int head_dim, int64_t capacity, const uint16_t *q, int n_q_heads, int T,
                      int64_t n_cached, int64_t page, double scale, double *out, double *lse,
                      double *page_out, double *page_lse, int k_fmt, int v_fmt)
{
    int G = n_q_heads / n_kv_heads;
    int64_t n_keys = n_cached + T;
    int64_t n_pages = (n_keys + page - 1) / page;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int t = 0; t < T; ++t)
        for (int qh = 0; qh < n_q_heads; ++qh) {
            double *qd = (double *)malloc(sizeof(double) * head_dim);
            load_q(q + ((size_t)t * n_q_heads + qh) * head_dim, qd, head_dim);
            size_t row = (size_t)t * n_q_heads + qh;
            int64_t b = 0, e = n_cached + t + 1;
            attend(k_cache, v_cache, k_fmt, v_fmt, head_dim, capacity, qh / G, qd, 1, &b, &e,
                   scale, out + row * head_dim, lse + row);
            if (page_out) {
                for (int64_t p = 0; p < n_pages; ++p) {
                    int64_t p0 = p * page, p1 = p0 + page < e ? p0 + page : e;
                    if (p1 < p0)
                        p1 = p0;
                    attend(k_cache, v_cache, k_fmt, v_fmt, head_dim, capacity, qh / G, qd, 1,
                           &p0, &p1, scale, page_out + (row * n_pages + p) * head_dim,
                           page_lse + row * n_pages + p);
                }
            }
            free(qd);
        }
}
