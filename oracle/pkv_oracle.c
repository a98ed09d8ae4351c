/*
 * pkv_oracle.c -- plain fp64 CPU oracle for the paged-KV decode step.
 *
 * TEST INFRASTRUCTURE ONLY (tests, the smoke check and the benchmark's
 * CPU-baseline leg).  Single-threaded, deliberately unoptimised: every
 * function is the textbook definition written out so that it can be checked
 * by eye.  It shares nothing with the GPU library.
 *
 * Page citations use the page title and section:
 *   [P1] "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
 *        Production"
 *   [P2] "TensorRT-LLM: NVIDIA's Optimized Inference Engine"
 *   [P4] "TensorRT-LLM Guide: High-Throughput GPU Inference Engine"
 *
 * Parity pins (tests/test_oracle_*.py, tests/test_codecs.py) tie each
 * function to facts outside this file: exhaustive codec tables from the
 * formats' closed forms and a library cast, RoPE identities and a complex-
 * number formulation, brute-force attention loops, a library SDPA in fp64,
 * and the closed-form special cases (one-token context, identical keys,
 * zero query, one offset added to every key, permuted physical pages).
 */
#include "pkv_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* bf16: the upper 16 bits of an IEEE binary32.                        */
/* ------------------------------------------------------------------ */

double orc_bf16_decode(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f; /* exact: every bf16 value is a binary32 value */
}

/* Round-to-nearest-even straight from fp64 to bf16 (8 significant bits,
 * exponent range of binary32, subnormal quantum 2^-133). */
uint16_t orc_bf16_encode_rne(double x)
{
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (isinf(a)) return sign | 0x7F80;
    if (a == 0.0) return sign;

    int e;
    frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1) */
    int lead = e - 1;         /* exponent of the leading bit */
    int qexp = lead - 7;      /* quantum: 8 significant bits */
    if (qexp < -133) qexp = -133;
    double r = nearbyint(ldexp(a, -qexp)); /* ties to even (default mode) */
    double v = ldexp(r, qexp);
    if (v > ldexp(255.0, 120)) return sign | 0x7F80; /* above max finite */

    float f = (float)v; /* exact */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)((u >> 16) & 0x7FFF);
}

/* ------------------------------------------------------------------ */
/* E4M3 (OCP FP8 E4M3FN): s eeee mmm, bias 7, no infinities,           */
/* S.1111.111 is NaN, max finite 448, subnormals 2^-6 * m/8.           */
/* ------------------------------------------------------------------ */

double orc_e4m3_decode(uint8_t code)
{
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    if (e == 15 && m == 7) return NAN;
    double mag = (e == 0) ? ldexp((double)m, -9)          /* 2^-6 * m/8 */
                          : ldexp(8.0 + m, e - 10);       /* 2^(e-7) * (1 + m/8) */
    return s ? -mag : mag;
}

/* Round-to-nearest-even from a binary32 value, saturating to +-448
 * ("satfinite"); NaN gives 0x7F. */
uint8_t orc_e4m3_encode_satfinite(float xf)
{
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    /* every value >= 448 (including inf) rounds to 448 or to a value above
     * the largest finite code, which satfinite clamps to 448 */
    if (a >= 448.0) return sign | 0x7E;
    if (a == 0.0) return sign;

    int e;
    frexp(a, &e);
    int lead = e - 1;
    if (lead < -6) {
        /* subnormal range: quantum 2^-9; r == 8 is 2^-6, which is code 0x08 */
        double r = nearbyint(ldexp(a, 9));
        return sign | (uint8_t)r;
    }
    /* normal: r = round(a / 2^(lead-3)) in [8, 16]; r == 16 carries into
     * the next exponent, which the code arithmetic below does by itself */
    double r = nearbyint(ldexp(a, 3 - lead));
    int code = ((lead + 7) << 3) + ((int)r - 8);
    return sign | (uint8_t)code;
}

void orc_bf16_decode_n(const uint16_t* in, double* out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = orc_bf16_decode(in[i]);
}

void orc_bf16_encode_rne_n(const double* in, uint16_t* out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = orc_bf16_encode_rne(in[i]);
}

void orc_e4m3_decode_n(const uint8_t* in, double* out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = orc_e4m3_decode(in[i]);
}

void orc_e4m3_encode_satfinite_n(const float* in, uint8_t* out, long long n)
{
    for (long long i = 0; i < n; ++i) out[i] = orc_e4m3_encode_satfinite(in[i]);
}

float orc_f32_round(double x)
{
    return (float)x; /* C conversion rounds to nearest even */
}

/* ------------------------------------------------------------------ */
/* RoPE, rotate-half pairing (i, i + d/2), theta_i = base^(-2i/d).     */
/* [P1] section "What Gets Fused" (RoPE applied inside the attention    */
/* projection kernel); the formula itself is the Llama convention.     */
/* ------------------------------------------------------------------ */

void orc_rope_f64(const double* x, double* y, int d, double pos, double base)
{
    int half = d / 2;
    for (int i = 0; i < half; ++i) {
        double theta = pow(base, (-2.0 * i) / d);
        double phi = pos * theta;
        double c = cos(phi), s = sin(phi);
        double xi = x[i], xj = x[i + half];
        y[i] = xi * c - xj * s;
        y[i + half] = xj * c + xi * s;
    }
}

static int cfg_ok(const orc_cfg* c)
{
    if (!c) return 0;
    if (c->num_q_heads <= 0 || c->num_kv_heads <= 0) return 0;
    if (c->num_q_heads % c->num_kv_heads) return 0;
    if (c->head_dim <= 0 || (c->head_dim & 1)) return 0;
    if (c->page_size <= 0 || c->num_pages <= 0) return 0;
    return 1;
}

/* Row index (in units of d elements) of token slot `slot` of kv head `kvh`
 * in physical page `page`: pools are [num_pages][Hkv][P][d]. */
static size_t pool_row(const orc_cfg* c, int page, int kvh, int slot)
{
    return ((size_t)page * c->num_kv_heads + kvh) * c->page_size + slot;
}

/* ------------------------------------------------------------------ */
/* Step part 1: RoPE of the new token's q and k, append of k and v.    */
/* Placement: page = block_tables[b][L_b / P], slot L_b % P            */
/* ([P4] "2. Paged KV Cache & Memory Virtualization": a lookup table   */
/* maps logical token positions to physical blocks).                    */
/* ------------------------------------------------------------------ */

int orc_rope_append(const orc_cfg* cfg,
                    uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                    void* k_pool, void* v_pool,
                    const float* k_scale, const float* v_scale,
                    const int32_t* block_tables, int bt_stride,
                    const int32_t* seq_lens, int batch)
{
    if (!cfg_ok(cfg) || batch < 0 || bt_stride <= 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!q || !k_new || !v_new || !k_pool || !v_pool || !block_tables || !seq_lens)
        return ORC_ERR_ARG;
    if (cfg->kv_fp8 && (!k_scale || !v_scale)) return ORC_ERR_ARG;

    const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
    const int P = cfg->page_size;
    double* x = (double*)malloc(sizeof(double) * d);
    double* y = (double*)malloc(sizeof(double) * d);
    if (!x || !y) { free(x); free(y); return ORC_ERR_ARG; }
    int status = ORC_OK;

    for (int b = 0; b < batch; ++b) {
        const int L = seq_lens[b];
        if (L < 0 || (long long)L >= (long long)bt_stride * P) { status = ORC_ERR_RANGE; continue; }
        const int page = block_tables[(size_t)b * bt_stride + L / P];
        if (page < 0 || page >= cfg->num_pages) { status = ORC_ERR_RANGE; continue; }
        const int slot = L % P;

        /* q: every query head rotated at position L, rounded back to bf16 */
        for (int h = 0; h < Hq; ++h) {
            uint16_t* row = q + ((size_t)b * Hq + h) * d;
            for (int j = 0; j < d; ++j) x[j] = orc_bf16_decode(row[j]);
            orc_rope_f64(x, y, d, (double)L, cfg->rope_base);
            for (int j = 0; j < d; ++j) row[j] = orc_bf16_encode_rne(y[j]);
        }
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            const uint16_t* krow = k_new + ((size_t)b * Hkv + kvh) * d;
            const uint16_t* vrow = v_new + ((size_t)b * Hkv + kvh) * d;
            for (int j = 0; j < d; ++j) x[j] = orc_bf16_decode(krow[j]);
            orc_rope_f64(x, y, d, (double)L, cfg->rope_base);
            const size_t dst = pool_row(cfg, page, kvh, slot) * (size_t)d;
            if (!cfg->kv_fp8) {
                uint16_t* kp = (uint16_t*)k_pool;
                uint16_t* vp = (uint16_t*)v_pool;
                for (int j = 0; j < d; ++j) {
                    kp[dst + j] = orc_bf16_encode_rne(y[j]);
                    vp[dst + j] = vrow[j]; /* v is never rotated */
                }
            } else {
                uint8_t* kp = (uint8_t*)k_pool;
                uint8_t* vp = (uint8_t*)v_pool;
                const double sk = k_scale[(size_t)page * Hkv + kvh];
                const double sv = v_scale[(size_t)page * Hkv + kvh];
                for (int j = 0; j < d; ++j) {
                    kp[dst + j] = orc_e4m3_encode_satfinite(orc_f32_round(y[j] / sk));
                    vp[dst + j] = orc_e4m3_encode_satfinite(
                        orc_f32_round(orc_bf16_decode(vrow[j]) / sv));
                }
            }
        }
    }
    free(x);
    free(y);
    return status;
}

/* ------------------------------------------------------------------ */
/* Step part 2: decode attention of the new query over n_b = L_b + 1   */
/* cached tokens, grouped-query (kv head = h / G).                      */
/* [P4] "3. Custom Fused Attention Kernels: FMHA and XQA": query heads  */
/* of a group share one KV head.  Definition: o_h = softmax(q_h K^T /   */
/* sqrt(d)) V, softmax taken with the maximum subtracted, all in fp64.  */
/* ------------------------------------------------------------------ */

static double kv_value(const orc_cfg* cfg, const void* pool, const float* scale,
                       int page, int kvh, int slot, int j)
{
    const size_t idx = pool_row(cfg, page, kvh, slot) * (size_t)cfg->head_dim + j;
    if (!cfg->kv_fp8) return orc_bf16_decode(((const uint16_t*)pool)[idx]);
    /* code value (exact) times the fp32 scale of this (page, kv head) */
    return orc_e4m3_decode(((const uint8_t*)pool)[idx]) *
           (double)scale[(size_t)page * cfg->num_kv_heads + kvh];
}

/* The definition for G query rows (bf16 bits, G x d, the heads kvh*G ..
 * kvh*G + G-1) over the first n tokens of one request's block-table row bt:
 * explicit gather of the tokens in logical order, then per row
 * o = softmax(q K^T / sqrt(d)) V with the maximum subtracted, in fp64. */
static int attend_rows(const orc_cfg* cfg, const uint16_t* qrows, const void* k_pool,
                       const void* v_pool, const float* k_scale, const float* v_scale,
                       const int32_t* bt, int n, int kvh, double* out)
{
    const int d = cfg->head_dim, P = cfg->page_size, G = cfg->num_q_heads / cfg->num_kv_heads;
    double* K = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* V = (double*)malloc(sizeof(double) * (size_t)n * d);
    double* w = (double*)malloc(sizeof(double) * (size_t)n);
    double* qh = (double*)malloc(sizeof(double) * (size_t)d);
    if (!K || !V || !w || !qh) { free(K); free(V); free(w); free(qh); return ORC_ERR_ARG; }
    int status = ORC_OK;
    for (int t = 0; t < n && status == ORC_OK; ++t) {
        const int page = bt[t / P];
        if (page < 0 || page >= cfg->num_pages) { status = ORC_ERR_RANGE; break; }
        for (int j = 0; j < d; ++j) {
            K[(size_t)t * d + j] = kv_value(cfg, k_pool, k_scale, page, kvh, t % P, j);
            V[(size_t)t * d + j] = kv_value(cfg, v_pool, v_scale, page, kvh, t % P, j);
        }
    }

    if (status == ORC_OK) {
        const double inv_sqrt_d = 1.0 / sqrt((double)d);
        for (int g = 0; g < G; ++g) {
            for (int j = 0; j < d; ++j) qh[j] = orc_bf16_decode(qrows[(size_t)g * d + j]);
            double m = -INFINITY;
            for (int t = 0; t < n; ++t) {
                double s = 0.0;
                for (int j = 0; j < d; ++j) s += qh[j] * K[(size_t)t * d + j];
                w[t] = s * inv_sqrt_d;
                if (w[t] > m) m = w[t];
            }
            double l = 0.0;
            for (int t = 0; t < n; ++t) {
                w[t] = exp(w[t] - m);
                l += w[t];
            }
            for (int j = 0; j < d; ++j) {
                double o = 0.0;
                for (int t = 0; t < n; ++t) o += w[t] * V[(size_t)t * d + j];
                out[(size_t)g * d + j] = o / l;
            }
        }
    }
    free(K);
    free(V);
    free(w);
    free(qh);
    return status;
}

int orc_decode_attn_group(const orc_cfg* cfg, const uint16_t* q,
                          const void* k_pool, const void* v_pool,
                          const float* k_scale, const float* v_scale,
                          const int32_t* block_tables, int bt_stride,
                          const int32_t* seq_lens, int b, int kvh, double* out)
{
    if (!cfg_ok(cfg) || !q || !k_pool || !v_pool || !block_tables || !seq_lens || !out)
        return ORC_ERR_ARG;
    if (cfg->kv_fp8 && (!k_scale || !v_scale)) return ORC_ERR_ARG;
    if (kvh < 0 || kvh >= cfg->num_kv_heads || b < 0 || bt_stride <= 0) return ORC_ERR_ARG;

    const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
    const int P = cfg->page_size, G = Hq / Hkv;
    const int L = seq_lens[b];
    if (L < 0 || (long long)L >= (long long)bt_stride * P) return ORC_ERR_RANGE;
    return attend_rows(cfg, q + ((size_t)b * Hq + (size_t)kvh * G) * d, k_pool, v_pool, k_scale, v_scale,
                       block_tables + (size_t)b * bt_stride, L + 1, kvh, out);
}

int orc_decode_attn(const orc_cfg* cfg, const uint16_t* q,
                    const void* k_pool, const void* v_pool,
                    const float* k_scale, const float* v_scale,
                    const int32_t* block_tables, int bt_stride,
                    const int32_t* seq_lens, int batch, double* out)
{
    if (!cfg_ok(cfg) || batch < 0 || !out) return ORC_ERR_ARG;
    const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
    const int G = Hq / Hkv;
    int status = ORC_OK;
    for (int b = 0; b < batch; ++b) {
        for (int kvh = 0; kvh < Hkv; ++kvh) {
            double* dst = out + ((size_t)b * Hq + (size_t)kvh * G) * d;
            int s = orc_decode_attn_group(cfg, q, k_pool, v_pool, k_scale, v_scale,
                                          block_tables, bt_stride, seq_lens, b, kvh, dst);
            if (s != ORC_OK) {
                for (size_t i = 0; i < (size_t)G * d; ++i) dst[i] = NAN;
                if (status == ORC_OK) status = s;
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* Several new tokens per request: a draft proposes tokens and the      */
/* target checks all of them in one pass ("Scaling TensorRT-LLM",       */
/* section "3. Speculative Decoding for Tail Latency"; "TensorRT-LLM    */
/* Guide", section "2. Pipelined Speculative Decoding").  New token t   */
/* (0 <= t < q_len) of request b sits at position L_b + t; q is         */
/* [batch][q_len][Hq][d], k_new / v_new [batch][q_len][Hkv][d].         */
/* ------------------------------------------------------------------ */

int orc_rope_append_tokens(const orc_cfg* cfg,
                           uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                           void* k_pool, void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, int q_len)
{
    if (!cfg_ok(cfg) || batch < 0 || bt_stride <= 0 || q_len <= 0) return ORC_ERR_ARG;
    if (batch == 0) return ORC_OK;
    if (!q || !k_new || !v_new || !k_pool || !v_pool || !block_tables || !seq_lens)
        return ORC_ERR_ARG;
    if (cfg->kv_fp8 && (!k_scale || !v_scale)) return ORC_ERR_ARG;

    const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
    const int P = cfg->page_size;
    double* x = (double*)malloc(sizeof(double) * d);
    double* y = (double*)malloc(sizeof(double) * d);
    if (!x || !y) { free(x); free(y); return ORC_ERR_ARG; }
    int status = ORC_OK;

    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < q_len; ++t) {
            const long long pos = (long long)seq_lens[b] + t;   /* position of new token t */
            if (seq_lens[b] < 0 || pos >= (long long)bt_stride * P) { status = ORC_ERR_RANGE; continue; }
            const int page = block_tables[(size_t)b * bt_stride + pos / P];
            if (page < 0 || page >= cfg->num_pages) { status = ORC_ERR_RANGE; continue; }
            const int slot = (int)(pos % P);
            const size_t bt_row = (size_t)b * q_len + t;   /* row of (b, t) in q, k_new, v_new */

            for (int h = 0; h < Hq; ++h) {
                uint16_t* row = q + (bt_row * Hq + h) * d;
                for (int j = 0; j < d; ++j) x[j] = orc_bf16_decode(row[j]);
                orc_rope_f64(x, y, d, (double)pos, cfg->rope_base);
                for (int j = 0; j < d; ++j) row[j] = orc_bf16_encode_rne(y[j]);
            }
            for (int kvh = 0; kvh < Hkv; ++kvh) {
                const uint16_t* krow = k_new + (bt_row * Hkv + kvh) * d;
                const uint16_t* vrow = v_new + (bt_row * Hkv + kvh) * d;
                for (int j = 0; j < d; ++j) x[j] = orc_bf16_decode(krow[j]);
                orc_rope_f64(x, y, d, (double)pos, cfg->rope_base);
                const size_t dst = pool_row(cfg, page, kvh, slot) * (size_t)d;
                if (!cfg->kv_fp8) {
                    uint16_t* kp = (uint16_t*)k_pool;
                    uint16_t* vp = (uint16_t*)v_pool;
                    for (int j = 0; j < d; ++j) {
                        kp[dst + j] = orc_bf16_encode_rne(y[j]);
                        vp[dst + j] = vrow[j];
                    }
                } else {
                    uint8_t* kp = (uint8_t*)k_pool;
                    uint8_t* vp = (uint8_t*)v_pool;
                    const double sk = k_scale[(size_t)page * Hkv + kvh];
                    const double sv = v_scale[(size_t)page * Hkv + kvh];
                    for (int j = 0; j < d; ++j) {
                        kp[dst + j] = orc_e4m3_encode_satfinite(orc_f32_round(y[j] / sk));
                        vp[dst + j] = orc_e4m3_encode_satfinite(
                            orc_f32_round(orc_bf16_decode(vrow[j]) / sv));
                    }
                }
            }
        }
    }
    free(x);
    free(y);
    return status;
}

/* New token t attends tokens 0 .. L_b + t: everything cached, the new
 * tokens before it and itself, none after it (each candidate is checked as
 * if the ones before it had been accepted). */
int orc_decode_attn_tokens_group(const orc_cfg* cfg, const uint16_t* q,
                                 const void* k_pool, const void* v_pool,
                                 const float* k_scale, const float* v_scale,
                                 const int32_t* block_tables, int bt_stride,
                                 const int32_t* seq_lens, int q_len, int b, int t, int kvh,
                                 double* out)
{
    if (!cfg_ok(cfg) || !q || !k_pool || !v_pool || !block_tables || !seq_lens || !out)
        return ORC_ERR_ARG;
    if (cfg->kv_fp8 && (!k_scale || !v_scale)) return ORC_ERR_ARG;
    if (q_len <= 0 || t < 0 || t >= q_len || kvh < 0 || kvh >= cfg->num_kv_heads || b < 0 || bt_stride <= 0)
        return ORC_ERR_ARG;
    const int Hq = cfg->num_q_heads, G = Hq / cfg->num_kv_heads, d = cfg->head_dim;
    const long long n = (long long)seq_lens[b] + t + 1;
    if (seq_lens[b] < 0 || n > (long long)bt_stride * cfg->page_size) return ORC_ERR_RANGE;
    const size_t bt_row = (size_t)b * q_len + t;
    return attend_rows(cfg, q + (bt_row * Hq + (size_t)kvh * G) * d, k_pool, v_pool, k_scale, v_scale,
                       block_tables + (size_t)b * bt_stride, (int)n, kvh, out);
}

int orc_decode_attn_tokens(const orc_cfg* cfg, const uint16_t* q,
                           const void* k_pool, const void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, int q_len, double* out)
{
    if (!cfg_ok(cfg) || batch < 0 || q_len <= 0 || !out) return ORC_ERR_ARG;
    const int Hq = cfg->num_q_heads, Hkv = cfg->num_kv_heads, d = cfg->head_dim;
    const int G = Hq / Hkv;
    int status = ORC_OK;
    for (int b = 0; b < batch; ++b) {
        for (int t = 0; t < q_len; ++t) {
            for (int kvh = 0; kvh < Hkv; ++kvh) {
                double* dst = out + (((size_t)b * q_len + t) * Hq + (size_t)kvh * G) * d;
                int s = orc_decode_attn_tokens_group(cfg, q, k_pool, v_pool, k_scale, v_scale, block_tables,
                                                     bt_stride, seq_lens, q_len, b, t, kvh, dst);
                if (s != ORC_OK) {
                    for (size_t i = 0; i < (size_t)G * d; ++i) dst[i] = NAN;
                    if (status == ORC_OK) status = s;
                }
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------ */
/* The QKV projection that produces q, k_new and v_new from the layer   */
/* input, fused with RoPE and the append on the GPU ("Scaling           */
/* TensorRT-LLM", section "What Gets Fused": the attention block's      */
/* projections with their epilogues).  Definition: out[t][n] =          */
/* bf16_RNE( sum_j x[t][j] * w[n][j] ) with the sum in fp64; w is        */
/* [N][hidden] (one row per output feature).                            */
/* ------------------------------------------------------------------ */

int orc_project_bf16(const uint16_t* x, const uint16_t* w, int T, int N, int hidden, uint16_t* out)
{
    if (!x || !w || !out || T < 0 || N <= 0 || hidden <= 0) return ORC_ERR_ARG;
    for (int t = 0; t < T; ++t) {
        for (int n = 0; n < N; ++n) {
            double s = 0.0;
            for (int j = 0; j < hidden; ++j)
                s += orc_bf16_decode(x[(size_t)t * hidden + j]) * orc_bf16_decode(w[(size_t)n * hidden + j]);
            out[(size_t)t * N + n] = orc_bf16_encode_rne(s);
        }
    }
    return ORC_OK;
}
