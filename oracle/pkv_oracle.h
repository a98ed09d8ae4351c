/*
 * pkv_oracle.h -- plain, slow, single-threaded fp64 CPU oracle for one
 * in-flight-batched decode step over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may call this library.  It shares no code,
 * header, table or helper with the GPU library (libpkv); the two are built
 * separately and neither includes or links the other.
 *
 * What it computes follows the pages:
 *   - paged KV with a per-request block table, looked up per token:
 *     "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
 *     Production", section "The Paged KV-Cache"; "TensorRT-LLM Guide:
 *     High-Throughput GPU Inference Engine", section "2. Paged KV Cache &
 *     Memory Virtualization".
 *   - rotary embedding of the new token's q/k before attention: first page,
 *     section "What Gets Fused" (RoPE bullet).
 *   - grouped-query decode attention, one new query per request over all of
 *     its cached tokens: "TensorRT-LLM Guide", section "3. Custom Fused
 *     Attention Kernels: FMHA and XQA".
 *   - an E4M3 KV cache: "TensorRT-LLM Guide", section "4. Native FP8
 *     Quantization on NVIDIA Hopper & Blackwell".
 * The pages give no formula for any of these; the readings taken (rotate-half
 * RoPE, softmax(q K^T / sqrt(d)) V, kvh = h / G, one fp32 scale per
 * (page, kv head)) are the plain Llama-style definitions, stated next to each
 * function below.
 *
 * Storage conventions (shared with the GPU library only by specification,
 * never by code):
 *   bf16 values are passed as their uint16_t bit patterns;
 *   E4M3 values as uint8_t codes (OCP FP8 E4M3FN: bias 7, no infinities,
 *   0x7F/0xFF are NaN, max finite 448);
 *   pools are [num_pages][Hkv][P][d]; block_tables is [batch][bt_stride]
 *   int32; seq_lens[b] = L_b = tokens cached BEFORE the step.
 */
#ifndef PKV_ORACLE_H
#define PKV_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct {
    int num_q_heads;      /* Hq */
    int num_kv_heads;     /* Hkv; Hq % Hkv == 0 */
    int head_dim;         /* d, even */
    int page_size;        /* P, tokens per page */
    int kv_fp8;           /* 0: bf16 pools, 1: E4M3 pools + per-(page, kv head) scales */
    int num_pages;        /* physical pages in each pool */
    double rope_base;     /* theta_i = rope_base^(-2i/d) */
} orc_cfg;

/* Return codes. */
#define ORC_OK 0
#define ORC_ERR_ARG 1     /* bad shape or pointer */
#define ORC_ERR_RANGE 2   /* page id or length outside the pool / block table */

/* ---- codecs ---------------------------------------------------------- */
double   orc_bf16_decode(uint16_t bits);
uint16_t orc_bf16_encode_rne(double x);
double   orc_e4m3_decode(uint8_t code);
uint8_t  orc_e4m3_encode_satfinite(float x);
float    orc_f32_round(double x);          /* IEEE round-to-nearest-even to fp32 */

/* Array forms of the four codecs (plain loops), for the tests. */
void orc_bf16_decode_n(const uint16_t* in, double* out, long long n);
void orc_bf16_encode_rne_n(const double* in, uint16_t* out, long long n);
void orc_e4m3_decode_n(const uint8_t* in, double* out, long long n);
void orc_e4m3_encode_satfinite_n(const float* in, uint8_t* out, long long n);

/* ---- RoPE ------------------------------------------------------------ */
/* y = RoPE(x, pos) in fp64; x and y are d doubles (may alias). */
void orc_rope_f64(const double* x, double* y, int d, double pos, double base);

/* ---- the step -------------------------------------------------------- */
/* Rotates q (all Hq heads, bf16 bits, in place) and k_new at position
 * L_b = seq_lens[b], then writes rotated k and raw v into slot L_b % P of
 * page block_tables[b][L_b / P] of each pool.  bf16 pools: k stored as
 * bf16-RNE of the fp64 rotation, v copied.  fp8 pools: code =
 * E4M3_RNE_satfinite(fl32(x / scale[page][kvh])). */
int orc_rope_append(const orc_cfg* cfg,
                    uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                    void* k_pool, void* v_pool,
                    const float* k_scale, const float* v_scale,
                    const int32_t* block_tables, int bt_stride,
                    const int32_t* seq_lens, int batch);

/* Attention output of one (request b, kv head kvh) group in fp64:
 * out[g*d + j] for the G = Hq/Hkv query heads h = kvh*G + g.
 * Attends n_b = seq_lens[b] + 1 tokens read through the block table. */
int orc_decode_attn_group(const orc_cfg* cfg, const uint16_t* q,
                          const void* k_pool, const void* v_pool,
                          const float* k_scale, const float* v_scale,
                          const int32_t* block_tables, int bt_stride,
                          const int32_t* seq_lens, int b, int kvh, double* out);

/* All groups: out is [batch][Hq][d] fp64. */
int orc_decode_attn(const orc_cfg* cfg, const uint16_t* q,
                    const void* k_pool, const void* v_pool,
                    const float* k_scale, const float* v_scale,
                    const int32_t* block_tables, int bt_stride,
                    const int32_t* seq_lens, int batch, double* out);

/* ---- several new tokens per request ---------------------------------- */
/* Speculative-decode verification: new token t (0 <= t < q_len) of request
 * b sits at position L_b + t.  q is [batch][q_len][Hq][d] (rotated in
 * place), k_new / v_new [batch][q_len][Hkv][d]; each token is rotated and
 * stored exactly as orc_rope_append stores the single new token. */
int orc_rope_append_tokens(const orc_cfg* cfg,
                           uint16_t* q, const uint16_t* k_new, const uint16_t* v_new,
                           void* k_pool, void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, int q_len);

/* New token t attends tokens 0 .. L_b + t (causal among the new tokens):
 * out[g*d + j] for the G query heads of kv head kvh. */
int orc_decode_attn_tokens_group(const orc_cfg* cfg, const uint16_t* q,
                                 const void* k_pool, const void* v_pool,
                                 const float* k_scale, const float* v_scale,
                                 const int32_t* block_tables, int bt_stride,
                                 const int32_t* seq_lens, int q_len, int b, int t, int kvh,
                                 double* out);

/* All groups: out is [batch][q_len][Hq][d] fp64. */
int orc_decode_attn_tokens(const orc_cfg* cfg, const uint16_t* q,
                           const void* k_pool, const void* v_pool,
                           const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride,
                           const int32_t* seq_lens, int batch, int q_len, double* out);

/* ---- the QKV projection ------------------------------------------------ */
/* out[t][n] = bf16_RNE(sum_j x[t][j] w[n][j]), the sum in fp64; x is
 * [T][hidden], w [N][hidden], out [T][N], all bf16 bits. */
int orc_project_bf16(const uint16_t* x, const uint16_t* w, int T, int N, int hidden, uint16_t* out);

#ifdef __cplusplus
}
#endif
#endif
