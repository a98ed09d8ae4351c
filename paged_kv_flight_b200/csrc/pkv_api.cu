// pkv_api.cu -- host side of the libpkv C ABI (include/pkv.h): validation,
// workspace ownership, TMA descriptor encoding and kernel launches.  No C++
// exception crosses the ABI (nothing here throws).
//
// Shapes are fixed when the context is created, like an engine built for one
// model and its limits ("TensorRT-LLM", section "What the build step is
// for"); errors come back per call as status codes.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>

#include <cudaTypedefs.h>

#include "pkv_internal.h"

struct pkv_ctx {
    pkv_config cfg;
    int device;
    int num_sms;
    int G;
    pkv::AttnLaunch attn;
    pkv::AttnLaunch attn_tok;     // several new tokens per request
    int workers;
    int tail_chunks;      // largest number of dynamic tail chunks per warp range
    void* ws;             // one allocation, carved below
    size_t ws_bytes;
    int* d_err;
    int* d_claim;         // chunk counter of the attention's dynamic tail
    double* d_theta;      // [head_dim / 2] rope_base^(-2i/d), fp64
    int* d_meta;
    int vmax;             // virtual requests a varlen attention call may have (bf16 pools)
    int4* d_vmap;         // [vmax] the varlen plan
    int* d_vcount;
    int prefill_rows;     // varlen requests with G x new tokens >= this go to the prefill-chunk kernel (0: none)
    int4* d_cmap;         // [vmax] its blocks
    int* d_ccount;
    float* d_part_o;
    float* d_part_ml;
    const void* tm_k_ptr;
    const void* tm_v_ptr;
    CUtensorMap tmk, tmv;
    // 16-row boxes for the several-new-tokens path where the one-token maps
    // use 32-row ones (E4M3 pools with pages of 32 tokens or more)
    const void* t16_k_ptr;
    const void* t16_v_ptr;
    CUtensorMap t16k, t16v;
    // page-high boxes (P rows) for the prefill-chunk kernel (bf16 pools)
    const void* tp_k_ptr;
    const void* tp_v_ptr;
    CUtensorMap tpk, tpv;
    const void* tm_w_ptr;        // QKV weight and input maps of pkv_qkv_rope_append
    int tm_w_hidden, tm_w_layout;
    int qkv_split;               // 0: automatic
    int plan_key[6];             // (x_rows, D, heads, tiles, hidden, forced split) of the cached plan
    pkv::QkvPlan plan;
    const void* tm_x_ptr;
    int tm_x_hidden, tm_x_rows;
    CUtensorMap tmw, tmx;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

pkv_status validate_config(const pkv_config* c)
{
    if (!c) return PKV_ERR_INVALID_ARG;
    if (c->num_q_heads <= 0 || c->num_kv_heads <= 0) return PKV_ERR_INVALID_ARG;
    if (c->num_q_heads % c->num_kv_heads) return PKV_ERR_INVALID_ARG;
    if (c->head_dim <= 0 || c->page_size <= 0) return PKV_ERR_INVALID_ARG;
    if (c->kv_dtype != PKV_KV_BF16 && c->kv_dtype != PKV_KV_FP8_E4M3) return PKV_ERR_INVALID_ARG;
    if (!(c->rope_base > 1.0) || !isfinite(c->rope_base)) return PKV_ERR_INVALID_ARG;
    if (c->max_batch <= 0 || c->max_blocks_per_seq <= 0 || c->num_pages <= 0) return PKV_ERR_INVALID_ARG;
    if ((long long)c->max_blocks_per_seq * c->page_size >= (1LL << 31)) return PKV_ERR_INVALID_ARG;
    if (c->num_q_heads / c->num_kv_heads > pkv::kMaxGroup) return PKV_ERR_UNSUPPORTED;
    if (c->head_dim != 64 && c->head_dim != 128) return PKV_ERR_UNSUPPORTED;
    if (c->page_size != 16 && c->page_size != 32 && c->page_size != 64) return PKV_ERR_UNSUPPORTED;
    if (c->max_batch > pkv::kMaxBatch) return PKV_ERR_UNSUPPORTED;
    // TMA row coordinates are int32
    if ((long long)c->num_pages * c->num_kv_heads * c->page_size >= (1LL << 31)) return PKV_ERR_UNSUPPORTED;
    return PKV_OK;
}

pkv_status check_call(const pkv_ctx* ctx, int batch, int bt_stride, const void* k_pool,
                      const void* v_pool, const float* k_scale, const float* v_scale,
                      const int32_t* block_tables, const int32_t* seq_lens)
{
    if (!ctx) return PKV_ERR_INVALID_ARG;
    if (batch < 0 || batch > ctx->cfg.max_batch) return PKV_ERR_INVALID_ARG;
    if (batch == 0) return PKV_OK;
    if (bt_stride <= 0 || bt_stride > ctx->cfg.max_blocks_per_seq) return PKV_ERR_INVALID_ARG;
    if (!k_pool || !v_pool || !block_tables || !seq_lens) return PKV_ERR_INVALID_ARG;
    if (!aligned16(k_pool) || !aligned16(v_pool) || !aligned16(block_tables) || !aligned16(seq_lens))
        return PKV_ERR_INVALID_ARG;
    if (ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3) {
        if (!k_scale || !v_scale || !aligned16(k_scale) || !aligned16(v_scale)) return PKV_ERR_INVALID_ARG;
    }
    return PKV_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// 2-D view of a pool: rows = num_pages * Hkv * P token rows of head_dim
// elements; box = one attention tile of rows (16, or 32 for E4M3 pools with
// pages of at least 32 tokens) x (128 or 64 bytes), swizzled to match the
// kernel's shared-memory addressing.
bool encode_pool_rows(const pkv_ctx* ctx, const void* pool, int box_rows, CUtensorMap* map);

bool encode_pool(const pkv_ctx* ctx, const void* pool, CUtensorMap* map)
{
    const bool fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    return encode_pool_rows(ctx, pool, pkv::attn_tile(fp8, ctx->cfg.page_size), map);
}

bool encode_pool_rows(const pkv_ctx* ctx, const void* pool, int box_rows, CUtensorMap* map)
{
    auto fn = encode_fn();
    if (!fn) return false;
    const bool fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    const int elem = fp8 ? 1 : 2;
    const int rowb = ctx->cfg.head_dim * elem;
    const int boxb = rowb > 128 ? 128 : rowb;
    cuuint64_t dims[2] = {(cuuint64_t)ctx->cfg.head_dim,
                          (cuuint64_t)ctx->cfg.num_pages * ctx->cfg.num_kv_heads * ctx->cfg.page_size};
    cuuint64_t strides[1] = {(cuuint64_t)rowb};
    cuuint32_t box[2] = {(cuuint32_t)(boxb / elem), (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                    const_cast<void*>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    boxb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D view of a row-major bf16 matrix [rows][cols] for the projection's TMA
// loads: box = box_rows x 64 elements (one 128-byte row), 128-byte swizzle,
// rows past the end read as zero.
bool encode_rows(const void* base, int rows, int cols, int box_rows, CUtensorMap* map)
{
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The cached projection plan for (batch, hidden) under the context's shapes.
bool qkv_plan_for(pkv_ctx* ctx, int batch, int hidden)
{
    const int x_rows = batch >= 128 ? 128 : (batch + 15) / 16 * 16;
    const int heads = ctx->cfg.num_q_heads + 2 * ctx->cfg.num_kv_heads, tiles = (batch + 127) / 128;
    const int key[6] = {x_rows, ctx->cfg.head_dim, heads, tiles, hidden, ctx->qkv_split};
    if (memcmp(key, ctx->plan_key, sizeof(key)) == 0) return true;
    if (pkv::qkv_plan(x_rows, ctx->cfg.head_dim, heads, tiles, hidden, ctx->num_sms, ctx->qkv_split,
                      &ctx->plan) != cudaSuccess)
        return false;
    memcpy(ctx->plan_key, key, sizeof(key));
    return true;
}

}  // namespace

extern "C" {

pkv_status pkv_create(const pkv_config* cfg, pkv_ctx** out)
{
    if (!out) return PKV_ERR_INVALID_ARG;
    const pkv_status v = validate_config(cfg);
    if (v != PKV_OK) return v;

    pkv_ctx* ctx = static_cast<pkv_ctx*>(calloc(1, sizeof(pkv_ctx)));
    if (!ctx) return PKV_ERR_OOM;
    ctx->cfg = *cfg;
    ctx->G = cfg->num_q_heads / cfg->num_kv_heads;
    if (cudaGetDevice(&ctx->device) != cudaSuccess ||
        cudaDeviceGetAttribute(&ctx->num_sms, cudaDevAttrMultiProcessorCount, ctx->device) != cudaSuccess) {
        free(ctx);
        return PKV_ERR_CUDA;
    }
    const bool fp8 = cfg->kv_dtype == PKV_KV_FP8_E4M3;
    if (pkv::attn_prepare(cfg->head_dim, fp8, cfg->page_size, ctx->num_sms, cfg->max_batch, &ctx->attn) !=
        cudaSuccess) {
        free(ctx);
        return PKV_ERR_CUDA;
    }
    // varlen calls cut requests into virtual ones: room for 4 per request
    ctx->vmax = std::min(4 * cfg->max_batch, pkv::kMaxBatch);
    if (pkv::attn_tokens_prepare(cfg->head_dim, fp8, ctx->num_sms, std::max(cfg->max_batch, ctx->vmax),
                                 &ctx->attn_tok) != cudaSuccess) {
        free(ctx);
        return PKV_ERR_CUDA;
    }
    if (pkv::qkv_prepare() != cudaSuccess || pkv::chunk_attn_prepare(cfg->head_dim) != cudaSuccess) {
        free(ctx);
        return PKV_ERR_CUDA;
    }

    // [error word, chunk counter | split geometry | partial rows | partial (m, l)];
    // two partial slots per unit of the split: G rows each for one new token
    // per request (up to kMaxTailChunks + 1 units per warp), up to
    // kMaxTokenRows rows for several (one unit per warp)
    const size_t units = pkv::max_units(ctx->attn.ctas * pkv::kAttnWarps, pkv::kMaxTailChunks);
    const size_t rows_units = std::max(units * ctx->G, (size_t)ctx->attn.ctas * pkv::kAttnWarps * pkv::kMaxTokenRows);
    const size_t b_err = 256;
    const size_t b_cnt = ((size_t)(std::max(cfg->max_batch, ctx->vmax) + 8) * sizeof(int) + 255) & ~(size_t)255;
    const size_t b_po = 2 * rows_units * cfg->head_dim * sizeof(float);
    const size_t b_pml = 2 * rows_units * 2 * sizeof(float);
    const size_t b_vm = 2 * ((size_t)ctx->vmax * sizeof(int4) + 256);   // varlen plans (virtual, chunk) + counts
    const size_t b_th = ((size_t)cfg->head_dim / 2 * sizeof(double) + 255) & ~(size_t)255;   // RoPE frequencies
    ctx->ws_bytes = b_err + b_cnt + b_po + b_pml + b_vm + b_th;
    if (cudaMalloc(&ctx->ws, ctx->ws_bytes) != cudaSuccess) {
        cudaGetLastError();
        free(ctx);
        return PKV_ERR_OOM;
    }
    uint8_t* base = static_cast<uint8_t*>(ctx->ws);
    ctx->d_err = reinterpret_cast<int*>(base);
    ctx->d_claim = reinterpret_cast<int*>(base + 128);
    ctx->tail_chunks = pkv::kDefaultTailChunks;
    ctx->d_meta = reinterpret_cast<int*>(base + b_err);
    ctx->d_part_o = reinterpret_cast<float*>(base + b_err + b_cnt);
    ctx->d_part_ml = reinterpret_cast<float*>(base + b_err + b_cnt + b_po);
    ctx->d_vcount = reinterpret_cast<int*>(base + b_err + b_cnt + b_po + b_pml);
    ctx->d_vmap = reinterpret_cast<int4*>(base + b_err + b_cnt + b_po + b_pml + 256);
    ctx->d_ccount = reinterpret_cast<int*>(base + b_err + b_cnt + b_po + b_pml + b_vm / 2);
    ctx->d_cmap = reinterpret_cast<int4*>(base + b_err + b_cnt + b_po + b_pml + b_vm / 2 + 256);
    ctx->prefill_rows = pkv::kDefaultPrefillRows;
    ctx->d_theta = reinterpret_cast<double*>(base + b_err + b_cnt + b_po + b_pml + b_vm);
    // theta_i = rope_base^(-2i/d) once, in fp64 on the host
    double theta[64];
    for (int i = 0; i < cfg->head_dim / 2; ++i) theta[i] = pow(cfg->rope_base, (-2.0 * i) / cfg->head_dim);
    if (cudaMemset(ctx->ws, 0, b_err + b_cnt) != cudaSuccess ||
        cudaMemcpy(ctx->d_theta, theta, sizeof(double) * (size_t)(cfg->head_dim / 2), cudaMemcpyHostToDevice) !=
            cudaSuccess) {
        cudaFree(ctx->ws);
        free(ctx);
        return PKV_ERR_CUDA;
    }
    *out = ctx;
    return PKV_OK;
}

pkv_status pkv_rope_append(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new, void* k_pool,
                           void* v_pool, const float* k_scale, const float* v_scale,
                           const int32_t* block_tables, int bt_stride, const int32_t* seq_lens, int batch,
                           cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (!q || !k_new || !v_new || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new))
        return PKV_ERR_INVALID_ARG;

    pkv::RopeParams p;
    p.q = static_cast<__nv_bfloat16*>(q);
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = ctx->d_err;
    p.rope_base = ctx->cfg.rope_base;
    p.theta = ctx->d_theta;
    p.prefetch_tables = 1;
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.D = ctx->cfg.head_dim;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    p.q_len = 1;
    return pkv::launch_rope_append(p, stream) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // extern "C"

namespace {

// pkv_decode_attn after its checks; pdl: as a programmatic dependent of the
// RoPE + append kernel just launched on the stream (pkv_decode_step only).
pkv_status decode_attn_launch(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                              const float* k_scale, const float* v_scale, const int32_t* block_tables,
                              int bt_stride, const int32_t* seq_lens, int batch, void* out,
                              cudaStream_t stream, bool pdl)
{

    if (ctx->tm_k_ptr != k_pool) {
        if (!encode_pool(ctx, k_pool, &ctx->tmk)) return PKV_ERR_CUDA;
        ctx->tm_k_ptr = k_pool;
    }
    if (ctx->tm_v_ptr != v_pool) {
        if (!encode_pool(ctx, v_pool, &ctx->tmv)) return PKV_ERR_CUDA;
        ctx->tm_v_ptr = v_pool;
    }

    pkv::AttnParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.part_o = ctx->d_part_o;
    p.part_ml = ctx->d_part_ml;
    p.meta = ctx->d_meta;
    p.err = ctx->d_err;
    p.claim = ctx->d_claim;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)ctx->cfg.head_dim));
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.G = ctx->G;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.stages = ctx->attn.stages;
    p.workers = ctx->workers;
    p.tail_chunks = ctx->tail_chunks;
    p.q_len = 1;
    const cudaError_t e = pkv::launch_decode_attn(p, ctx->tmk, ctx->tmv, ctx->cfg.head_dim,
                                                  ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3, ctx->attn, stream, pdl);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace

extern "C" {

pkv_status pkv_decode_attn(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                           const float* k_scale, const float* v_scale, const int32_t* block_tables,
                           int bt_stride, const int32_t* seq_lens, int batch, void* out,
                           cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (!q || !out || !aligned16(q) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    return decode_attn_launch(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride, seq_lens, batch,
                              out, stream, false);
}

pkv_status pkv_rope_append_tokens(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new, void* k_pool,
                                  void* v_pool, const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride, const int32_t* seq_lens, int batch,
                                  int q_len, cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (q_len < 1 || (long long)batch * q_len > (1LL << 31) - 1) return PKV_ERR_INVALID_ARG;
    if (!q || !k_new || !v_new || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new))
        return PKV_ERR_INVALID_ARG;

    pkv::RopeParams p;
    p.q = static_cast<__nv_bfloat16*>(q);
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = ctx->d_err;
    p.rope_base = ctx->cfg.rope_base;
    p.theta = ctx->d_theta;
    p.prefetch_tables = 1;
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.D = ctx->cfg.head_dim;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    p.q_len = q_len;
    return pkv::launch_rope_append(p, stream) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // extern "C"

namespace {

// The several-new-tokens attention launch, for the uniform calls (vmap null:
// `batch` requests of q_len tokens) and the varlen ones (batch = the plan's
// capacity, q_len = the block length).
pkv_status attn_tokens_launch(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                              const float* k_scale, const float* v_scale, const int32_t* block_tables,
                              int bt_stride, const int32_t* seq_lens, int batch, int q_len, const int4* vmap,
                              const int* vcount, void* out, cudaStream_t stream, bool pdl = false)
{
    const bool fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    const CUtensorMap* mk = &ctx->tmk;
    const CUtensorMap* mv = &ctx->tmv;
    if (pkv::attn_tile(fp8, ctx->cfg.page_size) == pkv::kTile) {
        // the one-token maps already have 16-row boxes
        if (ctx->tm_k_ptr != k_pool) {
            if (!encode_pool(ctx, k_pool, &ctx->tmk)) return PKV_ERR_CUDA;
            ctx->tm_k_ptr = k_pool;
        }
        if (ctx->tm_v_ptr != v_pool) {
            if (!encode_pool(ctx, v_pool, &ctx->tmv)) return PKV_ERR_CUDA;
            ctx->tm_v_ptr = v_pool;
        }
    } else {
        if (ctx->t16_k_ptr != k_pool) {
            if (!encode_pool_rows(ctx, k_pool, pkv::kTile, &ctx->t16k)) return PKV_ERR_CUDA;
            ctx->t16_k_ptr = k_pool;
        }
        if (ctx->t16_v_ptr != v_pool) {
            if (!encode_pool_rows(ctx, v_pool, pkv::kTile, &ctx->t16v)) return PKV_ERR_CUDA;
            ctx->t16_v_ptr = v_pool;
        }
        mk = &ctx->t16k;
        mv = &ctx->t16v;
    }

    pkv::AttnParams p;
    p.q = static_cast<const __nv_bfloat16*>(q);
    p.out = static_cast<__nv_bfloat16*>(out);
    p.k_scale = fp8 ? k_scale : nullptr;
    p.v_scale = fp8 ? v_scale : nullptr;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.part_o = ctx->d_part_o;
    p.part_ml = ctx->d_part_ml;
    p.meta = ctx->d_meta;
    p.err = ctx->d_err;
    p.claim = ctx->d_claim;
    p.scale_log2 = (float)(1.4426950408889634 / sqrt((double)ctx->cfg.head_dim));
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.G = ctx->G;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.stages = ctx->attn_tok.stages;
    p.workers = ctx->workers;
    p.tail_chunks = 0;
    p.q_len = q_len;
    p.vmap = vmap;
    p.vcount = vcount;
    const cudaError_t e = pkv::launch_decode_attn_tokens(p, *mk, *mv, ctx->cfg.head_dim, fp8, ctx->attn_tok, stream,
                                                         pdl);
    return e == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

}  // namespace

extern "C" {

pkv_status pkv_decode_attn_tokens(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                                  const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                  int bt_stride, const int32_t* seq_lens, int batch, int q_len, void* out,
                                  cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (q_len < 1) return PKV_ERR_INVALID_ARG;
    if ((long long)ctx->G * q_len > pkv::kMaxTokenRows) return PKV_ERR_UNSUPPORTED;
    if (!q || !out || !aligned16(q) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    return attn_tokens_launch(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride, seq_lens, batch,
                              q_len, nullptr, nullptr, out, stream);
}

pkv_status pkv_decode_step(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new, void* k_pool,
                           void* v_pool, const float* k_scale, const float* v_scale, const int32_t* block_tables,
                           int bt_stride, const int32_t* seq_lens, int batch, int q_len, void* out,
                           cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (q_len < 1 || (long long)batch * q_len > (1LL << 31) - 1) return PKV_ERR_INVALID_ARG;
    if (q_len > 1 && (long long)ctx->G * q_len > pkv::kMaxTokenRows) return PKV_ERR_UNSUPPORTED;
    if (!q || !k_new || !v_new || !out || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new) ||
        !aligned16(out))
        return PKV_ERR_INVALID_ARG;
    st = pkv_rope_append_tokens(ctx, q, k_new, v_new, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride,
                                seq_lens, batch, q_len, stream);
    if (st != PKV_OK) return st;
    // the attention starts its prologue while the RoPE + append kernel runs
    if (q_len == 1)
        return decode_attn_launch(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride, seq_lens,
                                  batch, out, stream, true);
    return attn_tokens_launch(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride, seq_lens, batch,
                              q_len, nullptr, nullptr, out, stream, true);
}

pkv_status pkv_rope_append_varlen(pkv_ctx* ctx, void* q, const void* k_new, const void* v_new, void* k_pool,
                                  void* v_pool, const float* k_scale, const float* v_scale,
                                  const int32_t* block_tables, int bt_stride, const int32_t* seq_lens,
                                  const int32_t* cu_q, int batch, int n_tokens, cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK) return st;
    if (n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (batch == 0 || n_tokens == 0) return PKV_OK;
    if (!cu_q || !aligned16(cu_q)) return PKV_ERR_INVALID_ARG;
    if (!q || !k_new || !v_new || !aligned16(q) || !aligned16(k_new) || !aligned16(v_new))
        return PKV_ERR_INVALID_ARG;

    pkv::RopeParams p;
    p.q = static_cast<__nv_bfloat16*>(q);
    p.k_new = static_cast<const __nv_bfloat16*>(k_new);
    p.v_new = static_cast<const __nv_bfloat16*>(v_new);
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.block_tables = block_tables;
    p.seq_lens = seq_lens;
    p.err = ctx->d_err;
    p.rope_base = ctx->cfg.rope_base;
    p.theta = ctx->d_theta;
    p.prefetch_tables = 1;
    p.batch = batch;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.D = ctx->cfg.head_dim;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    p.q_len = 1;
    p.cu_q = cu_q;
    p.n_tokens = n_tokens;
    return pkv::launch_rope_append(p, stream) == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}

pkv_status pkv_decode_attn_varlen(pkv_ctx* ctx, const void* q, const void* k_pool, const void* v_pool,
                                  const float* k_scale, const float* v_scale, const int32_t* block_tables,
                                  int bt_stride, const int32_t* seq_lens, const int32_t* cu_q, int batch,
                                  int n_tokens, void* out, cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK) return st;
    if (n_tokens < 0) return PKV_ERR_INVALID_ARG;
    if (batch == 0 || n_tokens == 0) return PKV_OK;
    if (!cu_q || !aligned16(cu_q) || !q || !out || !aligned16(q) || !aligned16(out)) return PKV_ERR_INVALID_ARG;
    // blocks of `block` new tokens: G x block <= 16 query rows per (block, kv head)
    const int block = pkv::kMaxTokenRows / ctx->G;
    if ((long long)batch + (n_tokens + block - 1) / block > ctx->vmax) return PKV_ERR_UNSUPPORTED;
    // requests with at least cmin new tokens: blocks of cblock on the tensor
    // cores (bf16 pools).  At most min(batch, n_tokens / cmin) requests take
    // that path, so it has at most n_tokens / cblock + that many blocks: within
    // vmax (>= batch + n_tokens / block) by the check above
    const bool fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    const int cblock = pkv::kChunkRows / ctx->G;
    const int cmin = (!fp8 && ctx->prefill_rows > 0) ? std::max(1, (ctx->prefill_rows + ctx->G - 1) / ctx->G) : 0;
    const long long creq = cmin > 0 ? std::min<long long>(batch, n_tokens / cmin) : 0;
    const int citems = creq > 0 ? (int)std::min<long long>(ctx->vmax, (long long)n_tokens / cblock + creq) : 0;
    if (pkv::launch_varlen_plan(cu_q, seq_lens, batch, block, ctx->vmax, ctx->d_vmap, ctx->d_vcount, cmin, cblock,
                                ctx->vmax, cmin > 0 ? ctx->d_cmap : nullptr, ctx->d_ccount, ctx->d_err,
                                stream) != cudaSuccess)
        return PKV_ERR_CUDA;
    if (citems > 0) {
        if (ctx->tp_k_ptr != k_pool) {
            if (!encode_pool_rows(ctx, k_pool, ctx->cfg.page_size, &ctx->tpk)) return PKV_ERR_CUDA;
            ctx->tp_k_ptr = k_pool;
        }
        if (ctx->tp_v_ptr != v_pool) {
            if (!encode_pool_rows(ctx, v_pool, ctx->cfg.page_size, &ctx->tpv)) return PKV_ERR_CUDA;
            ctx->tp_v_ptr = v_pool;
        }
        pkv::AttnParams cp;
        cp.q = static_cast<const __nv_bfloat16*>(q);
        cp.out = static_cast<__nv_bfloat16*>(out);
        cp.k_scale = nullptr;
        cp.v_scale = nullptr;
        cp.block_tables = block_tables;
        cp.seq_lens = seq_lens;
        cp.part_o = nullptr;
        cp.part_ml = nullptr;
        cp.meta = nullptr;
        cp.err = ctx->d_err;
        cp.claim = nullptr;
        cp.scale_log2 = (float)(1.4426950408889634 / sqrt((double)ctx->cfg.head_dim));
        cp.batch = batch;
        cp.bt_stride = bt_stride;
        cp.Hq = ctx->cfg.num_q_heads;
        cp.Hkv = ctx->cfg.num_kv_heads;
        cp.G = ctx->G;
        cp.P = ctx->cfg.page_size;
        cp.num_pages = ctx->cfg.num_pages;
        cp.stages = 0;
        cp.workers = 0;
        cp.tail_chunks = 0;
        cp.q_len = cblock;
        cp.cmap = ctx->d_cmap;
        cp.ccount = ctx->d_ccount;
        if (pkv::launch_chunk_attn(cp, ctx->tpk, ctx->tpv, ctx->cfg.head_dim, citems, stream) != cudaSuccess)
            return PKV_ERR_CUDA;
    }
    return attn_tokens_launch(ctx, q, k_pool, v_pool, k_scale, v_scale, block_tables, bt_stride, seq_lens,
                              ctx->vmax, block, ctx->d_vmap, ctx->d_vcount, out, stream);
}

pkv_status pkv_qkv_pack_weight(pkv_ctx* ctx, const void* w_qkv, int hidden, void* w_tiled, cudaStream_t stream)
{
    if (!ctx || !w_qkv || !w_tiled || !aligned16(w_qkv) || !aligned16(w_tiled)) return PKV_ERR_INVALID_ARG;
    if (hidden < 64 || hidden % 64 != 0) return PKV_ERR_UNSUPPORTED;
    const int N = (ctx->cfg.num_q_heads + 2 * ctx->cfg.num_kv_heads) * ctx->cfg.head_dim;
    const size_t bytes = (size_t)N * hidden * 2;
    const uintptr_t a = reinterpret_cast<uintptr_t>(w_qkv), b = reinterpret_cast<uintptr_t>(w_tiled);
    if (a < b + bytes && b < a + bytes) return PKV_ERR_INVALID_ARG;
    return pkv::launch_qkv_pack_weight(static_cast<const __nv_bfloat16*>(w_qkv), static_cast<__nv_bfloat16*>(w_tiled),
                                       N, hidden, ctx->cfg.head_dim, stream) == cudaSuccess
               ? PKV_OK
               : PKV_ERR_CUDA;
}

pkv_status pkv_qkv_rope_append(pkv_ctx* ctx, const void* x, const void* w_qkv, int hidden, int w_layout,
                               void* q_out, void* k_pool, void* v_pool, const float* k_scale, const float* v_scale,
                               const int32_t* block_tables, int bt_stride, const int32_t* seq_lens, int batch,
                               cudaStream_t stream)
{
    pkv_status st = check_call(ctx, batch, bt_stride, k_pool, v_pool, k_scale, v_scale, block_tables, seq_lens);
    if (st != PKV_OK || batch == 0) return st;
    if (w_layout != PKV_W_ROWS && w_layout != PKV_W_TILED) return PKV_ERR_INVALID_ARG;
    if (hidden < 64 || hidden % 64 != 0) return PKV_ERR_UNSUPPORTED;
    if (!x || !w_qkv || !q_out || !aligned16(x) || !aligned16(w_qkv) || !aligned16(q_out))
        return PKV_ERR_INVALID_ARG;
    const int N = (ctx->cfg.num_q_heads + 2 * ctx->cfg.num_kv_heads) * ctx->cfg.head_dim;
    if (ctx->tm_w_ptr != w_qkv || ctx->tm_w_hidden != hidden || ctx->tm_w_layout != w_layout) {
        // tiled: a 2-D view of 64-element rows, one box = the d rows of one
        // (head, 64-slice) run
        const bool ok = w_layout == PKV_W_TILED
                            ? encode_rows(w_qkv, N * (hidden / 64), 64, ctx->cfg.head_dim, &ctx->tmw)
                            : encode_rows(w_qkv, N, hidden, ctx->cfg.head_dim, &ctx->tmw);
        if (!ok) return PKV_ERR_CUDA;
        ctx->tm_w_ptr = w_qkv;
        ctx->tm_w_hidden = hidden;
        ctx->tm_w_layout = w_layout;
    }
    const int x_rows = batch >= 128 ? 128 : (batch + 15) / 16 * 16;
    if (ctx->tm_x_ptr != x || ctx->tm_x_hidden != hidden || ctx->tm_x_rows != batch) {
        if (!encode_rows(x, batch, hidden, x_rows, &ctx->tmx)) return PKV_ERR_CUDA;
        ctx->tm_x_ptr = x;
        ctx->tm_x_hidden = hidden;
        ctx->tm_x_rows = batch;
    }
    pkv::QkvParams p;
    p.seq_lens = seq_lens;
    p.block_tables = block_tables;
    p.q_out = static_cast<__nv_bfloat16*>(q_out);
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_scale = k_scale;
    p.v_scale = v_scale;
    p.err = ctx->d_err;
    p.rope_base = ctx->cfg.rope_base;
    p.theta = ctx->d_theta;
    p.batch = batch;
    p.hidden = hidden;
    p.bt_stride = bt_stride;
    p.Hq = ctx->cfg.num_q_heads;
    p.Hkv = ctx->cfg.num_kv_heads;
    p.D = ctx->cfg.head_dim;
    p.P = ctx->cfg.page_size;
    p.num_pages = ctx->cfg.num_pages;
    p.fp8 = ctx->cfg.kv_dtype == PKV_KV_FP8_E4M3;
    p.x_rows = x_rows;
    p.w_tiled = w_layout == PKV_W_TILED;
    if (!qkv_plan_for(ctx, batch, hidden)) return PKV_ERR_CUDA;
    return pkv::launch_qkv_rope_append(p, ctx->plan, ctx->tmx, ctx->tmw, stream) == cudaSuccess ? PKV_OK
                                                                                                : PKV_ERR_CUDA;
}

pkv_status pkv_destroy(pkv_ctx* ctx)
{
    if (!ctx) return PKV_OK;
    pkv_status st = PKV_OK;
    if (cudaDeviceSynchronize() != cudaSuccess) st = PKV_ERR_CUDA;
    if (ctx->ws && cudaFree(ctx->ws) != cudaSuccess) st = PKV_ERR_CUDA;
    free(ctx);
    return st;
}

const char* pkv_status_str(pkv_status s)
{
    switch (s) {
    case PKV_OK: return "ok";
    case PKV_ERR_INVALID_ARG: return "invalid argument";
    case PKV_ERR_UNSUPPORTED: return "unsupported configuration";
    case PKV_ERR_CUDA: return "CUDA error";
    case PKV_ERR_OOM: return "out of device memory";
    case PKV_ERR_DEVICE_BOUNDS: return "device saw a page id or length out of range";
    case PKV_ERR_DEVICE_TIMEOUT: return "a bounded wait inside a kernel timed out";
    }
    return "unknown status";
}

pkv_status pkv_check_device_error(pkv_ctx* ctx, cudaStream_t stream, int* bits)
{
    if (!ctx) return PKV_ERR_INVALID_ARG;
    int word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return PKV_ERR_CUDA;
    if (cudaMemcpy(&word, ctx->d_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return PKV_ERR_CUDA;
    if (word && cudaMemset(ctx->d_err, 0, sizeof(int)) != cudaSuccess) return PKV_ERR_CUDA;
    if (bits) *bits = word;
    if (word & pkv::kErrTimeout) return PKV_ERR_DEVICE_TIMEOUT;
    if (word & (pkv::kErrLength | pkv::kErrPage)) return PKV_ERR_DEVICE_BOUNDS;
    return PKV_OK;
}

pkv_status pkv_set_workers(pkv_ctx* ctx, int workers)
{
    if (!ctx || workers < 0) return PKV_ERR_INVALID_ARG;
    ctx->workers = workers;
    return PKV_OK;
}

pkv_status pkv_qkv_launch_shape(pkv_ctx* ctx, int batch, int hidden, int* shape)
{
    if (!ctx || !shape || batch <= 0 || batch > ctx->cfg.max_batch) return PKV_ERR_INVALID_ARG;
    if (hidden < 64 || hidden % 64 != 0) return PKV_ERR_UNSUPPORTED;
    if (!qkv_plan_for(ctx, batch, hidden)) return PKV_ERR_CUDA;
    shape[0] = ctx->plan.split;
    shape[1] = ctx->plan.stages;
    shape[2] = (int)ctx->plan.smem;
    shape[3] = ctx->plan.max_clusters;
    return PKV_OK;
}

pkv_status pkv_set_qkv_split(pkv_ctx* ctx, int split)
{
    if (!ctx || split < 0 || split > pkv::kQkvMaxSplit) return PKV_ERR_INVALID_ARG;
    ctx->qkv_split = split;
    return PKV_OK;
}

pkv_status pkv_set_tail_chunks(pkv_ctx* ctx, int max_chunks)
{
    if (!ctx || max_chunks < pkv::kTailAuto || max_chunks > pkv::kMaxTailChunks) return PKV_ERR_INVALID_ARG;
    ctx->tail_chunks = max_chunks;
    return PKV_OK;
}

pkv_status pkv_set_prefill_rows(pkv_ctx* ctx, int rows)
{
    if (!ctx || rows < 0 || rows > pkv::kChunkRows) return PKV_ERR_INVALID_ARG;
    ctx->prefill_rows = rows;
    return PKV_OK;
}

size_t pkv_workspace_bytes(const pkv_ctx* ctx) { return ctx ? ctx->ws_bytes : 0; }

}  // extern "C"
