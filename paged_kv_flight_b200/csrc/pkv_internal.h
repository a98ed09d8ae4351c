// pkv_internal.h -- structures shared by the host API (pkv_api.cu) and the
// kernel launchers (rope_append.cu, decode_attn.cu).  Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "../../include/pkv.h"

namespace pkv {

// Device error bits (sticky word in the context workspace).
enum : int { kErrLength = 1, kErrPage = 2, kErrTimeout = 4 };

// Warps per attention CTA (one CTA per SM) and the deepest per-warp TMA
// ring; both can be overridden at build time for tuning sweeps.
#ifndef PKV_ATTN_WARPS
#define PKV_ATTN_WARPS 8
#endif
#ifndef PKV_ATTN_MAX_STAGES
#define PKV_ATTN_MAX_STAGES 2
#endif

constexpr int kTile = 16;          // tokens per attention tile (one TMA box height)
constexpr int kTileWide = 32;      // E4M3 tiles when pages hold at least 32 tokens

// Tokens per tile of the one-new-token attention: 32 for E4M3 pools whose
// pages hold a whole 32-token tile (the same bytes as a 16-token bf16 tile,
// half the per-tile work per token), else 16.
inline int attn_tile(bool fp8, int page_size) { return (fp8 && page_size >= kTileWide) ? kTileWide : kTile; }
constexpr int kMaxGroup = 8;       // query heads per kv head handled by one mma row block
constexpr int kMaxTokenRows = 16;  // G x q_len rows of the several-new-tokens attention
// Prefill chunks of a varlen call on the tensor cores (chunk_attn.cu): blocks
// of kChunkRows / G new tokens (G x that query rows), tiles of kChunkKeys
// keys; a request takes that path when it has at least kDefaultPrefillRows / G
// new tokens (pkv_set_prefill_rows; 0: never).
constexpr int kChunkRows = 128;
constexpr int kChunkKeys = 128;
constexpr int kDefaultPrefillRows = 64;
constexpr int kAttnWarps = PKV_ATTN_WARPS;
constexpr int kAttnMaxStages = PKV_ATTN_MAX_STAGES;
constexpr int kMinTilesPerWorker = 8;
constexpr int kMaxBatch = 8192;

// Dynamic tail of the attention split: the last 1/kTailDen of every warp's
// range (at most kTailMaxTiles tiles) is cut into at most kMaxTailChunks
// chunks of at least kTailChunkTiles tiles that any warp may claim once its
// own static part is done.  Only applies when every warp range holds at
// least kTailMinTiles tiles.
constexpr int kTailDen = 4;
constexpr int kTailMaxTiles = 48;
constexpr int kTailChunkTiles = 4;
constexpr int kTailMinTiles = 32;
constexpr int kMaxTailChunks = 8;
// a chunk must outlast the producer's lead over the consumer (see decode_attn.cu)
static_assert(kTailChunkTiles > PKV_ATTN_MAX_STAGES, "tail chunks must be longer than the TMA ring");
// -1 (the default): automatic, kAutoTailChunks chunks when every warp range
// holds at least kAutoTailTiles tiles (long contexts, where a chunk's fresh
// page lookahead and query load are amortised), a static split otherwise
constexpr int kTailAuto = -1;
constexpr int kAutoTailChunks = 4;
constexpr int kAutoTailTiles = 192;
constexpr int kDefaultTailChunks = kTailAuto;

// Units the split may cut the tiles into (two partial slots each).
inline size_t max_units(int max_workers, int tail_chunks)
{
    return (size_t)max_workers * (size_t)(tail_chunks + 1);
}

struct RopeParams {
    __nv_bfloat16* q;
    const __nv_bfloat16* k_new;
    const __nv_bfloat16* v_new;
    void* k_pool;
    void* v_pool;
    const float* k_scale;
    const float* v_scale;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    int* err;
    double rope_base;
    int batch, bt_stride, Hq, Hkv, D, P, num_pages, fp8;
    int q_len;            // new tokens per request, at positions L_b .. L_b + q_len - 1
    // varlen: token i of request b (cu_q[b] <= i < cu_q[b + 1]) sits at
    // position L_b + i - cu_q[b]; the grid covers n_tokens rows; q_len unused
    const int32_t* cu_q = nullptr;
    int n_tokens = 0;
    const double* theta = nullptr;   // [D / 2] rope_base^(-2i/D) in fp64, from the context
    int prefetch_tables = 0;         // 1: prefetch each request's block-table row into L2
};

struct AttnParams {
    const __nv_bfloat16* q;
    __nv_bfloat16* out;
    const float* k_scale;
    const float* v_scale;
    const int32_t* block_tables;
    const int32_t* seq_lens;
    float* part_o;        // [2 * units][G][D] fp32, unnormalised
    float* part_ml;       // [2 * units][G][2] fp32 (m in log2 units, l)
    int* meta;            // [4 + max_batch + 1]: W, T (lo, hi), K, tile prefix; written by the attention kernel for the combine
    int* err;
    int* claim;           // chunk counter of the dynamic tail; zero when a launch starts, reset by the combine
    float scale_log2;     // log2(e) / sqrt(d)
    int batch, bt_stride, Hq, Hkv, G, P, num_pages;
    int stages;           // pipeline depth per warp
    int workers;          // 0: automatic
    int tail_chunks;      // largest K (chunks per warp tail); 0: static split only; kTailAuto: automatic
    int q_len;            // new tokens per request (1: one new token); partial rows = G x q_len
    // varlen (several new tokens, a different count per request): the kernel
    // works on virtual requests, blocks of at most q_len new tokens of one
    // request; vmap[v] = {request, first token row, tokens, position of the
    // first}, *vcount of them (at most batch), both written on the device by
    // the varlen plan; null for the other calls
    const int4* vmap = nullptr;
    const int* vcount = nullptr;
    // varlen prefill blocks for chunk_attn (same entries as vmap, blocks of
    // kChunkRows / G tokens), *ccount of them
    const int4* cmap = nullptr;
    const int* ccount = nullptr;
    // the combine of the one-token attention runs as its programmatic
    // dependent (own_split = 1): it derives the split itself from seq_lens
    // (tiles of `tile` tokens over `grid_warps` warps, as the attention did)
    // before it waits for the attention grid, instead of reading meta after
    int own_split = 0;
    int tile = 0;
    int grid_warps = 0;
};

cudaError_t launch_rope_append(const RopeParams& p, cudaStream_t stream);

// Host-side shape of the attention launch for a given head_dim / kv type.
struct AttnLaunch {
    int ctas;
    int stages;
    size_t smem_bytes;
    int tile;             // tokens per tile (attn_tile)
};
cudaError_t attn_prepare(int head_dim, bool fp8, int page_size, int num_sms, int max_batch, AttnLaunch* out);
// pdl: launch the attention as a programmatic dependent of the kernel before
// it on the stream (only where that kernel is this library's RoPE + append,
// which triggers its dependents at once and writes nothing the attention's
// prologue reads).
cudaError_t launch_decode_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                               int head_dim, bool fp8, const AttnLaunch& L, cudaStream_t stream,
                               bool pdl = false);

// Attention of several new tokens per request (decode_attn_tokens.cu, bf16
// or E4M3 pools with 16-token tiles, G x q_len <= 16): shape of its launch
// and the launch itself (attention, then the combine).
cudaError_t attn_tokens_prepare(int head_dim, bool fp8, int num_sms, int max_batch, AttnLaunch* out);
// The virtual requests of a varlen call: blocks of `block` new tokens (the
// last of a request may be shorter) of requests with cu_q[b + 1] > cu_q[b];
// writes vmap and the count (capped at vmax; more sets kErrLength).  With
// cmin > 0 a request of at least cmin new tokens goes instead to cmap in
// blocks of cblock tokens (capped at cmax), for the prefill-chunk kernel.
cudaError_t launch_varlen_plan(const int32_t* cu_q, const int32_t* seq_lens, int batch, int block, int vmax,
                               int4* vmap, int* vcount, int cmin, int cblock, int cmax, int4* cmap,
                               int* ccount, int* err, cudaStream_t stream);
// The prefill-chunk attention (chunk_attn.cu, bf16 pools): sets its shared-
// memory limit once, and launches max_items x Hkv CTAs for p.cmap (the CTAs
// past *p.ccount return at once).  It writes its rows of p.out directly.
cudaError_t chunk_attn_prepare(int head_dim);
cudaError_t launch_chunk_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                              int max_items, cudaStream_t stream);
cudaError_t launch_decode_attn_tokens(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                      int head_dim, bool fp8, const AttnLaunch& L, cudaStream_t stream,
                                      bool pdl = false);

// QKV projection of the new tokens on tcgen05, fused with RoPE and the append
// (qkv_rope_append.cu).
constexpr int kQkvMaxSplit = 4;   // CTAs (one cluster) that share a head's hidden dimension

struct QkvParams {
    const int32_t* seq_lens;
    const int32_t* block_tables;
    __nv_bfloat16* q_out;     // [batch][Hq][D], rotated
    void* k_pool;
    void* v_pool;
    const float* k_scale;
    const float* v_scale;
    int* err;
    double rope_base;
    const double* theta;      // [D / 2] rope_base^(-2i/D) in fp64, from the context
    int batch, hidden, bt_stride, Hq, Hkv, D, P, num_pages, fp8;
    int x_rows;               // token rows per x TMA box: min(128, batch rounded up to 16)
    int w_tiled;              // 1: weights in the tiled layout of pkv_qkv_pack_weight
    int split;                // hidden-dimension split = cluster size (set from the plan)
    int stages;               // ring depth (set from the plan)
    int ring_bytes;           // ring area; the rotation table follows it (set from the plan)
};

// Launch shape of the projection for one (x_rows, D, heads, token tiles,
// hidden): the split, the ring and the shared memory.
struct QkvPlan {
    int split, stages, ring_bytes;
    size_t smem;
    int max_clusters;         // clusters of this shape the GPU holds at once (0: unknown)
};
cudaError_t qkv_prepare();
cudaError_t qkv_plan(int x_rows, int D, int heads, int tiles, int hidden, int num_sms, int forced_split,
                     QkvPlan* out);
cudaError_t launch_qkv_rope_append(const QkvParams& p, const QkvPlan& plan, const CUtensorMap& tmx,
                                   const CUtensorMap& tmw, cudaStream_t stream);
// Copies w [N][hidden] into the tiled layout [N / D][hidden / 64][D][64].
cudaError_t launch_qkv_pack_weight(const __nv_bfloat16* w, __nv_bfloat16* out, int N, int hidden, int D,
                                   cudaStream_t stream);

// The split combine (combine.cu), run after either attention kernel: sets its
// shared-memory limits once per head_dim, and launches it for p (max_units_n:
// units the split may use; ctas: attention CTAs, for the choice of mode).
// dependent (one new token per request, p.tile and p.grid_warps set): the
// combine is the attention's programmatic dependent and derives the split
// from seq_lens while that grid runs; otherwise it reads the split from meta.
cudaError_t combine_prepare(int head_dim);
cudaError_t launch_combine(const AttnParams& p, int head_dim, int max_units_n, int ctas, cudaStream_t stream,
                           bool dependent = false);

}  // namespace pkv
