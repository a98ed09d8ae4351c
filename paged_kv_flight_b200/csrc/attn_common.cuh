// attn_common.cuh -- pieces shared by the attention kernels (one new token
// per request: decode_attn.cu; several: decode_attn_tokens.cu) and the split
// combine (combine.cu): tile geometry in shared memory, the split of the
// flattened tile sequence into units, and the page lookahead.
#pragma once

#include "pkv_internal.h"
#include "pkv_device.cuh"

namespace pkv {
namespace attn {

using namespace dev;

constexpr uint64_t kWaitLimitNs = 500ull * 1000ull * 1000ull;  // 0.5 s per wait
constexpr unsigned kFull = 0xFFFFFFFFu;

// Tile geometry: TT tokens per tile (16, or 32 for E4M3 pools with pages of
// at least 32 tokens), one TMA box of TT rows per 128 (or 64) bytes of row.
template <int D, bool FP8, int TT = kTile>
struct Geo {
    static constexpr int ELEM = FP8 ? 1 : 2;
    static constexpr int ROWB = D * ELEM;                  // bytes per token row
    static constexpr int BOXB = ROWB > 128 ? 128 : ROWB;   // bytes per TMA box row
    static constexpr int NBOX = ROWB / BOXB;               // boxes per tile per tensor
    static constexpr int CPB = BOXB / 16;                  // 16-byte chunks per box row
    static constexpr int BOX_BYTES = TT * BOXB;
    static constexpr int TILEB = TT * ROWB;                // one K (or V) tile
    static constexpr int STAGEB = 2 * TILEB;               // K + V
};

// Byte offset inside a tile of 16-byte chunk `ch` (counted along the token
// row) of tile row `row`, as the TMA swizzle placed it.
template <int D, bool FP8, int TT = kTile>
__device__ __forceinline__ uint32_t tile_off(int row, int ch)
{
    using Gm = Geo<D, FP8, TT>;
    const int box = ch / Gm::CPB, cib = ch % Gm::CPB;
    const int x = (Gm::BOXB == 128) ? (row & 7) : ((row >> 1) & 3);
    return (uint32_t)(box * Gm::BOX_BYTES + row * Gm::BOXB + ((cib ^ x) << 4));
}

struct StageInfo {
    float ks, vs;   // fp8 scales of the tile's page and kv head
    int valid;      // 0: page id was out of range, tile skipped
    int pad;
};

// Units of the split.  Warp range v is [r(v), r(v+1)), r(v) = v T / W.  With
// K = 0 a range is one unit.  With K > 0 unit v (K+1) is the head
// [r(v), s(v)) and units v (K+1) + 1 + j, j < K, cut the tail [s(v), r(v+1))
// of tl = min(range / kTailDen, kTailMaxTiles) tiles at s(v) + j tl / K.
// Units are numbered in the order of the tiles they hold, none is empty, and
// together they cover [0, T) once.  W < 2^16, so r(v) needs one 32-bit
// division (T = qT W + rT), and tl is small.
struct Split {
    long long T, qT;
    int W, K, rT;

    __device__ __forceinline__ long long r(int v) const
    {
        return (long long)v * qT + (long long)(((unsigned)v * (unsigned)rT) / (unsigned)W);
    }
    __device__ __forceinline__ static int tail_of(long long range)
    {
        return (int)min(range / kTailDen, (long long)kTailMaxTiles);
    }
    // first tile of unit U (U = W (K+1) gives T)
    __device__ __forceinline__ long long ustart(int U) const
    {
        if (K == 0) return r(U);
        const int v = U / (K + 1), j = U - v * (K + 1);
        const long long rv = r(v);
        if (j == 0) return rv;
        const long long range = r(v + 1) - rv;
        const int tl = tail_of(range);
        return rv + range - tl + (j - 1) * tl / K;
    }
    // index of the unit holding tile x, 0 <= x < T
    __device__ __forceinline__ int unit_of(long long x) const
    {
        const int v = (int)(((x + 1) * W - 1) / T);
        if (K == 0) return v;
        const long long rv = r(v), range = r(v + 1) - rv;
        const int tl = tail_of(range);
        const long long sv = rv + range - tl;
        if (x < sv) return v * (K + 1);
        const int y = (int)(x - sv);
        return v * (K + 1) + 1 + ((y + 1) * K - 1) / tl;
    }
};

// K for T tiles over W warps, at most `max_chunks`: chunks of at least
// kTailChunkTiles tiles, none when the shortest range is under kTailMinTiles
// tiles (its tail then holds at least 8 tiles, and the head at least 24).
__device__ __forceinline__ Split make_split(long long T, int W, int max_chunks)
{
    Split sp;
    sp.T = T;
    sp.W = W;
    sp.qT = T / W;
    sp.rT = (int)(T - sp.qT * W);
    sp.K = 0;
    if (max_chunks == kTailAuto) max_chunks = sp.qT >= kAutoTailTiles ? kAutoTailChunks : 0;
    if (max_chunks > 0 && sp.qT >= kTailMinTiles)
        sp.K = min(max_chunks, max(1, Split::tail_of(sp.qT) / kTailChunkTiles));
    return sp;
}

// Warp workers of the split of T tiles when the grid has `grid_warps`
// warps: all of them, at most `workers` when that is set, else one per
// kMinTilesPerWorker tiles; at least one and at most T.  The attention and
// the combine that derives the split itself both use this.
__device__ __forceinline__ int split_workers(long long T, long long grid_warps, int workers)
{
    long long Wl = grid_warps;
    if (workers > 0) Wl = min(Wl, (long long)workers);
    else Wl = min(Wl, (T + kMinTilesPerWorker - 1) / kMinTilesPerWorker);
    return (int)max(1LL, min(Wl, max(T, 1LL)));
}

// One warp: request b's tile count, the tiles of the requests before it and
// of all requests, from seq_lens with the attention's rule (ceil((L + 1) /
// tile) tiles, none for a length out of range).  seq_lens is read-only in a
// step, so this may run before the wait for the attention grid.
__device__ __forceinline__ void warp_request_span(const AttnParams& p, int b, int lane, int& before, int& mine,
                                                  int& all)
{
    const long long cap = (long long)p.bt_stride * p.P;
    int bf = 0, mn = 0, al = 0;
    for (int c = lane; c < p.batch; c += 32) {
        const int L = __ldg(&p.seq_lens[c]);
        const int n = (L >= 0 && (long long)L < cap) ? (L + p.tile) / p.tile : 0;
        al += n;
        if (c < b) bf += n;
        if (c == b) mn = n;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        bf += __shfl_xor_sync(kFull, bf, o);
        mn += __shfl_xor_sync(kFull, mn, o);
        al += __shfl_xor_sync(kFull, al, o);
    }
    before = bf;
    mine = mn;
    all = al;
}

// Largest b with prefix[b] * Hkv <= x, for 0 <= x < prefix[B] * Hkv.
__device__ __forceinline__ int seek_request(const int* prefix, int B, int Hkv, long long x)
{
    int lo = 0, hi = B;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if ((long long)prefix[mid] * Hkv <= x) lo = mid;
        else hi = mid;
    }
    return lo;
}

// (request, kv head, tile within the pair) of flattened tile x
__device__ __forceinline__ void locate(const int* prefix, int B, int Hkv, long long x, int& b, int& kvh,
                                       int& tt, int& cnt)
{
    b = seek_request(prefix, B, Hkv, x);
    cnt = prefix[b + 1] - prefix[b];
    const long long r = x - (long long)prefix[b] * Hkv;
    if (r <= 0x7fffffffll) {   // the usual case: 32-bit division
        kvh = (int)r / cnt;
        tt = (int)r - kvh * cnt;
    } else {
        kvh = (int)(r / cnt);
        tt = (int)(r % cnt);
    }
}

// Page ids (as TMA row coordinates) and scales of 32 consecutive tiles of
// TT tokens (TT <= P, so a tile never crosses a page), one per lane.
struct Lookahead {
    int valid;   // 0: past the range, 1: ok, 2: page id out of range
    int row;
    float ks, vs;
};

template <bool FP8, int TT = kTile>
__device__ __forceinline__ Lookahead lookahead_fill(const AttnParams& p, const int* prefix, long long x0,
                                                    long long t_end, int lane)
{
    Lookahead la{0, 0, 1.f, 1.f};
    const long long y = x0 + lane;
    if (y < t_end) {
        const int b = seek_request(prefix, p.batch, p.Hkv, y);
        const int ntb = prefix[b + 1] - prefix[b];
        const long long r = y - (long long)prefix[b] * p.Hkv;
        const int kvh = (int)(r / ntb), tt = (int)(r % ntb);
        const int tok0 = tt * TT;
        const int lp = tok0 / p.P;
        const int brow = p.vmap ? __ldg(&p.vmap[b].x) : b;   // a virtual request reads its request's row
        const int page = __ldg(&p.block_tables[(size_t)brow * p.bt_stride + lp]);
        if ((unsigned)page < (unsigned)p.num_pages) {
            la.valid = 1;
            la.row = (page * p.Hkv + kvh) * p.P + (tok0 - lp * p.P);
            if (FP8) {
                la.ks = __ldg(&p.k_scale[(size_t)page * p.Hkv + kvh]);
                la.vs = __ldg(&p.v_scale[(size_t)page * p.Hkv + kvh]);
            }
        } else {
            la.valid = 2;
        }
    }
    return la;
}

// Launches an attention kernel (K / V tensor maps, parameters); with `pdl`
// as a programmatic dependent of the kernel before it on the stream, which
// lets its prologue (split, page lookahead) run while that kernel finishes.
// The kernel waits for it (grid_dependency_wait) before it reads q or issues
// a tile load.
template <typename... Args>
cudaError_t launch_attn_kernel(void (*kern)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                               bool pdl, const CUtensorMap& tmk, const CUtensorMap& tmv, const AttnParams& p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, tmk, tmv, p);
}

}  // namespace attn
}  // namespace pkv
