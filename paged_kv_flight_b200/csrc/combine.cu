// combine.cu -- the split combine that follows both attention kernels: the
// partial results of a (request, kv head) pair cut between units of the
// split are merged by log-sum-exp into the bf16 output.  Split-KV decoding
// is not described on the pages; the merge is the standard rescaling of
// partial softmax sums (log-sum-exp), exact up to rounding.
#include "attn_common.cuh"

namespace pkv {
namespace {

using namespace dev;
using namespace attn;

// Split combine: one CTA per (request, kv head) pair.  A pair whose tiles lay
// in more than one unit left one partial per unit (unnormalised o, running max
// m in log2 units, sum l, for each of its R = G x q_len rows: head h of new
// token t at row t G + h); here they are merged by log-sum-exp,
//   m* = max m_v,  l* = sum l_v 2^(m_v - m*),  o = sum o_v 2^(m_v - m*) / l*,
// and written as bf16.  Pairs finished inside one unit, and requests with an
// impossible length, are skipped.  Runs after the attention kernel on the
// same stream, which orders every partial before it is read; it also resets
// the chunk counter of the attention's dynamic tail for the next launch.
// Contributors are staged in shared memory kCombineBlock at a time: one pass
// for m* and l* (one warp per head), one for the weighted sum (in reverse
// block order, so a pair with at most kCombineBlock contributors is staged
// once) in which warp j sums contributors j, j + 8, ... over all G x D
// values with 16-byte loads, and the eight warp sums are added in a fixed
// order.
constexpr int kCombineThreads = 256;
constexpr int kCombineWarps = kCombineThreads / 32;
constexpr int kCombineBlock = 256;

// floats of the staging area (slots, m, l of kb contributors, R rows each),
// rounded up to 16 bytes
inline __host__ __device__ size_t combine_stage_floats(int kb, int R)
{
    return (((size_t)kb * (2 * R + 1)) + 3) & ~(size_t)3;
}

// Dynamic shared memory of the combine for at most `contributors` per pair
// and R partial rows.
inline size_t combine_smem_bytes(int contributors, int R, int D)
{
    const int kb = contributors < kCombineBlock ? contributors : kCombineBlock;
    return sizeof(float) * (combine_stage_floats(kb, R) + (size_t)kCombineWarps * R * D);
}

template <int D, int MAXR>
__global__ void __launch_bounds__(kCombineThreads, 2) combine_kernel(const AttnParams p)
{
    constexpr unsigned kFullMask = 0xFFFFFFFFu;
    constexpr int F4 = MAXR * D / 4 / 32;          // 16-byte chunks per lane per contributor, at most
    constexpr int RPW = (MAXR + kCombineWarps - 1) / kCombineWarps;   // rows reduced per warp in pass 1
    extern __shared__ float4 s_dyn4[];
    float* const s_dyn = reinterpret_cast<float*>(s_dyn4);
    __shared__ float s_m[MAXR], s_l[MAXR];

    const int pair = blockIdx.x;
    const int b = pair / p.Hkv, kvh = pair - b * p.Hkv;
    int pb, nt, W, K;
    long long T;
    if (p.own_split) {
        // one new token per request: the attention's split from seq_lens
        // (every warp alike), then wait for that grid
        int all;
        warp_request_span(p, b, threadIdx.x & 31, pb, nt, all);
        T = (long long)all * p.Hkv;
        W = split_workers(T, p.grid_warps, p.workers);
        K = make_split(max(T, 1LL), W, p.tail_chunks).K;
        grid_dependency_wait();
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.claim = 0;   // the attention launch has ended
    if (!p.own_split) {
        W = __ldg(&p.meta[0]);
        T = (long long)(unsigned)__ldg(&p.meta[1]) | ((long long)__ldg(&p.meta[2]) << 32);
        K = __ldg(&p.meta[3]);
        const int B = p.vmap ? min(__ldg(p.vcount), p.batch) : p.batch;   // requests, or virtual requests
        if (T == 0 || b >= B) return;
        pb = __ldg(&p.meta[4 + b]);
        nt = __ldg(&p.meta[4 + b + 1]) - pb;
    }
    if (T == 0 || nt == 0) return;
    Split sp = make_split(T, W, 0);
    sp.K = K;   // as the attention launch chose it
    const long long ts = (long long)pb * p.Hkv + (long long)kvh * nt;
    const int U0 = sp.unit_of(ts), U1 = sp.unit_of(ts + nt - 1);
    if (U0 == U1) return;
    const int G = p.G, R = G * p.q_len;            // partial rows: new token t, head h at row t G + h
    // rows that hold partials: a virtual request of e.z < q_len tokens
    // leaves only its G e.z rows (the rest of its slot is stale)
    const int Rv = p.vmap ? G * min(max(__ldg(&p.vmap[b].z), 0), p.q_len) : R;
    const int k = U1 - U0 + 1, RD4 = Rv * D / 4;
    const int side0 = sp.ustart(U0) < ts ? 1 : 0;   // slot side of the first unit
    const int kb = min(k, kCombineBlock);              // the dynamic shared memory holds kb contributors
    const int nblk = (k + kCombineBlock - 1) / kCombineBlock;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    float* const s_mv = s_dyn;                                                  // [kb * R] m, later the weight
    float* const s_lv = s_dyn + (size_t)kb * R;                                 // [kb * R] l
    int* const s_slot = reinterpret_cast<int*>(s_dyn + 2 * (size_t)kb * R);    // [kb]
    float4* const s_red = s_dyn4 + combine_stage_floats(kb, R) / 4;            // [warps][R * D / 4]

    // slots, m and l of the contributors of block blk; returns how many
    auto stage = [&](int blk) -> int {
        const int i0 = blk * kCombineBlock, n = min(kCombineBlock, k - i0);
        for (int i = tid; i < n; i += kCombineThreads)
            s_slot[i] = 2 * (U0 + i0 + i) + (i0 + i == 0 ? side0 : 0);
        __syncthreads();
        for (int e = tid; e < n * Rv; e += kCombineThreads) {
            const int i = e / Rv, rr = e - i * Rv;
            const float2 ml = __ldg(reinterpret_cast<const float2*>(p.part_ml + ((size_t)s_slot[i] * R + rr) * 2));
            s_mv[i * R + rr] = ml.x;
            s_lv[i * R + rr] = ml.y;
        }
        __syncthreads();
        return n;
    };

    // pass 1: m* and l* per row (warp w reduces rows w, w + 8, ...), merged over blocks
    float Mg[RPW], Lg[RPW];
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
        Mg[j] = -INFINITY;
        Lg[j] = 0.f;
    }
    int n_last = 0;
    for (int blk = 0; blk < nblk; ++blk) {
        if (blk > 0) __syncthreads();
        const int n = stage(blk);
        n_last = n;
#pragma unroll
        for (int j = 0; j < RPW; ++j) {
            const int row = warp + kCombineWarps * j;
            if (row < Rv) {
                float m = -INFINITY;
                for (int i = lane; i < n; i += 32) m = fmaxf(m, s_mv[i * R + row]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(kFullMask, m, o));
                const float m_new = fmaxf(Mg[j], m);
                const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
                float l = 0.f;
                for (int i = lane; i < n; i += 32) l += s_lv[i * R + row] * ex2(s_mv[i * R + row] - m_ref);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) l += __shfl_xor_sync(kFullMask, l, o);
                Lg[j] = Lg[j] * ex2(Mg[j] - m_ref) + l;
                Mg[j] = m_new;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
        const int row = warp + kCombineWarps * j;
        if (row < Rv && lane == 0) {
            s_m[row] = (Mg[j] == -INFINITY) ? 0.f : Mg[j];
            s_l[row] = Lg[j];
        }
    }
    __syncthreads();

    // pass 2: warp j sums contributors j, j + 8, ... (all R x D values)
    float4 acc[F4];
#pragma unroll
    for (int t = 0; t < F4; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int blk = nblk - 1; blk >= 0; --blk) {
        int n = n_last;
        if (blk != nblk - 1) {
            __syncthreads();
            n = stage(blk);
        }
        for (int e = tid; e < n * Rv; e += kCombineThreads) {
            const int i = e / Rv, rr = e - i * Rv;
            s_mv[i * R + rr] = ex2(s_mv[i * R + rr] - s_m[rr]) / s_l[rr];   // now the weight
        }
        __syncthreads();
#pragma unroll 2
        for (int i = warp; i < n; i += kCombineWarps) {
            const float4* src = reinterpret_cast<const float4*>(p.part_o + (size_t)s_slot[i] * R * D);
#pragma unroll
            for (int t = 0; t < F4; ++t) {
                const int f = lane + 32 * t;
                if (f < RD4) {
                    const float wgt = s_mv[i * R + (4 * f) / D];
                    const float4 v = __ldg(src + f);
                    acc[t].x += wgt * v.x;
                    acc[t].y += wgt * v.y;
                    acc[t].z += wgt * v.z;
                    acc[t].w += wgt * v.w;
                }
            }
        }
    }
#pragma unroll
    for (int t = 0; t < F4; ++t) {
        const int f = lane + 32 * t;
        if (f < RD4) s_red[warp * RD4 + f] = acc[t];
    }
    __syncthreads();
    for (int f = tid; f < RD4; f += kCombineThreads) {
        float4 sum = s_red[f];
#pragma unroll
        for (int j = 1; j < kCombineWarps; ++j) {
            const float4 v = s_red[j * RD4 + f];
            sum.x += v.x;
            sum.y += v.y;
            sum.z += v.z;
            sum.w += v.w;
        }
        // row r = t G + h -> out[q0 + t][kvh G + h] (token-major output; q0 =
        // the first q row of the request, or of the virtual request, whose
        // tokens past its count are not stored)
        const int r = (4 * f) / D, col = 4 * f - r * D;
        const int t = r / G, h = r - t * G;
        int q0 = b * p.q_len;
        if (p.vmap) {
            const int4 e = p.vmap[b];
            if (t >= e.z) continue;
            q0 = e.y;
        }
        uint2* const dst = reinterpret_cast<uint2*>(
            p.out + (((size_t)q0 + t) * p.Hq + (size_t)kvh * G + h) * D + col);
        *dst = make_uint2(pack_bf16(sum.x, sum.y), pack_bf16(sum.z, sum.w));
    }
}

// The same merge with one warp per pair, for batches with many pairs: all
// pairs then fit in about one wave and no shared memory or CTA barrier is
// needed.  One pass over the contributors with a running log-sum-exp per
// head (the online form of the merge: o* = sum_i 2^(m_i - m*) o_i / l*): lane
// piece t is float4 f = lane + 32 t of the G x D values, of head f / (d/4),
// and each contributor's (m, l) and values are read together.  With at most
// 4 pieces a lane (GMAX d <= 512) the next contributor's loads are in flight
// while one merges; with 8 the registers hold one contributor at a time.
constexpr int kCombineWarpThreads = 256;

template <int D, int GMAX>
__global__ void __launch_bounds__(kCombineWarpThreads, 2) combine_warp_kernel(const AttnParams p)
{
    constexpr int F4 = GMAX * D / 4 / 32;   // 16-byte pieces per lane
    constexpr bool kAhead = F4 <= 4;
    static_assert(D == 128 || D == 64, "head_dim");

    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x * (kCombineWarpThreads / 32) + (threadIdx.x >> 5);
    if (pair >= p.batch * p.Hkv) return;
    const int b = pair / p.Hkv, kvh = pair - b * p.Hkv;
    int pb, nt, W, K;
    long long T;
    if (p.own_split) {
        // the attention's split from seq_lens, then wait for that grid
        int all;
        warp_request_span(p, b, lane, pb, nt, all);
        T = (long long)all * p.Hkv;
        W = split_workers(T, p.grid_warps, p.workers);
        K = make_split(max(T, 1LL), W, p.tail_chunks).K;
        grid_dependency_wait();
    } else {
        W = __ldg(&p.meta[0]);
        T = (long long)(unsigned)__ldg(&p.meta[1]) | ((long long)__ldg(&p.meta[2]) << 32);
        K = __ldg(&p.meta[3]);
        pb = __ldg(&p.meta[4 + b]);
        nt = __ldg(&p.meta[4 + b + 1]) - pb;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) *p.claim = 0;   // the attention launch has ended
    if (T == 0 || nt == 0) return;
    Split sp = make_split(T, W, 0);
    sp.K = K;   // as the attention launch chose it
    const long long ts = (long long)pb * p.Hkv + (long long)kvh * nt;
    const int U0 = sp.unit_of(ts), U1 = sp.unit_of(ts + nt - 1);
    if (U0 == U1) return;
    const int k = U1 - U0 + 1, G = p.G, GD4 = G * D / 4;
    const int side0 = sp.ustart(U0) < ts ? 1 : 0;

    float4 acc[F4];
    float Mr[F4], Lr[F4];
#pragma unroll
    for (int t = 0; t < F4; ++t) {
        acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
        Mr[t] = -INFINITY;
        Lr[t] = 0.f;
    }
    auto load = [&](int i, float4 (&v)[F4], float2 (&ml)[F4]) {
        const int slot = 2 * (U0 + i) + (i == 0 ? side0 : 0);
        const float4* src = reinterpret_cast<const float4*>(p.part_o + (size_t)slot * G * D);
#pragma unroll
        for (int t = 0; t < F4; ++t) {
            const int f = lane + 32 * t;
            if (f < GD4) {
                ml[t] = __ldg(reinterpret_cast<const float2*>(p.part_ml + ((size_t)slot * G + f / (D / 4)) * 2));
                v[t] = __ldg(src + f);
            }
        }
    };
    auto merge = [&](const float4 (&v)[F4], const float2 (&ml)[F4]) {
#pragma unroll
        for (int t = 0; t < F4; ++t) {
            if (lane + 32 * t < GD4) {
                const float m_new = fmaxf(Mr[t], ml[t].x);
                const float ref = (m_new == -INFINITY) ? 0.f : m_new;
                const float a = ex2(Mr[t] - ref), w = ex2(ml[t].x - ref);
                acc[t].x = acc[t].x * a + w * v[t].x;
                acc[t].y = acc[t].y * a + w * v[t].y;
                acc[t].z = acc[t].z * a + w * v[t].z;
                acc[t].w = acc[t].w * a + w * v[t].w;
                Lr[t] = Lr[t] * a + w * ml[t].y;
                Mr[t] = m_new;
            }
        }
    };
    if constexpr (kAhead) {
        float4 va[F4], vb[F4];
        float2 ma[F4], mb[F4];
        load(0, va, ma);
        for (int i = 0; i < k; i += 2) {
            if (i + 1 < k) load(i + 1, vb, mb);
            merge(va, ma);
            if (i + 1 < k) {
                if (i + 2 < k) load(i + 2, va, ma);
                merge(vb, mb);
            }
        }
    } else {
        float4 va[F4];
        float2 ma[F4];
        for (int i = 0; i < k; ++i) {
            load(i, va, ma);
            merge(va, ma);
        }
    }
    uint2* const dst = reinterpret_cast<uint2*>(p.out + ((size_t)b * p.Hq + (size_t)kvh * G) * D);
#pragma unroll
    for (int t = 0; t < F4; ++t) {
        const int f = lane + 32 * t;
        if (f < GD4) {
            const float inv = 1.f / Lr[t];
            dst[f] = make_uint2(pack_bf16(acc[t].x * inv, acc[t].y * inv), pack_bf16(acc[t].z * inv, acc[t].w * inv));
        }
    }
}

template <int D>
cudaError_t prepare_d()
{
    cudaError_t e = cudaFuncSetAttribute(combine_kernel<D, 8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)combine_smem_bytes(kCombineBlock, 8, D));
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(combine_kernel<D, 16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)combine_smem_bytes(kCombineBlock, 16, D));
}

template <typename Kern>
cudaError_t launch_one(Kern kern, int grid, int threads, size_t smem, cudaStream_t stream, bool pdl,
                       const AttnParams& p)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kern, p);
}

template <int D>
cudaError_t launch_d(const AttnParams& p, int max_units_n, int ctas, cudaStream_t stream, bool pdl)
{
    const int pairs = p.batch * p.Hkv, R = p.G * p.q_len;
    // a warp per pair when there are at least two pairs per attention CTA
    // (many pairs, each with few contributors) and at most 8 rows; else a
    // CTA per pair
    if (p.q_len == 1 && pairs >= 2 * ctas) {
        const int wpc = kCombineWarpThreads / 32, grid = (pairs + wpc - 1) / wpc;
        if (p.G <= 4) return launch_one(combine_warp_kernel<D, 4>, grid, kCombineWarpThreads, 0, stream, pdl, p);
        return launch_one(combine_warp_kernel<D, 8>, grid, kCombineWarpThreads, 0, stream, pdl, p);
    }
    const size_t smem = combine_smem_bytes(max_units_n, R, D);
    if (R <= 8) return launch_one(combine_kernel<D, 8>, pairs, kCombineThreads, smem, stream, pdl, p);
    return launch_one(combine_kernel<D, 16>, pairs, kCombineThreads, smem, stream, pdl, p);
}

}  // namespace

cudaError_t combine_prepare(int head_dim)
{
    return head_dim == 128 ? prepare_d<128>() : prepare_d<64>();
}

cudaError_t launch_combine(const AttnParams& p, int head_dim, int max_units_n, int ctas, cudaStream_t stream,
                           bool dependent)
{
    AttnParams q = p;
    q.own_split = dependent ? 1 : 0;
    return head_dim == 128 ? launch_d<128>(q, max_units_n, ctas, stream, dependent)
                           : launch_d<64>(q, max_units_n, ctas, stream, dependent);
}

}  // namespace pkv
