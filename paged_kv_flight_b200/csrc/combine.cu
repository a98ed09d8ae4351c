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

    if (blockIdx.x == 0 && threadIdx.x == 0) *p.claim = 0;   // the attention launch has ended
    const int pair = blockIdx.x;
    const int b = pair / p.Hkv, kvh = pair - b * p.Hkv;
    const int W = __ldg(&p.meta[0]);
    const long long T = (long long)(unsigned)__ldg(&p.meta[1]) | ((long long)__ldg(&p.meta[2]) << 32);
    const int B = p.vmap ? min(__ldg(p.vcount), p.batch) : p.batch;   // requests, or virtual requests
    if (T == 0 || b >= B) return;
    const int* prefix = p.meta + 4;
    const int nt = __ldg(&prefix[b + 1]) - __ldg(&prefix[b]);
    if (nt == 0) return;
    Split sp = make_split(T, W, 0);
    sp.K = __ldg(&p.meta[3]);   // as the attention launch chose it
    const long long ts = (long long)__ldg(&prefix[b]) * p.Hkv + (long long)kvh * nt;
    const int U0 = sp.unit_of(ts), U1 = sp.unit_of(ts + nt - 1);
    if (U0 == U1) return;
    const int G = p.G, R = G * p.q_len;            // partial rows: new token t, head h at row t G + h
    const int k = U1 - U0 + 1, RD4 = R * D / 4;
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
        for (int e = tid; e < n * R; e += kCombineThreads) {
            const int i = e / R, rr = e - i * R;
            const float2 ml = __ldg(reinterpret_cast<const float2*>(p.part_ml + ((size_t)s_slot[i] * R + rr) * 2));
            s_mv[e] = ml.x;
            s_lv[e] = ml.y;
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
            if (row < R) {
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
        if (row < R && lane == 0) {
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
        for (int e = tid; e < n * R; e += kCombineThreads) {
            const int rr = e % R;
            s_mv[e] = ex2(s_mv[e] - s_m[rr]) / s_l[rr];   // now the weight
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
// needed.  Lanes take contributors 32 at a time for m* and l* (online, then a
// butterfly over the lanes) and for the weights; the weighted sum walks the
// contributors with every lane on its own 16-byte pieces of the G x D
// values, a piece of D = 128 belonging to head t for the t-th piece of the
// lane and a piece of D = 64 to head 2t or 2t + 1 by lane half.
constexpr int kCombineWarpThreads = 256;

template <int D>
__global__ void __launch_bounds__(kCombineWarpThreads, 2) combine_warp_kernel(const AttnParams p)
{
    constexpr unsigned kFullMask = 0xFFFFFFFFu;
    constexpr int F4 = kMaxGroup * D / 4 / 32;   // 16-byte pieces per lane, at most
    static_assert(D == 128 || D == 64, "head_dim");

    if (blockIdx.x == 0 && threadIdx.x == 0) *p.claim = 0;   // the attention launch has ended
    const int lane = threadIdx.x & 31;
    const int pair = blockIdx.x * (kCombineWarpThreads / 32) + (threadIdx.x >> 5);
    if (pair >= p.batch * p.Hkv) return;
    const int b = pair / p.Hkv, kvh = pair - b * p.Hkv;
    const int W = __ldg(&p.meta[0]);
    const long long T = (long long)(unsigned)__ldg(&p.meta[1]) | ((long long)__ldg(&p.meta[2]) << 32);
    const int* prefix = p.meta + 4;
    const int pb = __ldg(&prefix[b]);
    const int nt = __ldg(&prefix[b + 1]) - pb;
    if (T == 0 || nt == 0) return;
    Split sp = make_split(T, W, 0);
    sp.K = __ldg(&p.meta[3]);   // as the attention launch chose it
    const long long ts = (long long)pb * p.Hkv + (long long)kvh * nt;
    const int U0 = sp.unit_of(ts), U1 = sp.unit_of(ts + nt - 1);
    if (U0 == U1) return;
    const int k = U1 - U0 + 1, G = p.G, GD4 = G * D / 4;
    const int side0 = sp.ustart(U0) < ts ? 1 : 0;

    // pass 1: m* and l* per head; lane j keeps the m of its first contributor
    // (j) so that the weights of the first 32 need no second load
    float M[kMaxGroup], L[kMaxGroup], m_own[kMaxGroup];
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        M[g] = -INFINITY;
        L[g] = 0.f;
        m_own[g] = -INFINITY;
    }
    for (int i = lane; i < k; i += 32) {
        const int slot = 2 * (U0 + i) + (i == 0 ? side0 : 0);
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) {
            if (g < G) {
                const float2 ml = __ldg(reinterpret_cast<const float2*>(p.part_ml + ((size_t)slot * G + g) * 2));
                if (i == lane) m_own[g] = ml.x;
                const float m_new = fmaxf(M[g], ml.x);
                const float ref = (m_new == -INFINITY) ? 0.f : m_new;
                L[g] = L[g] * ex2(M[g] - ref) + ml.y * ex2(ml.x - ref);
                M[g] = m_new;
            }
        }
    }
#pragma unroll
    for (int g = 0; g < kMaxGroup; ++g) {
        if (g < G) {
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) {
                const float m2 = __shfl_xor_sync(kFullMask, M[g], o), l2 = __shfl_xor_sync(kFullMask, L[g], o);
                const float m_new = fmaxf(M[g], m2);
                const float ref = (m_new == -INFINITY) ? 0.f : m_new;
                L[g] = L[g] * ex2(M[g] - ref) + l2 * ex2(m2 - ref);
                M[g] = m_new;
            }
            if (M[g] == -INFINITY) M[g] = 0.f;
        }
    }

    // pass 2: weighted sum, contributors in batches of 32 (lane j holds the
    // slot and the weights of contributor i0 + j)
    float4 acc[F4];
#pragma unroll
    for (int t = 0; t < F4; ++t) acc[t] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < k; i0 += 32) {
        const int i = i0 + lane;
        int slot_l = 0;
        float wl[kMaxGroup];
#pragma unroll
        for (int g = 0; g < kMaxGroup; ++g) wl[g] = 0.f;
        if (i < k) {
            slot_l = 2 * (U0 + i) + (i == 0 ? side0 : 0);
#pragma unroll
            for (int g = 0; g < kMaxGroup; ++g) {
                if (g < G) {
                    const float m = (i0 == 0) ? m_own[g] : __ldg(p.part_ml + ((size_t)slot_l * G + g) * 2);
                    wl[g] = ex2(m - M[g]) / L[g];
                }
            }
        }
        const int n = min(32, k - i0);
        for (int j = 0; j < n; ++j) {
            const int slot = __shfl_sync(kFullMask, slot_l, j);
            const float4* src = reinterpret_cast<const float4*>(p.part_o + (size_t)slot * G * D);
#pragma unroll
            for (int t = 0; t < F4; ++t) {
                float w;
                if constexpr (D == 128) {
                    w = __shfl_sync(kFullMask, wl[t], j);
                } else {
                    const float wa = __shfl_sync(kFullMask, wl[2 * t], j);
                    const float wb = __shfl_sync(kFullMask, wl[2 * t + 1], j);
                    w = lane < 16 ? wa : wb;
                }
                const int f = lane + 32 * t;
                if (f < GD4) {
                    const float4 v = __ldg(src + f);
                    acc[t].x += w * v.x;
                    acc[t].y += w * v.y;
                    acc[t].z += w * v.z;
                    acc[t].w += w * v.w;
                }
            }
        }
    }
    uint2* const dst = reinterpret_cast<uint2*>(p.out + ((size_t)b * p.Hq + (size_t)kvh * G) * D);
#pragma unroll
    for (int t = 0; t < F4; ++t) {
        const int f = lane + 32 * t;
        if (f < GD4) dst[f] = make_uint2(pack_bf16(acc[t].x, acc[t].y), pack_bf16(acc[t].z, acc[t].w));
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

template <int D>
cudaError_t launch_d(const AttnParams& p, int max_units_n, int ctas, cudaStream_t stream)
{
    const int pairs = p.batch * p.Hkv, R = p.G * p.q_len;
    // a warp per pair when there are at least two pairs per attention CTA
    // (many pairs, each with few contributors) and at most 8 rows; else a
    // CTA per pair
    if (p.q_len == 1 && pairs >= 2 * ctas) {
        const int wpc = kCombineWarpThreads / 32;
        combine_warp_kernel<D><<<(pairs + wpc - 1) / wpc, kCombineWarpThreads, 0, stream>>>(p);
    } else {
        const size_t smem = combine_smem_bytes(max_units_n, R, D);
        if (R <= 8) combine_kernel<D, 8><<<pairs, kCombineThreads, smem, stream>>>(p);
        else combine_kernel<D, 16><<<pairs, kCombineThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t combine_prepare(int head_dim)
{
    return head_dim == 128 ? prepare_d<128>() : prepare_d<64>();
}

cudaError_t launch_combine(const AttnParams& p, int head_dim, int max_units_n, int ctas, cudaStream_t stream)
{
    return head_dim == 128 ? launch_d<128>(p, max_units_n, ctas, stream) : launch_d<64>(p, max_units_n, ctas, stream);
}

}  // namespace pkv
