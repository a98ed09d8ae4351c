// rope_append.cu -- step part 1: rotary embedding of the new token's q and
// k, and append of k / v into the paged pools.
//
// "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in Production",
// section "What Gets Fused" (RoPE applied inside the attention-side kernel
// rather than as a separate pass) and section "The Paged KV-Cache" (fixed-size
// blocks named by a per-request block table); "TensorRT-LLM Guide:
// High-Throughput GPU Inference Engine", section "2. Paged KV Cache & Memory
// Virtualization" (pages written on demand, a lookup table maps logical
// positions to physical blocks) and section "4. Native FP8 Quantization"
// (E4M3 storage).
//
// Several new tokens per request (speculative-decode verification: "Scaling
// TensorRT-LLM", section "3. Speculative Decoding for Tail Latency") are the
// same operation at positions L_b + t: the grid's first axis runs over
// (request, new token) and q / k_new / v_new carry a token axis.  With a
// count of new tokens per request (chunked prefill mixed with decodes:
// "Scaling TensorRT-LLM", section "What the Scheduler Actually Does") the
// rows are packed, cu_q[b] .. cu_q[b + 1] - 1 being request b's, and the
// grid's first axis runs over the packed rows; each finds its request by a
// binary search of cu_q.
//
// Grid (request x new token, chunk): a token's Hq + Hkv rows are cut into work items of
// 8 rotation pairs (two 16-byte loads, two 16-byte bf16 or 8-byte E4M3
// stores), 128 items per CTA.  Each thread issues its row loads first; the
// CTA meanwhile builds the cos/sin table of the request's position in fp64:
// angle p * theta_i rounded once, reduced to [-pi, pi] with a two-part 2*pi
// (Cody & Waite), then sincos.  Rotation is fp64 with separate roundings and
// one final rounding to the storage type.
#include "pkv_internal.h"
#include "pkv_device.cuh"

namespace pkv {
namespace {

constexpr int kRopeThreads = 128;

// 2*pi = kTwoPiHi + kTwoPiLo; kTwoPiHi is the double nearest 2*pi.
constexpr double kTwoPiHi = 6.283185307179586;
constexpr double kTwoPiLo = 2.4492935982947064e-16;
constexpr double kInvTwoPi = 0.15915494309189535;

__device__ __forceinline__ void sincos_reduced(double phi, double* s, double* c)
{
    const double k = rint(phi * kInvTwoPi);
    double r = fma(-k, kTwoPiHi, phi);
    r = fma(-k, kTwoPiLo, r);
    sincos(r, s, c);
}

// bf16 pools: nine CTAs per SM (at most 56 registers) keep the largest
// batches' grids to one wave (256 requests x 5 CTAs for 64 + 8 heads of
// d = 128); the E4M3 stores need more registers and are left unbounded.
template <int D, bool FP8>
__global__ void __launch_bounds__(kRopeThreads, FP8 ? 1 : 9) rope_append_kernel(const RopeParams p)
{
    constexpr int HALF = D / 2;
    constexpr int PIECES = HALF / 8;  // 8 pairs per work item
    __shared__ double s_cos[HALF], s_sin[HALF];

    // a decode attention launched as this grid's programmatic dependent may
    // start its prologue now; it reads q and the pools only once this grid
    // has finished
    dev::grid_launch_dependents();
    const int bt = blockIdx.x;               // (request, new token) row of q, k_new, v_new
    int b, t;
    if (p.cu_q) {
        // varlen: the request whose rows [cu_q[b], cu_q[b + 1]) hold row bt
        // (the last b with cu_q[b] <= bt: requests with no new token are skipped)
        int lo = 0, hi = p.batch;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.cu_q[mid] <= bt) lo = mid;
            else hi = mid;
        }
        b = lo;
        t = bt - p.cu_q[b];
    } else {
        b = bt / p.q_len;
        t = bt - b * p.q_len;
    }
    const int rows = p.Hq + p.Hkv;
    const int it = blockIdx.y * kRopeThreads + threadIdx.x;
    const bool active = it < rows * PIECES;
    const int r = it / PIECES;
    const int i0 = (it % PIECES) * 8;
    const bool is_q = r < p.Hq;
    const int kvh = r - p.Hq;

    // loads that do not depend on the position go out first
    uint4 xa = make_uint4(0, 0, 0, 0), xb = xa, va = xa, vb = xa;
    if (active) {
        const __nv_bfloat16* src = is_q ? p.q + ((size_t)bt * p.Hq + r) * D
                                        : p.k_new + ((size_t)bt * p.Hkv + kvh) * D;
        xa = *reinterpret_cast<const uint4*>(src + i0);          // x_i
        xb = *reinterpret_cast<const uint4*>(src + i0 + HALF);   // x_{i+d/2}
        if (!is_q) {
            const __nv_bfloat16* vsrc = p.v_new + ((size_t)bt * p.Hkv + kvh) * D;
            va = *reinterpret_cast<const uint4*>(vsrc + i0);
            vb = *reinterpret_cast<const uint4*>(vsrc + i0 + HALF);
        }
    }

    const int L0 = p.seq_lens[b];
    const long long Lt = (long long)L0 + t;  // position of this new token
    const bool len_ok = L0 >= 0 && Lt >= 0 && Lt < (long long)p.bt_stride * p.P;   // (t < 0: bad cu_q)
    const int L = (int)Lt;
    const int page = len_ok ? p.block_tables[(size_t)b * p.bt_stride + L / p.P] : -1;
    if (!len_ok) {
        if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(p.err, kErrLength);
        return;
    }
    if (page < 0 || page >= p.num_pages) {
        if (threadIdx.x == 0 && blockIdx.y == 0) atomicOr(p.err, kErrPage);
        return;
    }
    const int slot = L % p.P;
    if (blockIdx.y == 0 && t == 0 && p.prefetch_tables) {
        // the attention that follows walks this request's block-table row:
        // bring it into L2 now (one 128-byte line per thread)
        const int lines = (p.bt_stride * 4 + 127) / 128;
        const char* row = reinterpret_cast<const char*>(p.block_tables + (size_t)b * p.bt_stride);
        for (int i = threadIdx.x; i < lines; i += blockDim.x)
            asm volatile("prefetch.global.L2 [%0];" ::"l"(row + 128 * i));
    }

    for (int i = threadIdx.x; i < HALF; i += blockDim.x) {
        const double theta = p.theta[i];    // rope_base^(-2i/d), computed once per context
        double s, c;
        sincos_reduced((double)L * theta, &s, &c);
        s_cos[i] = c;
        s_sin[i] = s;
    }
    __syncthreads();
    if (!active) return;

    const uint32_t wa[4] = {xa.x, xa.y, xa.z, xa.w};
    const uint32_t wb[4] = {xb.x, xb.y, xb.z, xb.w};
    double ya[8], yb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const double a = (double)((k & 1) ? dev::bf16_hi(wa[k >> 1]) : dev::bf16_lo(wa[k >> 1]));
        const double bb = (double)((k & 1) ? dev::bf16_hi(wb[k >> 1]) : dev::bf16_lo(wb[k >> 1]));
        const double c = s_cos[i0 + k], s = s_sin[i0 + k];
        // separate roundings, no fused multiply-add
        ya[k] = __dsub_rn(__dmul_rn(a, c), __dmul_rn(bb, s));
        yb[k] = __dadd_rn(__dmul_rn(bb, c), __dmul_rn(a, s));
    }

    const size_t prow = ((size_t)page * p.Hkv + kvh) * p.P + slot;   // pool row (k rows only)
    if (is_q || !FP8) {
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            oa[k] = (uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(ya[2 * k])) |
                    ((uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(ya[2 * k + 1])) << 16);
            ob[k] = (uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(yb[2 * k])) |
                    ((uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(yb[2 * k + 1])) << 16);
        }
        __nv_bfloat16* dst = is_q ? p.q + ((size_t)bt * p.Hq + r) * D
                                  : reinterpret_cast<__nv_bfloat16*>(p.k_pool) + prow * D;
        *reinterpret_cast<uint4*>(dst + i0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        *reinterpret_cast<uint4*>(dst + i0 + HALF) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
    if (is_q) return;

    if (!FP8) {
        __nv_bfloat16* vdst = reinterpret_cast<__nv_bfloat16*>(p.v_pool) + prow * D;
        *reinterpret_cast<uint4*>(vdst + i0) = va;
        *reinterpret_cast<uint4*>(vdst + i0 + HALF) = vb;
    } else {
        const size_t si = (size_t)page * p.Hkv + kvh;
        const double sk = (double)p.k_scale[si];
        const float sv = p.v_scale[si];
        const uint32_t vwa[4] = {va.x, va.y, va.z, va.w};
        const uint32_t vwb[4] = {vb.x, vb.y, vb.z, vb.w};
        uint8_t ka[8], kb[8], qa8[8], qb8[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
            // k: fp64 quotient rounded once to fp32, then E4M3 RNE satfinite
            ka[k] = dev::e4m3_satfinite(__double2float_rn(__ddiv_rn(ya[k], sk)));
            kb[k] = dev::e4m3_satfinite(__double2float_rn(__ddiv_rn(yb[k], sk)));
            // v: exact bf16 value, IEEE fp32 quotient
            const float a = (k & 1) ? dev::bf16_hi(vwa[k >> 1]) : dev::bf16_lo(vwa[k >> 1]);
            const float bb = (k & 1) ? dev::bf16_hi(vwb[k >> 1]) : dev::bf16_lo(vwb[k >> 1]);
            qa8[k] = dev::e4m3_satfinite(__fdiv_rn(a, sv));
            qb8[k] = dev::e4m3_satfinite(__fdiv_rn(bb, sv));
        }
        uint8_t* kdst = reinterpret_cast<uint8_t*>(p.k_pool) + prow * D;
        uint8_t* vdst = reinterpret_cast<uint8_t*>(p.v_pool) + prow * D;
        *reinterpret_cast<uint2*>(kdst + i0) = *reinterpret_cast<const uint2*>(ka);
        *reinterpret_cast<uint2*>(kdst + i0 + HALF) = *reinterpret_cast<const uint2*>(kb);
        *reinterpret_cast<uint2*>(vdst + i0) = *reinterpret_cast<const uint2*>(qa8);
        *reinterpret_cast<uint2*>(vdst + i0 + HALF) = *reinterpret_cast<const uint2*>(qb8);
    }
}

}  // namespace

cudaError_t launch_rope_append(const RopeParams& p, cudaStream_t stream)
{
    const int items = (p.Hq + p.Hkv) * (p.D / 16);
    const int rows = p.cu_q ? p.n_tokens : p.batch * p.q_len;
    const dim3 grid(rows, (items + kRopeThreads - 1) / kRopeThreads), block(kRopeThreads);
    if (p.D == 128) {
        if (p.fp8) rope_append_kernel<128, true><<<grid, block, 0, stream>>>(p);
        else rope_append_kernel<128, false><<<grid, block, 0, stream>>>(p);
    } else {
        if (p.fp8) rope_append_kernel<64, true><<<grid, block, 0, stream>>>(p);
        else rope_append_kernel<64, false><<<grid, block, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace pkv
