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
#include "rope_common.cuh"

namespace pkv {
namespace {

constexpr int kRopeThreads = 128;

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

    // loads that do not depend on the position go out first
    rope::Item item{};
    if (active) item = rope::load_item<D>(p.q, p.k_new, p.v_new, p.Hq, p.Hkv, bt, r, i0);

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
        dev::rope_sincos((double)L * theta, &s, &c);
        s_cos[i] = c;
        s_sin[i] = s;
    }
    __syncthreads();
    if (!active) return;
    rope::store_item<D, FP8>(item, p.q, p.k_pool, p.v_pool, p.k_scale, p.v_scale, p.Hq, p.Hkv, p.P, bt, r, i0,
                             page, L % p.P, s_cos, s_sin);
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
