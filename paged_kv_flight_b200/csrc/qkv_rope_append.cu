// qkv_rope_append.cu -- the QKV projection of the step's new tokens on the
// Blackwell tensor cores (tcgen05, accumulators in tensor memory), fused with
// RoPE and the append into the paged pools: the projection's output never
// goes to memory as a whole ("Scaling TensorRT-LLM: Kernel Fusion and
// Inflight Batching in Production", section "What Gets Fused": attention-side
// projections with RoPE folded in; "TensorRT-LLM Guide: High-Throughput GPU
// Inference Engine", section "2. Paged KV Cache & Memory Virtualization").
//
// What it computes, per token t (request t, one new token each) and output
// feature n of the weight W [(Hq + 2 Hkv) d][hidden] (q heads, then k heads,
// then v heads; row h d + i is dimension i of head h):
//   y[t][n] = bf16_RNE(sum_j x[t][j] W[n][j]),
// then exactly what rope_append stores for q, k_new = y's k part and
// v_new = y's v part: q rotated at position L_t in place of the q output,
// rotated k and raw v into slot L_t % P of page block_tables[t][L_t / P].
//
// Tiling: one CTA per (32-feature slice, 128-token tile).  A slice holds the
// 16 rotation pairs i = 16 j .. 16 j + 15 of one head together with their
// partners i + d/2, so the epilogue thread of a token has both halves of
// every pair it rotates.  The MMA is D[128 tokens][32 features] += X W^T
// (A = x rows, K-major; B = the slice's 32 weight rows, K-major; bf16 in,
// fp32 in tensor memory), M = 128, N = 32, K = 16 per instruction, 64 hidden
// elements (one 128-byte swizzle row) per pipeline stage.  Warp 0's lane
// issues the TMA loads into a ring of stages, warp 1's lane issues
// tcgen05.mma and commits each stage back to the producer; all four warps then
// read their 32 token rows out of tensor memory (tcgen05.ld) and run the
// epilogue.  The weights are read once; the kernel is bound by that stream
// at decode batch sizes (arithmetic intensity = tokens flop per weight byte).
// Every mbarrier wait is bounded; a timeout sets an error bit and the CTA
// still frees its tensor memory.
#include "pkv_internal.h"
#include "pkv_device.cuh"

namespace pkv {
namespace {

using namespace dev;

constexpr int kQkvThreads = 128;
constexpr int kQkvM = 128;                 // tokens per tile (TMEM lanes, rows of A)
constexpr int kQkvN = 32;                  // features per CTA: 16 pairs x 2 halves
constexpr int kQkvBK = 64;                 // hidden elements per stage: one 128-byte row
constexpr int kQkvStages = 5;                // 5 x 20 KB: two CTAs per SM
constexpr int kQkvAB = kQkvM * kQkvBK * 2; // 16 KB
constexpr int kQkvBB = kQkvN * kQkvBK * 2; // 4 KB
constexpr int kQkvStageB = kQkvAB + kQkvBB;
constexpr uint32_t kQkvTmemCols = 32;      // fp32 accumulator columns (= N)
constexpr uint64_t kQkvWaitNs = 500ull * 1000ull * 1000ull;

constexpr double kTwoPiHi = 6.283185307179586;
constexpr double kTwoPiLo = 2.4492935982947064e-16;
constexpr double kInvTwoPi = 0.15915494309189535;

// Shared-memory matrix descriptor of a K-major tile with 128-byte rows and
// the 128-byte swizzle (the layout the TMA loads write): start address >> 4,
// leading byte offset 1 (unused by this layout), stride byte offset 1024 B
// (8 rows), descriptor version 1, layout type 2 (128-byte swizzle).  The tile
// base is 1024-byte aligned; a K step of 16 elements adds 32 bytes to the
// start address.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t saddr)
{
    uint64_t d = (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1u << 16;
    d |= (uint64_t)(1024u >> 4) << 32;
    d |= (uint64_t)1u << 46;
    d |= (uint64_t)2u << 61;
    return d;
}

// Instruction descriptor of kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kQkvIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kQkvN >> 3) << 17) |
                               ((uint32_t)(kQkvM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t"
        ".reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t"
        "}\n" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(kQkvIdesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}

__device__ __forceinline__ void umma_commit(uint32_t bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void sincos_reduced(double phi, double* s, double* c)
{
    const double k = rint(phi * kInvTwoPi);
    double r = fma(-k, kTwoPiHi, phi);
    r = fma(-k, kTwoPiLo, r);
    sincos(r, s, c);
}

template <int D>
__global__ void __launch_bounds__(kQkvThreads, 2)
qkv_rope_append_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                       const QkvParams p)
{
    constexpr int HALF = D / 2;
    constexpr int SLICES = D / 32;          // 32-feature slices per head
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kQkvStages], s_empty[kQkvStages], s_done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int slice = blockIdx.x, m0 = blockIdx.y * kQkvM;
    const int head = slice / SLICES, j = slice - head * SLICES;   // head over q, then k, then v
    const int row_lo = head * D + 16 * j, row_hi = row_lo + HALF;
    const int KB = p.hidden / kQkvBK;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t stage0 = (raw + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&s_full[0]), empty0 = smem_u32(&s_empty[0]), done = smem_u32(&s_done);

    if (tid == 0) {
        s_fail = 0;
        for (int s = 0; s < kQkvStages; ++s) {
            mbar_init(full0 + 8u * s, 1u);
            mbar_init(empty0 + 8u * s, 1u);
        }
        mbar_init(done, 1u);
        fence_mbar_init();
        prefetch_tensormap(&tmx);
        prefetch_tensormap(&tmw);
    }
    if (warp == 0) {
        __syncwarp();   // converged for the aligned allocation
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&s_tmem)),
                     "r"(kQkvTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ---- producer: TMA loads of x rows m0.. and the slice's 2 x 16 weight rows
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kQkvStages;
                if (kb >= kQkvStages &&
                    !mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((kb / kQkvStages - 1) & 1), kQkvWaitNs)) {
                    atomicOr(p.err, kErrTimeout);
                    s_fail = 1;
                    break;
                }
                const uint32_t a = stage0 + (uint32_t)(s * kQkvStageB), b = a + kQkvAB;
                // x_rows (<= 128) token rows; the MMA reads all 128 rows of the
                // stage's A area, rows past x_rows only feed accumulator rows
                // of no token
                mbar_arrive_expect_tx(full0 + 8u * s, (uint32_t)(p.x_rows * kQkvBK * 2 + kQkvBB));
                tma_load_2d(a, &tmx, kb * kQkvBK, m0, full0 + 8u * s);
                tma_load_2d(b, &tmw, kb * kQkvBK, row_lo, full0 + 8u * s);
                tma_load_2d(b + kQkvBB / 2, &tmw, kb * kQkvBK, row_hi, full0 + 8u * s);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: one thread; each stage is committed back to the producer
        if (lane == 0) {
            for (int kb = 0; kb < KB; ++kb) {
                const int s = kb % kQkvStages;
                if (!mbar_wait_bounded(full0 + 8u * s, (uint32_t)((kb / kQkvStages) & 1), kQkvWaitNs)) {
                    atomicOr(p.err, kErrTimeout);
                    s_fail = 1;
                    break;
                }
                tmem_fence_after();
                const uint32_t a = stage0 + (uint32_t)(s * kQkvStageB), b = a + kQkvAB;
#pragma unroll
                for (int kk = 0; kk < kQkvBK / 16; ++kk)
                    umma_bf16(tmem, sw128_kmajor_desc(a + 32u * kk), sw128_kmajor_desc(b + 32u * kk),
                              (kb | kk) != 0 ? 1u : 0u);
                umma_commit(empty0 + 8u * s);
            }
            umma_commit(done);   // arrives once every MMA issued above has completed
        }
    }
    // the other lanes of warps 0 and 1 wait here, not in a spin beside the
    // issuing lane, which keeps its warp's issue slots
    __syncwarp();

    // ---- epilogue: every warp reads its 32 token rows out of tensor memory
    const bool ok = mbar_wait_bounded(done, 0u, kQkvWaitNs);
    if (!ok && tid == 0) atomicOr(p.err, kErrTimeout);
    tmem_fence_after();
    float acc[32];
    tmem_ld32(tmem + ((uint32_t)(32 * warp) << 16), acc);

    const int t = m0 + 32 * warp + lane;     // token = request
    __syncthreads();                         // s_fail settled
    if (ok && !s_fail && t < p.batch) {
        const int kind = head < p.Hq ? 0 : (head < p.Hq + p.Hkv ? 1 : 2);   // q, k, v
        const int hh = kind == 0 ? head : (kind == 1 ? head - p.Hq : head - p.Hq - p.Hkv);
        const int i0 = 16 * j;
        // the projection's bf16 outputs, as the unfused pipeline would store them
        double lo[16], hi[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            lo[c] = (double)__bfloat162float(__float2bfloat16_rn(acc[c]));
            hi[c] = (double)__bfloat162float(__float2bfloat16_rn(acc[16 + c]));
        }
        const int L = p.seq_lens[t];
        const bool len_ok = L >= 0 && (long long)L < (long long)p.bt_stride * p.P;
        uint32_t olo[8], ohi[8];
        if (kind < 2) {    // q and k are rotated at position L; v is stored as is
            if (!len_ok) {
                atomicOr(p.err, kErrLength);
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const int i = i0 + c;
                    const double theta = pow(p.rope_base, (-2.0 * i) / D);
                    double sn, cs;
                    sincos_reduced((double)L * theta, &sn, &cs);
                    const double ylo = __dsub_rn(__dmul_rn(lo[c], cs), __dmul_rn(hi[c], sn));
                    const double yhi = __dadd_rn(__dmul_rn(hi[c], cs), __dmul_rn(lo[c], sn));
                    lo[c] = ylo;
                    hi[c] = yhi;
                }
            }
        }
        if (kind == 0 || !p.fp8) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                olo[c] = (uint32_t)__bfloat16_as_ushort(bf16_from_f64(lo[2 * c])) |
                         ((uint32_t)__bfloat16_as_ushort(bf16_from_f64(lo[2 * c + 1])) << 16);
                ohi[c] = (uint32_t)__bfloat16_as_ushort(bf16_from_f64(hi[2 * c])) |
                         ((uint32_t)__bfloat16_as_ushort(bf16_from_f64(hi[2 * c + 1])) << 16);
            }
        }
        if (kind == 0) {
            if (len_ok) {
                uint4* dst = reinterpret_cast<uint4*>(p.q_out + ((size_t)t * p.Hq + hh) * D + i0);
                uint4* dsth = reinterpret_cast<uint4*>(p.q_out + ((size_t)t * p.Hq + hh) * D + i0 + HALF);
                dst[0] = make_uint4(olo[0], olo[1], olo[2], olo[3]);
                dst[1] = make_uint4(olo[4], olo[5], olo[6], olo[7]);
                dsth[0] = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
                dsth[1] = make_uint4(ohi[4], ohi[5], ohi[6], ohi[7]);
            }
        } else if (len_ok) {
            const int page = p.block_tables[(size_t)t * p.bt_stride + L / p.P];
            if (page < 0 || page >= p.num_pages) {
                atomicOr(p.err, kErrPage);
            } else {
                const size_t prow = ((size_t)page * p.Hkv + hh) * p.P + (L % p.P);
                void* pool = kind == 1 ? p.k_pool : p.v_pool;
                if (!p.fp8) {
                    __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(pool) + prow * D;
                    uint4* a = reinterpret_cast<uint4*>(dst + i0);
                    uint4* b = reinterpret_cast<uint4*>(dst + i0 + HALF);
                    a[0] = make_uint4(olo[0], olo[1], olo[2], olo[3]);
                    a[1] = make_uint4(olo[4], olo[5], olo[6], olo[7]);
                    b[0] = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
                    b[1] = make_uint4(ohi[4], ohi[5], ohi[6], ohi[7]);
                } else {
                    // E4M3 as the append stores it: k from the fp64 rotation over the
                    // scale, v from its bf16 value over the scale (fp32 division)
                    const size_t si = (size_t)page * p.Hkv + hh;
                    uint8_t qlo[16], qhi[16];
                    if (kind == 1) {
                        const double sk = (double)p.k_scale[si];
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            qlo[c] = e4m3_satfinite(__double2float_rn(__ddiv_rn(lo[c], sk)));
                            qhi[c] = e4m3_satfinite(__double2float_rn(__ddiv_rn(hi[c], sk)));
                        }
                    } else {
                        const float sv = p.v_scale[si];
#pragma unroll
                        for (int c = 0; c < 16; ++c) {
                            qlo[c] = e4m3_satfinite(__fdiv_rn((float)lo[c], sv));
                            qhi[c] = e4m3_satfinite(__fdiv_rn((float)hi[c], sv));
                        }
                    }
                    uint8_t* dst = reinterpret_cast<uint8_t*>(pool) + prow * D;
                    *reinterpret_cast<uint4*>(dst + i0) = *reinterpret_cast<const uint4*>(qlo);
                    *reinterpret_cast<uint4*>(dst + i0 + HALF) = *reinterpret_cast<const uint4*>(qhi);
                }
            }
        }
    }

    // ---- tensor memory back to the allocator (the warp that allocated it)
    tmem_fence_before();
    __syncthreads();
    if (warp == 0) asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kQkvTmemCols));
}

}  // namespace

size_t qkv_smem_bytes() { return 1024 + (size_t)kQkvStages * kQkvStageB; }

cudaError_t qkv_prepare()
{
    cudaError_t e = cudaFuncSetAttribute(qkv_rope_append_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)qkv_smem_bytes());
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(qkv_rope_append_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)qkv_smem_bytes());
}

cudaError_t launch_qkv_rope_append(const QkvParams& p, const CUtensorMap& tmx, const CUtensorMap& tmw,
                                   cudaStream_t stream)
{
    const int heads = p.Hq + 2 * p.Hkv;
    const dim3 grid((unsigned)(heads * (p.D / 32)), (unsigned)((p.batch + kQkvM - 1) / kQkvM)), block(kQkvThreads);
    if (p.D == 128) qkv_rope_append_kernel<128><<<grid, block, qkv_smem_bytes(), stream>>>(tmx, tmw, p);
    else qkv_rope_append_kernel<64><<<grid, block, qkv_smem_bytes(), stream>>>(tmx, tmw, p);
    return cudaGetLastError();
}

}  // namespace pkv
