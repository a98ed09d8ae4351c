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
// Tiling.  A cluster of S CTAs (S = 1 .. 4, the "split") per (head, tile of
// up to 128 tokens); CTA r of the cluster sums the hidden elements of its
// 64-element blocks [KB r / S, KB (r + 1) / S) for all d features of the
// head: D[128 tokens][d] += X W_h^T on tcgen05 (A = x rows, B = the head's d
// weight rows, both K-major with the 128-byte swizzle; bf16 in, fp32 in
// tensor memory; M = 128, N = d, K = 16 per instruction).  Warp 0's lane
// issues the TMA loads into a ring of stages (the first ones before the
// tensor memory is even allocated; up to about 200 KB of shared memory: the
// weights are the stream to keep in flight), warp 1's lane issues the MMAs
// and commits each stage back to the producer.  Meanwhile warps 2 to 5 read
// the tile's positions and destinations and fill a table of (cos, sin) in
// fp64 for the rotation pairs this CTA will finish.
//
// The reduction is a reduce-scatter through distributed shared memory: the
// pairs (i, i + d/2) are cut into groups of 8 and CTA r of the cluster owns
// groups [G r / S, G (r + 1) / S) (G = d / 16).  Every CTA reads its partial
// sums out of tensor memory (tcgen05.ld; warps w and w + 4 share TMEM lane
// quarter w and split its groups) and stores each group's 16 values into the
// owner's shared memory (st.shared::cluster into the owner's ring, which the
// first cluster barrier has freed); after the second cluster barrier the
// owner adds the S partials in split order (a fixed order, so the result
// does not depend on timing), rounds to bf16, rotates with the table and
// stores.  So every SM streams 1/S of a head's weights, and the RoPE work
// of a head is spread over its S CTAs.
//
// Every mbarrier wait is bounded; after a timeout (error bit set) the CTA
// still takes both cluster barriers (every thread of every CTA reaches them
// on every path: there is no early exit), frees its tensor memory and skips
// its stores.
#include "pkv_internal.h"
#include "pkv_device.cuh"
#include "umma.cuh"

namespace pkv {
namespace {

using namespace dev;

constexpr int kQkvThreads = 192;            // 6 warps: producer, MMA, 4 for the table and the epilogue
constexpr int kQkvM = 128;                     // tokens per tile (TMEM lanes, rows of A)
constexpr int kQkvBK = 64;                     // hidden elements per stage: one 128-byte row
constexpr int kQkvMaxStages = 8;
#ifndef PKV_QKV_BUDGET_KB
#define PKV_QKV_BUDGET_KB 200
#endif
constexpr int kQkvBudgetWide = PKV_QKV_BUDGET_KB * 1024;   // ring + table: one CTA per SM
constexpr int kQkvBudgetNarrow = 104 * 1024;   // two CTAs per SM
constexpr int kQkvSmemLimit = 1024 + 220 * 1024;
constexpr int kQkvRecvRow = 80;                // bytes per row of received partials (64 + 16: no bank conflicts)
constexpr uint64_t kQkvWaitNs = 500ull * 1000ull * 1000ull;

// Instruction descriptor of the projection's MMA: M = 128 token rows, N = d.
template <int N>
__host__ __device__ constexpr uint32_t qkv_idesc()
{
    return umma_idesc_bf16<kQkvM, N>();
}

// The shared-memory address of the same variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t cluster_map(uint32_t local, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
    return r;
}


// Every thread of every CTA of the cluster; orders the shared::cluster stores
// before it against the loads after it.
__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ void st_cluster_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// Bytes of one ring stage's x area: at least the part of the 128-row A
// operand not covered by the weight tile that follows it, so every row the
// MMA reads lies inside the stage.
__host__ __device__ __forceinline__ int qkv_x_area(int x_rows, int D)
{
    const int need = x_rows * kQkvBK * 2, floor = kQkvM * kQkvBK * 2 - D * kQkvBK * 2;
    return ((need > floor ? need : floor) + 1023) & ~1023;
}

// Groups of 8 rotation pairs owned by CTA r of an S-way split (G = d / 16).
__host__ __device__ __forceinline__ int qkv_group0(int G, int S, int r) { return G * r / S; }
__host__ __device__ __forceinline__ int qkv_groups_max(int G, int S) { return (G + S - 1) / S; }
// (cos, sin) entries per table row: the own pairs plus one, so that rows
// 16 bytes x odd apart fall on different banks
__host__ __device__ __forceinline__ int qkv_tab_row(int G, int S) { return 8 * qkv_groups_max(G, S) + 1; }

template <int D>
__global__ void __launch_bounds__(kQkvThreads, 2)
qkv_rope_append_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                       const QkvParams p)
{
    constexpr int HALF = D / 2, G = D / 16;
    constexpr uint32_t kCols = D;           // fp32 accumulator columns (64 or 128: a power of two >= 32)
    constexpr int WB = D * kQkvBK * 2;      // weight tile bytes per stage
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kQkvMaxStages], s_empty[kQkvMaxStages], s_done;
    __shared__ uint32_t s_tmem;
    __shared__ int s_fail;
    __shared__ double s_theta[HALF];        // inverse frequencies of this CTA's pairs
    __shared__ int s_L[kQkvM];              // position of token row r (-1: out of range)
    __shared__ long long s_dst[kQkvM];      // q_out row (t Hq + h) or pool row; -1: nothing to store
    __shared__ float s_scale[kQkvM];        // E4M3 scale of the destination page

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int S = p.split, rank = blockIdx.x;               // the cluster spans blockIdx.x
    const int head = blockIdx.y, m0 = blockIdx.z * kQkvM;   // head over q, then k, then v
    const int KB = p.hidden / kQkvBK;
    const int kb0 = KB * rank / S, nkb = KB * (rank + 1) / S - kb0;
    const int g0 = qkv_group0(G, S, rank), ng = qkv_group0(G, S, rank + 1) - g0;
    const int rows = min(kQkvM, p.batch - m0);              // tokens of this tile
    const int XA = qkv_x_area(p.x_rows, D), STB = XA + WB, depth = p.stages;
    const int kind = head < p.Hq ? 0 : (head < p.Hq + p.Hkv ? 1 : 2);   // q, k, v
    const int hh = kind == 0 ? head : (kind == 1 ? head - p.Hq : head - p.Hq - p.Hkv);

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t stage0 = (raw + 1023u) & ~1023u;
    double2* tab = reinterpret_cast<double2*>(smem_raw + (stage0 - raw) + p.ring_bytes);   // [x_rows][TP]
    const int TP = qkv_tab_row(G, S);
    const uint32_t full0 = smem_u32(&s_full[0]), empty0 = smem_u32(&s_empty[0]), done = smem_u32(&s_done);
    // stage i of the ring: x rows m0.. (x_rows <= 128 of them; the MMA reads
    // 128 rows from the stage start, rows past x_rows only feed accumulator
    // rows of no token) and the head's d weight rows of 64-block kb0 + i
    auto load_stage = [&](int i) {
        const int s = i % depth, kb = kb0 + i;
        const uint32_t a = stage0 + (uint32_t)(s * STB), b = a + (uint32_t)XA;
        mbar_arrive_expect_tx(full0 + 8u * s, (uint32_t)(p.x_rows * kQkvBK * 2 + WB));
        tma_load_2d(a, &tmx, kb * kQkvBK, m0, full0 + 8u * s);
        if (p.w_tiled) tma_load_2d(b, &tmw, 0, (head * KB + kb) * D, full0 + 8u * s);   // one run
        else tma_load_2d(b, &tmw, kb * kQkvBK, head * D, full0 + 8u * s);
    };

    if (tid == 0) {
        s_fail = 0;
        for (int s = 0; s < depth; ++s) {
            mbar_init(full0 + 8u * s, 1u);
            mbar_init(empty0 + 8u * s, 1u);
        }
        mbar_init(done, 1u);
        fence_mbar_init();
        // the first stages' loads go out now, while the tensor memory is allocated
        for (int i = 0; i < depth && i < nkb; ++i) load_stage(i);
    }
    if (warp == 0) {
        __syncwarp();   // converged for the aligned allocation
        tmem_alloc(smem_u32(&s_tmem), kCols);
    }
    tmem_fence_before();
    __syncthreads();
    tmem_fence_after();
    const uint32_t tmem = s_tmem;

    if (warp == 0) {
        // ---- producer: the rest of the ring's loads, each once its stage is free
        if (lane == 0) {
            for (int i = depth; i < nkb; ++i) {
                const int s = i % depth;
                if (!mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((i / depth - 1) & 1), kQkvWaitNs)) {
                    atomicOr(p.err, kErrTimeout);
                    s_fail = 1;
                    break;
                }
                load_stage(i);
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue: one thread; each stage is committed back to the producer
        if (lane == 0) {
            for (int i = 0; i < nkb; ++i) {
                const int s = i % depth;
                if (!mbar_wait_bounded(full0 + 8u * s, (uint32_t)((i / depth) & 1), kQkvWaitNs)) {
                    atomicOr(p.err, kErrTimeout);
                    s_fail = 1;
                    break;
                }
                tmem_fence_after();
                const uint32_t a = stage0 + (uint32_t)(s * STB), b = a + (uint32_t)XA;
#pragma unroll
                for (int kk = 0; kk < kQkvBK / 16; ++kk)
                    umma_bf16(tmem, sw128_kmajor_desc(a + 32u * kk), sw128_kmajor_desc(b + 32u * kk), qkv_idesc<D>(),
                              (i | kk) != 0 ? 1u : 0u);
                umma_commit(empty0 + 8u * s);
            }
            umma_commit(done);   // arrives once every MMA issued above has completed
        }
    } else {
        // ---- warps 2 to 5, while the stream runs: destinations, then the
        // rotation table of this CTA's pairs
        constexpr int kTabThreads = kQkvThreads - 64;
        const int u = tid - 64;
        for (int r = u; r < rows; r += kTabThreads) {
            const int t = m0 + r;
            const int L = p.seq_lens[t];
            const bool len_ok = L >= 0 && (long long)L < (long long)p.bt_stride * p.P;
            long long dst = -1;
            float scale = 1.f;
            if (len_ok) {
                if (kind == 0) {
                    dst = (long long)t * p.Hq + hh;
                } else {
                    const int page = p.block_tables[(size_t)t * p.bt_stride + L / p.P];
                    if (page >= 0 && page < p.num_pages) {
                        dst = ((long long)page * p.Hkv + hh) * p.P + (L % p.P);
                        if (p.fp8) scale = (kind == 1 ? p.k_scale : p.v_scale)[(size_t)page * p.Hkv + hh];
                    } else if (kind == 1 && rank == 0) {
                        atomicOr(p.err, kErrPage);
                    }
                }
            } else if (kind < 2 && rank == 0) {
                atomicOr(p.err, kErrLength);
            }
            s_L[r] = len_ok ? L : -1;
            s_dst[r] = dst;
            s_scale[r] = scale;
        }
        if (kind < 2) {
            const int np = 8 * ng;
            for (int i = u; i < np; i += kTabThreads) s_theta[i] = p.theta[8 * g0 + i];
            asm volatile("bar.sync 1, %0;" ::"n"(kTabThreads) : "memory");   // s_L and s_theta complete
            for (int it = u; it < rows * np; it += kTabThreads) {
                const int r = it / np, i = it - r * np;
                const int L = s_L[r];
                double sn = 0.0, cs = 1.0;
                if (L >= 0) dev::rope_sincos((double)L * s_theta[i], &sn, &cs);
                tab[r * TP + i] = make_double2(cs, sn);
            }
        }
    }
    // the other lanes of warps 0 and 1 wait here, not in a spin beside the
    // issuing lane, which keeps its warp's issue slots
    __syncwarp();

    const bool ok = mbar_wait_bounded(done, 0u, kQkvWaitNs);
    if (!ok && tid == 0) atomicOr(p.err, kErrTimeout);
    tmem_fence_after();
    __syncthreads();                         // s_fail, the table and the destinations settled
    cluster_sync_all();                      // every ring of the cluster is free: it becomes the receive area

    // ---- reduce-scatter: each group's 16 partial sums of every token row go
    // to the group's owner, at [sender][owner's group][row] (rows 80 bytes
    // apart: neighbouring rows on different banks) of its ring.  Warp w
    // reads TMEM lane quarter w % 4; quarters 0 and 1 have two warps (w and
    // w + 4), which take alternate groups.
    const uint32_t recv0 = stage0;
    const int quarter = warp & 3, nh = quarter + 4 < kQkvThreads / 32 ? 2 : 1, h = warp >> 2;
    if (32 * quarter < rows) {               // warp-uniform
        const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
        const int r = 32 * quarter + lane;
        for (int g4 = h; g4 < G; g4 += 4 * nh) {
            // up to 4 of this warp's groups per batch of loads: g4, g4 + nh, ...
            uint32_t v[4][16];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int g = g4 + j * nh;
                if (g < G) {
                    tmem_ld8(lane_base + (uint32_t)(8 * g), *reinterpret_cast<uint32_t(*)[8]>(&v[j][0]));
                    tmem_ld8(lane_base + (uint32_t)(HALF + 8 * g), *reinterpret_cast<uint32_t(*)[8]>(&v[j][8]));
                }
            }
            tmem_wait_ld();
            if (r < rows) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int g = g4 + j * nh;
                    if (g < G) {
                        int o = 0;
                        while (o + 1 < S && qkv_group0(G, S, o + 1) <= g) ++o;
                        const int og0 = qkv_group0(G, S, o), ong = qkv_group0(G, S, o + 1) - og0;
                        const uint32_t a = cluster_map(recv0, (uint32_t)o) +
                                           (uint32_t)(((rank * ong + (g - og0)) * p.x_rows + r) * kQkvRecvRow);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            st_cluster_v4(a + 16u * q4, v[j][4 * q4], v[j][4 * q4 + 1], v[j][4 * q4 + 2], v[j][4 * q4 + 3]);
                    }
                }
            }
        }
    }
    tmem_fence_before();
    cluster_sync_all();                      // every partial delivered; no cluster access after this
    if (warp == 0) {
        tmem_fence_after();
        tmem_dealloc(tmem, kCols);
    }

    // ---- epilogue: (own group, token row) items over all threads, rows
    // fastest (neighbouring threads read rows on different banks)
    const int items = (ok && !s_fail) ? rows * ng : 0;
    for (int it = tid; it < items; it += kQkvThreads) {
        const int gl = it / rows, r = it - gl * rows;
        const long long dst = s_dst[r];
        if (dst < 0) continue;
        float sl[8], sh[8];
        for (int s = 0; s < S; ++s) {        // split order: the same sum whatever the timing
            const uint32_t a = recv0 + (uint32_t)(((s * ng + gl) * p.x_rows + r) * kQkvRecvRow);
            const uint4 v0 = lds128(a), v1 = lds128(a + 16u), v2 = lds128(a + 32u), v3 = lds128(a + 48u);
            const uint32_t w[16] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w,
                                    v2.x, v2.y, v2.z, v2.w, v3.x, v3.y, v3.z, v3.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float fl = __uint_as_float(w[c]), fh = __uint_as_float(w[8 + c]);
                sl[c] = s == 0 ? fl : __fadd_rn(sl[c], fl);
                sh[c] = s == 0 ? fh : __fadd_rn(sh[c], fh);
            }
        }
        // the projection's bf16 outputs, as the unfused pipeline would store them
        double lo[8], hi[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            lo[c] = (double)__bfloat162float(__float2bfloat16_rn(sl[c]));
            hi[c] = (double)__bfloat162float(__float2bfloat16_rn(sh[c]));
        }
        if (kind < 2) {   // q and k are rotated at position L; v is stored as is
            const double2* tr = tab + r * TP + 8 * gl;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const double2 cssn = tr[c];
                double ylo, yhi;
                dev::rope_rotate(lo[c], hi[c], cssn.x, cssn.y, &ylo, &yhi);
                lo[c] = ylo;
                hi[c] = yhi;
            }
        }
        const int off = 8 * (g0 + gl);
        if (kind == 0 || !p.fp8) {
            uint32_t olo[4], ohi[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                olo[c] = (uint32_t)__bfloat16_as_ushort(bf16_from_f64(lo[2 * c])) |
                         ((uint32_t)__bfloat16_as_ushort(bf16_from_f64(lo[2 * c + 1])) << 16);
                ohi[c] = (uint32_t)__bfloat16_as_ushort(bf16_from_f64(hi[2 * c])) |
                         ((uint32_t)__bfloat16_as_ushort(bf16_from_f64(hi[2 * c + 1])) << 16);
            }
            __nv_bfloat16* base = kind == 0 ? p.q_out
                                            : reinterpret_cast<__nv_bfloat16*>(kind == 1 ? p.k_pool : p.v_pool);
            __nv_bfloat16* row = base + dst * D;
            *reinterpret_cast<uint4*>(row + off) = make_uint4(olo[0], olo[1], olo[2], olo[3]);
            *reinterpret_cast<uint4*>(row + HALF + off) = make_uint4(ohi[0], ohi[1], ohi[2], ohi[3]);
        } else {
            // E4M3 as the append stores it: k from the fp64 rotation over the
            // scale, v from its bf16 value over the scale (fp32 division)
            const float sc = s_scale[r];
            uint32_t w0 = 0, w1 = 0, h0 = 0, h1 = 0;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                uint8_t cl, ch;
                if (kind == 1) {
                    cl = e4m3_satfinite(__double2float_rn(__ddiv_rn(lo[c], (double)sc)));
                    ch = e4m3_satfinite(__double2float_rn(__ddiv_rn(hi[c], (double)sc)));
                } else {
                    cl = e4m3_satfinite(__fdiv_rn((float)lo[c], sc));
                    ch = e4m3_satfinite(__fdiv_rn((float)hi[c], sc));
                }
                if (c < 4) {
                    w0 |= (uint32_t)cl << (8 * c);
                    h0 |= (uint32_t)ch << (8 * c);
                } else {
                    w1 |= (uint32_t)cl << (8 * (c - 4));
                    h1 |= (uint32_t)ch << (8 * (c - 4));
                }
            }
            uint8_t* row = reinterpret_cast<uint8_t*>(kind == 1 ? p.k_pool : p.v_pool) + dst * D;
            *reinterpret_cast<uint2*>(row + off) = make_uint2(w0, w1);
            *reinterpret_cast<uint2*>(row + HALF + off) = make_uint2(h0, h1);
        }
    }
}

// One thread per 16 bytes of the tiled output: out[((h KB + kb) D + i) 64 + j]
// = w[(h D + i) hidden + kb 64 + j].
__global__ void qkv_pack_weight_kernel(const uint4* __restrict__ w, uint4* __restrict__ out, long long chunks,
                                       int hidden, int D)
{
    const int KB = hidden / kQkvBK;
    for (long long c = blockIdx.x * (long long)blockDim.x + threadIdx.x; c < chunks;
         c += (long long)gridDim.x * blockDim.x) {
        const int j8 = (int)(c & 7);                 // 16-byte chunk of the 128-byte row
        const long long r = c >> 3;                  // tiled row = (h KB + kb) D + i
        const int i = (int)(r % D);
        const long long hk = r / D;
        const int kb = (int)(hk % KB);
        const long long h = hk / KB;
        out[c] = w[(((h * D + i) * hidden) >> 3) + kb * (kQkvBK / 8) + j8];
    }
}

// Shared memory of one launch shape: the ring (which later receives the
// partials: split x own groups x x_rows x 80 bytes), then the (cos, sin)
// table (x_rows x (own pairs + 1) x 16 bytes).
struct QkvSmem {
    int stages, ring_bytes;
    size_t smem;
};

QkvSmem qkv_smem(int x_rows, int D, int S, int budget)
{
    const int G = D / 16, gmax = qkv_groups_max(G, S);
    const int stb = qkv_x_area(x_rows, D) + D * kQkvBK * 2;
    const int tab = x_rows * qkv_tab_row(G, S) * 16;
    const int recv = S * gmax * x_rows * kQkvRecvRow;
    int st = (budget - tab) / stb;
    st = st < 2 ? 2 : (st > kQkvMaxStages ? kQkvMaxStages : st);
    QkvSmem m;
    m.stages = st;
    m.ring_bytes = ((st * stb > recv ? st * stb : recv) + 1023) & ~1023;
    m.smem = 1024 + (size_t)m.ring_bytes + (size_t)tab;
    return m;
}

cudaLaunchConfig_t qkv_config(dim3 grid, size_t smem, int split, cudaStream_t stream, cudaLaunchAttribute* attr)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(kQkvThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)split;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// Clusters of this shape the GPU holds at once (0 if the query fails).
int qkv_max_clusters(int D, int heads, int tiles, int split, size_t smem)
{
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg =
        qkv_config(dim3((unsigned)split, (unsigned)heads, (unsigned)tiles), smem, split, 0, attr);
    int n = 0;
    const cudaError_t e = D == 128 ? cudaOccupancyMaxActiveClusters(&n, qkv_rope_append_kernel<128>, &cfg)
                                   : cudaOccupancyMaxActiveClusters(&n, qkv_rope_append_kernel<64>, &cfg);
    if (e != cudaSuccess) {
        (void)cudaGetLastError();
        return 0;
    }
    return n;
}

}  // namespace

cudaError_t launch_qkv_pack_weight(const __nv_bfloat16* w, __nv_bfloat16* out, int N, int hidden, int D,
                                   cudaStream_t stream)
{
    const long long chunks = (long long)N * hidden / 8;
    const long long want = (chunks + 255) / 256;
    const unsigned blocks = (unsigned)(want < 148 * 16 ? want : 148 * 16);
    qkv_pack_weight_kernel<<<blocks, 256, 0, stream>>>(reinterpret_cast<const uint4*>(w), reinterpret_cast<uint4*>(out),
                                                        chunks, hidden, D);
    return cudaGetLastError();
}

cudaError_t qkv_prepare()
{
    cudaError_t e = cudaFuncSetAttribute(qkv_rope_append_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         kQkvSmemLimit);
    if (e != cudaSuccess) return e;
    return cudaFuncSetAttribute(qkv_rope_append_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kQkvSmemLimit);
}

// The split: as many CTAs per (head, token tile) as the SMs hold in one wave
// (at most 4, at most one 64-element block of hidden each, or forced_split);
// the ring: one CTA per SM when every cluster of that shape fits on the GPU
// at once (clusters are placed whole inside a GPC, so 48 clusters of 3 need
// not fit on 148 SMs), else the smaller ring that lets two CTAs share an SM.
cudaError_t qkv_plan(int x_rows, int D, int heads, int tiles, int hidden, int num_sms, int forced_split,
                     QkvPlan* out)
{
    const int KB = hidden / kQkvBK, units = heads * tiles;
    int split = forced_split > 0 ? forced_split : num_sms / (units > 0 ? units : 1);
    split = split < 1 ? 1 : (split > kQkvMaxSplit ? kQkvMaxSplit : split);
    if (split > KB) split = KB;
    QkvSmem m = qkv_smem(x_rows, D, split, kQkvBudgetWide);
    int fit = qkv_max_clusters(D, heads, tiles, split, m.smem);
    if (fit < units) {
        const QkvSmem n = qkv_smem(x_rows, D, split, kQkvBudgetNarrow);
        const int fit2 = qkv_max_clusters(D, heads, tiles, split, n.smem);
        if (fit2 >= fit) {
            m = n;
            fit = fit2;
        }
    }
    if (m.smem > (size_t)kQkvSmemLimit) return cudaErrorInvalidConfiguration;
    out->split = split;
    out->stages = m.stages;
    out->ring_bytes = m.ring_bytes;
    out->smem = m.smem;
    out->max_clusters = fit;
    return cudaSuccess;
}

cudaError_t launch_qkv_rope_append(const QkvParams& p, const QkvPlan& plan, const CUtensorMap& tmx,
                                   const CUtensorMap& tmw, cudaStream_t stream)
{
    QkvParams q = p;
    q.split = plan.split;
    q.stages = plan.stages;
    q.ring_bytes = plan.ring_bytes;
    const dim3 grid((unsigned)plan.split, (unsigned)(p.Hq + 2 * p.Hkv), (unsigned)((p.batch + kQkvM - 1) / kQkvM));
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = qkv_config(grid, plan.smem, plan.split, stream, attr);
    if (p.D == 128) return cudaLaunchKernelEx(&cfg, qkv_rope_append_kernel<128>, tmx, tmw, q);
    return cudaLaunchKernelEx(&cfg, qkv_rope_append_kernel<64>, tmx, tmw, q);
}

}  // namespace pkv
