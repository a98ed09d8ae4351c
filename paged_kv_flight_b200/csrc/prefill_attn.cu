// prefill_attn.cu -- attention of a chunk of new tokens over the paged KV
// cache, for the requests of a varlen call that bring many new tokens at
// once: chunked prefill mixed with decode in one batch ("Scaling
// TensorRT-LLM: Kernel Fusion and Inflight Batching in Production", section
// "What the Scheduler Actually Does"; "TensorRT-LLM Guide: High-Throughput
// GPU Inference Engine", section "1. In-Flight Batching").
//
// What it computes is pkv_decode_attn_varlen's definition: token i of request
// b sits at position L_b + i - cu_q[b] and attends tokens 0 .. that position
// (the cache, the chunk's earlier tokens and itself), o = softmax(q K^T /
// sqrt(d)) V per query head, K/V of kv head h / G.
//
// Work decomposition: the plan kernel (decode_attn_tokens.cu) cuts each
// such request's chunk into blocks of kTeamWarps x 16 / G tokens; one CTA
// per (block, kv head).  The CTA's kTeamWarps consumer warps own 16 query
// rows each (16 / G consecutive tokens x the G heads of the kv head, one
// m16n8k16 row block); they all read the same K/V tiles of 16 tokens from
// one ring of shared-memory stages that a producer warp fills by TMA, so
// the block's prefix crosses HBM once for all its tokens instead of once
// per 16 / G tokens.  A stage is refilled once every consumer warp has
// released it (an mbarrier per stage counting the warps).  Each row has its
// own causal limit; a warp skips the tiles that lie wholly past its last
// token.  Slots past the block's last token may hold anything (NaN
// sentinels): the first consumer warp zeroes them in the last V tile before
// any warp reads it.  The block is not split over CTAs, so each warp writes
// its rows' output directly (no partials, no combine).
//
// Every mbarrier wait is bounded in time; a timeout sets the device error bit
// and the thread stops waiting (its results are then not valid); the
// producer waits, bounded, for its outstanding copies before the CTA exits.
#include "attn_common.cuh"

namespace pkv {
namespace {

using namespace dev;
using namespace attn;

constexpr int kTeamWarps = 8;                           // consumer warps of a block
constexpr int kTeamThreads = (kTeamWarps + 1) * 32;     // and one producer warp
// The eight warps consume a tile in a fraction of the TMA latency, so the
// ring holds many tiles (the CTA is alone on its SM: registers bound it).
#ifndef PKV_TEAM_STAGES
#define PKV_TEAM_STAGES 16
#endif
constexpr int kTeamStages = PKV_TEAM_STAGES;

// m16n8k16, bf16 A and B, all 16 rows, fp32 accumulation in place.
__device__ __forceinline__ void mma16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                      uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Shared memory of one CTA: the stages (K tile then V tile each), then a
// valid flag and the full / empty barriers of each stage.
template <int D>
constexpr size_t team_smem_bytes()
{
    using Gm = Geo<D, false>;
    return 1024 + (size_t)kTeamStages * (Gm::STAGEB + 4 + 16);
}

// p.vmap / p.vcount hold the plan's blocks {request, first q row, tokens,
// position of the first token} and their count (at most p.batch); p.q_len
// is the block length in tokens (kTeamWarps x 16 / G).
template <int D>
__global__ void __launch_bounds__(kTeamThreads, 1)
prefill_attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                    const AttnParams p)
{
    using Gm = Geo<D, false>;
    constexpr int KSTEPS = D / 16, NTD = D / 8, S = kTeamStages;

    extern __shared__ uint8_t smem_raw[];
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int v = blockIdx.x, kvh = blockIdx.y;
    if (v >= min(__ldg(p.vcount), p.batch)) return;      // the whole CTA: no barrier is used yet
    const int4 e = p.vmap[v];
    const int b = e.x, q0 = e.y, nq = e.z, pos0 = e.w;
    const int G = p.G, TPW = kTile / G;                   // tokens per consumer warp
    const long long cap = (long long)p.bt_stride * p.P;
    if (pos0 < 0 || (long long)pos0 + nq > cap || nq <= 0) {
        // impossible length: zeros for the block's rows of this kv head and an error bit
        if (tid == 0 && kvh == 0) atomicOr(p.err, kErrLength);
        for (int i = tid; i < nq * G * D / 2; i += kTeamThreads) {
            const int t = i / (G * D / 2), rem = i - t * (G * D / 2);
            uint32_t* row = reinterpret_cast<uint32_t*>(p.out + ((size_t)(q0 + t) * p.Hq + (size_t)kvh * G) * D);
            row[rem] = 0u;
        }
        return;
    }
    const int n_max = pos0 + nq;                          // keys 0 .. n_max - 1
    const int ntiles = (n_max + kTile - 1) / kTile;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t stage0 = (raw + 1023u) & ~1023u;
    uint8_t* const area = smem_raw + (stage0 - raw);
    int* const s_valid = reinterpret_cast<int*>(area + S * Gm::STAGEB);
    const uint32_t full0 = smem_u32(s_valid + S + (S & 1));          // 8-byte aligned
    const uint32_t empty0 = full0 + 8u * S;
    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full0 + 8u * s, 1u);
            mbar_init(empty0 + 8u * s, (uint32_t)kTeamWarps);
        }
        fence_mbar_init();
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
    }
    __syncthreads();

    if (warp == kTeamWarps) {
        // ---- producer: page ids of 32 tiles at a time in the lanes, lane 0 issues
        bool dead = false;
        int issued = 0;
        int la_row = 0, la_ok = 0;
        for (int i = 0; i < ntiles; ++i) {
            if ((i & 31) == 0) {
                const int t = i + lane;
                la_ok = 0;
                if (t < ntiles) {
                    const int tok0 = t * kTile, lp = tok0 / p.P;
                    const int page = __ldg(&p.block_tables[(size_t)b * p.bt_stride + lp]);
                    la_ok = 2;
                    if ((unsigned)page < (unsigned)p.num_pages) {
                        la_ok = 1;
                        la_row = (page * p.Hkv + kvh) * p.P + (tok0 - lp * p.P);
                    }
                }
            }
            const int ok = __shfl_sync(kFull, la_ok, i & 31);
            const int row = __shfl_sync(kFull, la_row, i & 31);
            if (lane == 0 && !dead) {
                const int s = i % S;
                if (i >= S && !mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((i / S - 1) & 1), kWaitLimitNs)) {
                    dead = true;
                    atomicOr(p.err, kErrTimeout);
                } else {
                    s_valid[s] = ok == 1;
                    const uint32_t bar = full0 + 8u * s;
                    if (ok == 1) {
                        mbar_arrive_expect_tx(bar, (uint32_t)Gm::STAGEB);
                        const uint32_t kdst = stage0 + (uint32_t)(s * Gm::STAGEB), vdst = kdst + Gm::TILEB;
#pragma unroll
                        for (int j = 0; j < Gm::NBOX; ++j) {
                            tma_load_2d(kdst + j * Gm::BOX_BYTES, &tmk, j * (Gm::BOXB / Gm::ELEM), row, bar);
                            tma_load_2d(vdst + j * Gm::BOX_BYTES, &tmv, j * (Gm::BOXB / Gm::ELEM), row, bar);
                        }
                    } else {
                        atomicOr(p.err, kErrPage);
                        mbar_arrive(bar);
                    }
                    ++issued;
                }
            }
        }
        // no copy may still be landing in this CTA's shared memory when it exits
        if (lane == 0)
            for (int k = max(0, issued - S); k < issued; ++k)
                (void)mbar_wait_bounded(full0 + 8u * (k % S), (uint32_t)((k / S) & 1), kWaitLimitNs / 8);
        return;
    }

    // ---- consumers: warp w owns tokens [w TPW, w TPW + TPW) of the block
    const int g = lane >> 2, c4 = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;
    const int tokK = ((mi >> 1) << 3) + ri, tokV = ((mi & 1) << 3) + ri;
    const int t_lo = warp * TPW;
    const int my_n = max(0, min(nq - t_lo, TPW));        // tokens of this warp
    const int Rw = my_n * G;                             // its query rows (row r = t G + h)
    // keys visible to rows g and g + 8; tiles holding any key this warp sees
    const int lim0 = g < Rw ? pos0 + t_lo + g / G + 1 : 0;
    const int lim1 = g + 8 < Rw ? pos0 + t_lo + (g + 8) / G + 1 : 0;
    const int ntiles_w = Rw > 0 ? (pos0 + t_lo + my_n + kTile - 1) / kTile : 0;

    uint32_t qa[KSTEPS][4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int r = g + 8 * half;
        const bool ok = r < Rw;
        const int t = ok ? r / G : 0, h = ok ? r - t * G : 0;
        const __nv_bfloat16* qrow = p.q + (((size_t)q0 + t_lo + t) * p.Hq + (size_t)kvh * G + h) * D;
#pragma unroll
        for (int ks = 0; ks < KSTEPS; ++ks) {
            qa[ks][half] = ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4) : 0u;
            qa[ks][2 + half] = ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4) : 0u;
        }
    }
    float o[NTD][4];
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    bool dead = false;
    const int tail_rows = n_max - (ntiles - 1) * kTile;  // valid rows of the last tile

    for (int i = 0; i < ntiles; ++i) {
        const int s = i % S;
        const uint32_t parity = (uint32_t)((i / S) & 1);
        if (!dead) {
            const bool ok = __all_sync(kFull, mbar_wait_bounded(full0 + 8u * s, parity, kWaitLimitNs));
            if (!ok) {
                dead = true;
                if (lane == 0) atomicOr(p.err, kErrTimeout);
            }
        }
        const uint32_t kb = stage0 + (uint32_t)(s * Gm::STAGEB), vb = kb + Gm::TILEB;
        if (i == ntiles - 1 && tail_rows < kTile) {
            // slots past the block's last token: zero them in V once, for all warps
            if (warp == 0 && !dead && s_valid[s]) {
                constexpr int CPR = Gm::ROWB / 16;
                for (int c = lane; c < (kTile - tail_rows) * CPR; c += 32) {
                    const int r = tail_rows + c / CPR, ch = c % CPR;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + tile_off<D, false>(r, ch)),
                                 "r"(0u)
                                 : "memory");
                }
            }
            asm volatile("bar.sync 1, %0;" ::"n"(kTeamWarps * 32) : "memory");
        }
        if (!dead && i < ntiles_w && s_valid[s]) {
            const int tok0 = i * kTile;
            float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ks += 2) {
                uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
                ldsm_x4(kb + tile_off<D, false>(tokK, 2 * ks + (mi & 1)), r0, r1, r2, r3);
                ldsm_x4(kb + tile_off<D, false>(tokK, 2 * ks + 2 + (mi & 1)), r4, r5, r6, r7);
                mma16(sa[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r0, r1);
                mma16(sa[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r2, r3);
                mma16(sb[0], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], r4, r5);
                mma16(sb[1], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], r6, r7);
            }
            // online softmax per row in log2 units; keys at or past a row's limit are -inf
            float sc[2][4], mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const int tok = tok0 + 8 * j + 2 * c4 + (q & 1);
                    sc[j][q] = (tok < ((q >> 1) ? lim1 : lim0)) ? (sa[j][q] + sb[j][q]) * p.scale_log2 : -INFINITY;
                    mx[q >> 1] = fmaxf(mx[q >> 1], sc[j][q]);
                }
            float alpha[2], m_ref[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(kFull, mx[hf], 1));
                mx[hf] = fmaxf(mx[hf], __shfl_xor_sync(kFull, mx[hf], 2));
                const float m_new = fmaxf(m_run[hf], mx[hf]);
                m_ref[hf] = (m_new == -INFINITY) ? 0.f : m_new;
                alpha[hf] = ex2(m_run[hf] - m_ref[hf]);
                m_run[hf] = m_new;
            }
            // P as the A operand (bf16), l summed from the rounded values
            const uint32_t pa0 = pack_bf16(ex2(sc[0][0] - m_ref[0]), ex2(sc[0][1] - m_ref[0]));
            const uint32_t pa1 = pack_bf16(ex2(sc[0][2] - m_ref[1]), ex2(sc[0][3] - m_ref[1]));
            const uint32_t pa2 = pack_bf16(ex2(sc[1][0] - m_ref[0]), ex2(sc[1][1] - m_ref[0]));
            const uint32_t pa3 = pack_bf16(ex2(sc[1][2] - m_ref[1]), ex2(sc[1][3] - m_ref[1]));
            l_run[0] = l_run[0] * alpha[0] + ((bf16_lo(pa0) + bf16_hi(pa0)) + (bf16_lo(pa2) + bf16_hi(pa2)));
            l_run[1] = l_run[1] * alpha[1] + ((bf16_lo(pa1) + bf16_hi(pa1)) + (bf16_lo(pa3) + bf16_hi(pa3)));
            if (__any_sync(kFull, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
                for (int nt = 0; nt < NTD; ++nt) {
                    o[nt][0] *= alpha[0];
                    o[nt][1] *= alpha[0];
                    o[nt][2] *= alpha[1];
                    o[nt][3] *= alpha[1];
                }
            }
            // O += P V
#pragma unroll
            for (int dj = 0; dj < D / 16; ++dj) {
                uint32_t r0, r1, r2, r3;
                ldsm_x4_trans(vb + tile_off<D, false>(tokV, 2 * dj + (mi >> 1)), r0, r1, r2, r3);
                mma16(o[2 * dj], pa0, pa1, pa2, pa3, r0, r1);
                mma16(o[2 * dj + 1], pa0, pa1, pa2, pa3, r2, r3);
            }
        }
        // release the stage to the producer
        __syncwarp();
        if (lane == 0) mbar_arrive(empty0 + 8u * s);
    }

    // ---- this warp's rows: out[q0 + t_lo + t][kvh G + h] = o / l
    if (dead) return;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
        float lsum = l_run[hf] + __shfl_xor_sync(kFull, l_run[hf], 1);
        lsum += __shfl_xor_sync(kFull, lsum, 2);
        const int r = g + 8 * hf;
        if (r >= Rw) continue;
        const int t = r / G, h = r - t * G;
        const float inv = 1.f / lsum;
        uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + (((size_t)q0 + t_lo + t) * p.Hq + (size_t)kvh * G + h) * D);
#pragma unroll
        for (int nt = 0; nt < NTD; ++nt)
            dst[(8 * nt + 2 * c4) >> 1] = pack_bf16(o[nt][2 * hf] * inv, o[nt][2 * hf + 1] * inv);
    }
}

}  // namespace

int prefill_block_tokens(int G) { return kTeamWarps * (kTile / G); }

cudaError_t prefill_prepare(int head_dim)
{
    if (head_dim == 128)
        return cudaFuncSetAttribute(prefill_attn_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)team_smem_bytes<128>());
    return cudaFuncSetAttribute(prefill_attn_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)team_smem_bytes<64>());
}

cudaError_t launch_prefill_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                                int grid_blocks, cudaStream_t stream)
{
    if (grid_blocks <= 0) return cudaSuccess;
    const dim3 grid(grid_blocks, p.Hkv), block(kTeamThreads);
    if (head_dim == 128)
        prefill_attn_kernel<128><<<grid, block, team_smem_bytes<128>(), stream>>>(tmk, tmv, p);
    else
        prefill_attn_kernel<64><<<grid, block, team_smem_bytes<64>(), stream>>>(tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace pkv
