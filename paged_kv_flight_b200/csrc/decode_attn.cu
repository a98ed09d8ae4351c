// decode_attn.cu -- step part 2: grouped-query decode attention of one new
// query per request over its paged KV cache, split over all SMs.
//
// What it computes: o_h = softmax(q_h K^T / sqrt(d)) V over the request's
// n_b = L_b + 1 tokens, K/V of kv head h / G.  Page lookup happens inside the
// kernel ("Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
// Production", section "The Paged KV-Cache"); each KV element is read once
// for all G query heads sharing it ("TensorRT-LLM Guide: High-Throughput GPU
// Inference Engine", section "3. Custom Fused Attention Kernels: FMHA and
// XQA"); scores and softmax never leave registers (first page, section "What
// Gets Fused", Attention bullet).  E4M3 KV is dequantised in registers
// ("TensorRT-LLM Guide", section "4. Native FP8 Quantization").
//
// Work decomposition (no host sync, one launch):
//   * every CTA derives tiles-per-request (16 tokens per tile; 32 for E4M3
//     pools whose pages hold 32 tokens or more) from seq_lens
//     and keeps their exclusive prefix in shared memory;
//   * the flattened sequence of tiles, ordered (request, kv head, tile), is cut
//     into W equal contiguous ranges, one per warp worker (W <= warps x SMs),
//     so every worker streams the same number of bytes whatever the length
//     skew of the batch;
//   * optionally each range is cut into units: a static head that its own
//     warp streams, and (for ranges of 32 tiles or more) a tail of its last
//     quarter (at most 48 tiles) cut into K chunks of at least 4 tiles.  A
//     warp that has finished its head claims tail chunks of any range from
//     one atomic counter, so warps that the memory system served faster take
//     over the work of slower ones and all finish within about one chunk of
//     each other;
//   * a (request, kv head) pair that lies inside one unit is finished there; a
//     pair cut between units leaves one partial (unnormalised o, running max
//     m, sum l) per unit, stored without any fence; a small combine kernel
//     launched right after merges them by log-sum-exp (one CTA per pair) and
//     resets the chunk counter.  No worker waits for another.
//
// Per warp: a private ring of `stages` K+V tile buffers filled by 2-D TMA
// tile loads (128-byte or 64-byte swizzle) that complete on one mbarrier per
// stage; the warp's lane 0 issues the loads from a double-buffered 32-tile
// lookahead of page ids (and E4M3 scales), the warp consumes: QK^T and P V
// on warp-level mma.sync (query heads padded to 16 mma rows), online softmax
// in log2 units with quad shuffles, fp32 accumulators rescaled only when the
// running max moves.  The next pair's query fragments are fetched one tile
// ahead.  Every mbarrier wait is bounded in time; a timeout marks the worker
// dead, sets a device error bit and lets the control flow (and the combine
// protocol) run to the end without touching data.
#include <math.h>

#include "attn_common.cuh"

namespace pkv {
namespace {

using namespace dev;
using namespace attn;

// Query fragments of (request b, kv head kvh) for the mma A operand: row g =
// query head kvh*G + g (zero for g >= G), k-step ks covers d in [16ks, 16ks+16).
// bf16 path: a0 = d 16ks+2c..+1, a2 = d 16ks+8+2c..+1.  fp8 path (f16 operands):
// the k order inside a k-step follows the byte layout of E4M3 rows, a0 = d
// 16ks+4c..+1, a2 = d 16ks+4c+2..+3 (raw bf16 here, converted at pair start).
template <int D, bool FP8>
__device__ __forceinline__ void load_q(const AttnParams& p, int b, int kvh, int g, int c4,
                                       uint32_t (&qa)[D / 16][2])
{
    const __nv_bfloat16* qrow = p.q + ((size_t)b * p.Hq + (size_t)kvh * p.G + g) * D;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
        if (g < p.G) {
            if constexpr (!FP8) {
                qa[ks][0] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4);
                qa[ks][1] = *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4);
            } else {
                const uint2 v = *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * c4);
                qa[ks][0] = v.x;
                qa[ks][1] = v.y;
            }
        } else {
            qa[ks][0] = qa[ks][1] = 0u;
        }
    }
}

template <int D, bool FP8, int WARPS, int TT>
__global__ void __launch_bounds__(WARPS * 32, 1)
decode_attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                   const AttnParams p)
{
    using Gm = Geo<D, FP8, TT>;
    constexpr int KSTEPS = D / 16;      // mma k-steps along d for QK^T
    constexpr int NTD = D / 8;          // mma n-tiles along d for P V
    constexpr int NT = WARPS * 32;

    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp_tot[WARPS];
    __shared__ int s_bad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.batch, Hkv = p.Hkv, P = p.P, S = p.stages;

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t stage_area = (raw + 1023u) & ~1023u;
    uint8_t* const area_ptr = smem_raw + (stage_area - raw);
    StageInfo* const info_all = reinterpret_cast<StageInfo*>(area_ptr + WARPS * S * Gm::STAGEB);
    uint8_t* const bar_ptr = reinterpret_cast<uint8_t*>(info_all + WARPS * S);
    int* const prefix = reinterpret_cast<int*>(bar_ptr + WARPS * S * 8);

    if (tid == 0) {
        s_bad = 0;
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
    }
    // the combine launched after this grid as its programmatic dependent may
    // take SMs as they free up: it derives the split and then waits for this
    // grid to finish before it reads anything this grid writes
    grid_launch_dependents();
    __syncthreads();

    // ---- 1. tiles per request and their exclusive prefix ----------------------
    const long long cap = (long long)p.bt_stride * P;
    const int per = (B + NT - 1) / NT;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    int local = 0;
    for (int b = lo; b < hi; ++b) {
        const int L = p.seq_lens[b];
        const bool ok = L >= 0 && (long long)L < cap;
        const int nt = ok ? (L + TT) / TT : 0;   // ceil((L + 1) / TT)
        if (!ok) s_bad = 1;
        prefix[b] = nt;
        local += nt;
    }
    int incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp_tot[warp] = incl;
    __syncthreads();
    int run = incl - local;
    for (int w2 = 0; w2 < warp; ++w2) run += s_warp_tot[w2];
    for (int b = lo; b < hi; ++b) {
        const int c = prefix[b];
        prefix[b] = run;
        run += c;
    }
    if (tid == NT - 1) prefix[B] = run;
    __syncthreads();

    if (s_bad && blockIdx.x == 0) {
        // requests with an impossible length produce zeros and an error bit
        if (tid == 0) atomicOr(p.err, kErrLength);
        for (int b = warp; b < B; b += WARPS) {
            const int L = p.seq_lens[b];
            if (L >= 0 && (long long)L < cap) continue;
            uint32_t* o32 = reinterpret_cast<uint32_t*>(p.out + (size_t)b * p.Hq * D);
            for (int i = lane; i < p.Hq * D / 2; i += 32) o32[i] = 0u;
        }
    }

    // ---- 2. split geometry and this warp's head unit ------------------------------
    const long long T = (long long)prefix[B] * Hkv;
    const int W = split_workers(T, (long long)gridDim.x * WARPS, p.workers);
    const Split sp = make_split(max(T, 1LL), W, p.tail_chunks);
    if (blockIdx.x == 0) {
        // the combine kernel that follows needs the same split geometry
        if (tid == 0) {
            p.meta[0] = W;
            p.meta[1] = (int)(T & 0xFFFFFFFFll);
            p.meta[2] = (int)(T >> 32);
            p.meta[3] = sp.K;
        }
        for (int b = tid; b <= B; b += NT) p.meta[4 + b] = prefix[b];
    }
    if (T == 0) return;
    const int w = warp * gridDim.x + blockIdx.x;   // spread workers over SMs first
    if (w >= W) return;
    const long long n_chunks = (long long)W * sp.K;

    const uint32_t my_stage0 = stage_area + (uint32_t)(warp * S * Gm::STAGEB);
    StageInfo* const my_info = info_all + warp * S;
    const uint32_t my_bar0 = smem_u32(bar_ptr) + (uint32_t)(warp * S * 8);
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(my_bar0 + 8u * s, 1u);
        fence_mbar_init();
    }
    __syncwarp();

    // ---- 3. producer: units in issue order, 32-tile lookahead, TMA issue ------------
    // The producer issues the tiles of its current unit [pu0, pu0 + p_left
    // ...) from two 32-tile lookahead windows (la_cur from index la_i, la_nxt;
    // la_fill is the first tile of the window after them).  When kClaimAhead
    // tiles of the unit are left to issue it claims the next tail chunk
    // (atomic on the chunk counter); when kResolveAhead are left it reads the
    // claim and starts the page-id (and scale) loads of the next unit's first
    // window (nU, la_new), so that neither latency stalls the first issue of
    // the next unit.
    constexpr int kNone = -1, kPending = -2;
    constexpr int kClaimAhead = 4, kResolveAhead = 2;
    int pU = w * (sp.K + 1);
    long long pu0 = sp.ustart(pU), pu1 = sp.ustart(pU + 1);
    int p_left = (int)(pu1 - pu0);   // a head holds at most T / W + 1 tiles
    int la_i = 0;
    long long la_fill = pu0 + 64;
    Lookahead la_cur = lookahead_fill<FP8, TT>(p, prefix, pu0, pu1, lane);
    Lookahead la_nxt = lookahead_fill<FP8, TT>(p, prefix, pu0 + 32, pu1, lane);
    int nU = sp.K > 0 ? kPending : kNone;
    long long nu0 = 0, nu1 = 0;
    Lookahead la_new{0, 0, 1.f, 1.f};
    int claim = 0;
    bool claim_sent = false;

    // issues the next tile of this warp's sequence into stage s; false when
    // there is none left
    auto issue_next = [&](int s) -> bool {
        if (p_left == 0) {
            if (nU < 0) return false;
            pU = nU;
            pu0 = nu0;
            pu1 = nu1;
            p_left = (int)(nu1 - nu0);
            la_i = 0;
            la_cur = la_new;
            la_nxt = lookahead_fill<FP8, TT>(p, prefix, nu0 + 32, nu1, lane);
            la_fill = nu0 + 64;
            nU = kPending;
        }
        if (la_i == 32) {
            la_i = 0;
            la_cur = la_nxt;
            la_nxt = lookahead_fill<FP8, TT>(p, prefix, la_fill, pu1, lane);
            la_fill += 32;
        }
        const int src = la_i++;
        --p_left;
        const int v = __shfl_sync(kFull, la_cur.valid, src);
        const int row = __shfl_sync(kFull, la_cur.row, src);
        float ks = 1.f, vs = 1.f;
        if (FP8) {
            ks = __shfl_sync(kFull, la_cur.ks, src);
            vs = __shfl_sync(kFull, la_cur.vs, src);
        }
        if (lane == 0) {
            const uint32_t bar = my_bar0 + 8u * s;
            StageInfo si;
            si.ks = ks;
            si.vs = vs;
            si.valid = (v == 1);
            si.pad = 0;
            my_info[s] = si;
            if (v == 1) {
                mbar_arrive_expect_tx(bar, (uint32_t)Gm::STAGEB);
                const uint32_t kdst = my_stage0 + (uint32_t)(s * Gm::STAGEB);
                const uint32_t vdst = kdst + Gm::TILEB;
#pragma unroll
                for (int j = 0; j < Gm::NBOX; ++j) {
                    tma_load_2d(kdst + j * Gm::BOX_BYTES, &tmk, j * (Gm::BOXB / Gm::ELEM), row, bar);
                    tma_load_2d(vdst + j * Gm::BOX_BYTES, &tmv, j * (Gm::BOXB / Gm::ELEM), row, bar);
                }
            } else {
                atomicOr(p.err, kErrPage);
                mbar_arrive(bar);
            }
        }
        if (nU == kPending) {
            if (!claim_sent && p_left <= kClaimAhead) {
                if (lane == 0) claim = atomicAdd(p.claim, 1);
                claim_sent = true;
            }
            if (claim_sent && p_left <= kResolveAhead) {
                const int c = __shfl_sync(kFull, claim, 0);
                claim_sent = false;
                if (c >= n_chunks) {
                    nU = kNone;
                } else {
                    const int v2 = c % W;
                    nU = v2 * (sp.K + 1) + 1 + (c - v2) / W;
                    nu0 = sp.ustart(nU);
                    nu1 = sp.ustart(nU + 1);
                    la_new = lookahead_fill<FP8, TT>(p, prefix, nu0, nu1, lane);
                }
            }
        }
        return true;
    };

    // everything above reads only seq_lens and block_tables; q and the slots
    // the RoPE + append kernel writes are read after it has finished (a
    // no-op unless launched as its programmatic dependent)
    grid_dependency_wait();
    int issued = 0;
    while (issued < S && issue_next(issued)) ++issued;

    // ---- 4. consumer ----------------------------------------------------------------
    const int g = lane >> 2;     // mma row = query head within the group
    const int c4 = lane & 3;
    const int G = p.G;
    const int mi = lane >> 3, ri = lane & 7;        // ldmatrix: matrix index, row
    const int tokK = ((mi >> 1) << 3) + ri;         // token row addressed for K
    const int tokV = ((mi & 1) << 3) + ri;          // token row addressed for V (trans)

    float o[NTD][2];
    uint32_t qa[KSTEPS][2], qn[KSTEPS][2];
    float m_run = -INFINITY, l_run = 0.f;
    // E4M3: o holds the pair's P V sum over the V codes in units of the V
    // scale vs_cur (the true sum is o x vs_cur); a tile of another scale
    // rescales o by vs_cur / vs together with the softmax rescale, so the
    // P V mma accumulates into o directly
    float vs_cur = 1.f;
    int n_cur = 0, n_next = 0;
    bool dead = false;
    int k_dead = 0;
    int s = 0;
    uint32_t parity = 0;

    // consumer: unit [cu0, cu1) with index cU and c_left tiles still to
    // consume; cursor = pair (cb, ckvh) of cnt tiles, tile ctt of it.  A unit
    // is longer than the producer's lead (at most S tiles), so when the
    // consumer reaches the end of a unit the producer is already inside the
    // next one, whose bounds it still holds.
    int cU = pU;
    long long cu0 = pu0, cu1 = pu1;
    int c_left = (int)(pu1 - pu0);
    bool unit_first = true;
    int cb, ckvh, ctt, cnt;
    locate(prefix, B, Hkv, cu0, cb, ckvh, ctt, cnt);
    load_q<D, FP8>(p, cb, ckvh, g, c4, qn);
    n_next = p.seq_lens[cb] + 1;

    for (int k = 0; k < issued; ++k) {
        if (!dead) {
            const bool ok = __all_sync(kFull, mbar_wait_bounded(my_bar0 + 8u * s, parity, kWaitLimitNs));
            if (!ok) {
                dead = true;
                k_dead = k;
                if (lane == 0) atomicOr(p.err, kErrTimeout);
            }
        }
        if (dead) {
            // control flow only: no data, no writes
            if (++s == S) {
                s = 0;
                parity ^= 1u;
            }
            continue;
        }
        const StageInfo si = my_info[s];
        const bool unit_end = c_left == 1;
        const bool pair_end = ctt == cnt - 1 || unit_end;

        if (ctt == 0 || unit_first) {
            // start of a (request, kv head) pair or of a unit: take the prefetched query
#pragma unroll
            for (int ks = 0; ks < KSTEPS; ++ks) {
                if constexpr (!FP8) {
                    qa[ks][0] = qn[ks][0];
                    qa[ks][1] = qn[ks][1];
                } else {
                    qa[ks][0] = pack_f16(bf16_lo(qn[ks][0]), bf16_hi(qn[ks][0]));
                    qa[ks][1] = pack_f16(bf16_lo(qn[ks][1]), bf16_hi(qn[ks][1]));
                }
            }
            n_cur = n_next;
#pragma unroll
            for (int nt = 0; nt < NTD; ++nt) o[nt][0] = o[nt][1] = 0.f;
            m_run = -INFINITY;
            l_run = 0.f;
            vs_cur = 1.f;
            unit_first = false;
        }
        if (pair_end && k + 1 < issued) {
            // the next tile starts another pair: fetch its query now
            int nb = cb, nkvh = ckvh + 1;
            if (unit_end) {
                int ntt, ncnt;
                locate(prefix, B, Hkv, pu0, nb, nkvh, ntt, ncnt);   // the producer's unit is the next one
            } else if (nkvh == Hkv) {
                nkvh = 0;
                do { ++nb; } while (nb < B - 1 && prefix[nb + 1] == prefix[nb]);
            }
            load_q<D, FP8>(p, nb, nkvh, g, c4, qn);
            n_next = p.seq_lens[nb] + 1;
        }

        bool zeroed = false;
        if (si.valid) {
            const uint32_t kb = my_stage0 + (uint32_t)(s * Gm::STAGEB);
            const uint32_t vb = kb + Gm::TILEB;
            const int tok0 = ctt * TT;
            const int rows_valid = min(TT, n_cur - tok0);
            if (rows_valid < TT) {
                // slots past the request's end may hold anything (NaN): zero them in V
                constexpr int CPR = Gm::ROWB / 16;
                const int nch = (TT - rows_valid) * CPR;
                for (int e = lane; e < nch; e += 32) {
                    const int r = rows_valid + e / CPR, ch = e % CPR;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + tile_off<D, FP8, TT>(r, ch)),
                                 "r"(0u)
                                 : "memory");
                }
                zeroed = true;
                __syncwarp();
            }
            // S = Q K^T (NJ n-tiles of 8 tokens), two accumulation chains
            constexpr int NJ = TT / 8;
            float sa[NJ][2], sb[NJ][2];
#pragma unroll
            for (int j = 0; j < NJ; ++j) sa[j][0] = sa[j][1] = sb[j][0] = sb[j][1] = 0.f;
            if constexpr (!FP8) {
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ks += 2) {
                    uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
                    ldsm_x4(kb + tile_off<D, FP8, TT>(tokK, 2 * ks + (mi & 1)), r0, r1, r2, r3);
                    ldsm_x4(kb + tile_off<D, FP8, TT>(tokK, 2 * ks + 2 + (mi & 1)), r4, r5, r6, r7);
                    mma_bf16_r8(sa[0][0], sa[0][1], qa[ks][0], qa[ks][1], r0, r1);
                    mma_bf16_r8(sa[1][0], sa[1][1], qa[ks][0], qa[ks][1], r2, r3);
                    mma_bf16_r8(sb[0][0], sb[0][1], qa[ks + 1][0], qa[ks + 1][1], r4, r5);
                    mma_bf16_r8(sb[1][0], sb[1][1], qa[ks + 1][0], qa[ks + 1][1], r6, r7);
                }
            } else {
#pragma unroll
                for (int s4 = 0; s4 < D / 32; ++s4)
#pragma unroll
                    for (int h16 = 0; h16 < TT / 16; ++h16) {   // tokens 16 h16 .. 16 h16 + 15
                        uint32_t r0, r1, r2, r3;
                        ldsm_x4(kb + tile_off<D, FP8, TT>(16 * h16 + tokK, 2 * s4 + (mi & 1)), r0, r1, r2, r3);
                        // two n-tiles: even and odd k-steps on separate chains; four
                        // n-tiles already make four independent chains (fewer registers)
                        float(&odd)[NJ][2] = NJ == 2 ? sb : sa;
                        mma_f16_r8(sa[2 * h16][0], sa[2 * h16][1], qa[2 * s4][0], qa[2 * s4][1], cvt_lo(r0),
                                   cvt_hi(r0));
                        mma_f16_r8(odd[2 * h16][0], odd[2 * h16][1], qa[2 * s4 + 1][0], qa[2 * s4 + 1][1],
                                   cvt_lo(r1), cvt_hi(r1));
                        mma_f16_r8(sa[2 * h16 + 1][0], sa[2 * h16 + 1][1], qa[2 * s4][0], qa[2 * s4][1], cvt_lo(r2),
                                   cvt_hi(r2));
                        mma_f16_r8(odd[2 * h16 + 1][0], odd[2 * h16 + 1][1], qa[2 * s4 + 1][0], qa[2 * s4 + 1][1],
                                   cvt_lo(r3), cvt_hi(r3));
                    }
            }

            // online softmax in log2 units; masked tokens are -inf (never 0 * NaN)
            const float slog2 = FP8 ? p.scale_log2 * si.ks : p.scale_log2;
            float sc[NJ][2];
            float mx = -INFINITY;
#pragma unroll
            for (int j = 0; j < NJ; ++j)
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int tok = tok0 + 8 * j + 2 * c4 + e;
                    sc[j][e] = (tok < n_cur) ? (sa[j][e] + sb[j][e]) * slog2 : -INFINITY;
                    mx = fmaxf(mx, sc[j][e]);
                }
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
            const float m_new = fmaxf(m_run, mx);
            const float m_ref = (m_new == -INFINITY) ? 0.f : m_new;
            const float alpha = ex2(m_run - m_ref);
            // P as the A operand of the P V mma, one k-step of 16 tokens per h16:
            // a0 = tokens 16 h16 + 2c4, +1; a2 = tokens 16 h16 + 8 + 2c4, +1
            uint32_t pa0[TT / 16], pa2[TT / 16];
            float psum = 0.f;
#pragma unroll
            for (int h16 = 0; h16 < TT / 16; ++h16) {
                const float p00 = ex2(sc[2 * h16][0] - m_ref), p01 = ex2(sc[2 * h16][1] - m_ref);
                const float p10 = ex2(sc[2 * h16 + 1][0] - m_ref), p11 = ex2(sc[2 * h16 + 1][1] - m_ref);
                if constexpr (!FP8) {
                    pa0[h16] = pack_bf16(p00, p01);
                    pa2[h16] = pack_bf16(p10, p11);
                    psum += (bf16_lo(pa0[h16]) + bf16_hi(pa0[h16])) + (bf16_lo(pa2[h16]) + bf16_hi(pa2[h16]));
                } else {
                    pa0[h16] = pack_f16(p00, p01);
                    pa2[h16] = pack_f16(p10, p11);
                    const float2 f0 = f16x2_to_f32(pa0[h16]), f2 = f16x2_to_f32(pa2[h16]);
                    psum += (f0.x + f0.y) + (f2.x + f2.y);
                }
            }
            l_run = l_run * alpha + psum;
            m_run = m_new;
            float rescale = alpha;
            if constexpr (FP8) {
                rescale = alpha * (vs_cur / si.vs);
                vs_cur = si.vs;
            }
            if (__any_sync(kFull, rescale != 1.f)) {
#pragma unroll
                for (int nt = 0; nt < NTD; ++nt) {
                    o[nt][0] *= rescale;
                    o[nt][1] *= rescale;
                }
            }

            // O += P V
            if constexpr (!FP8) {
#pragma unroll
                for (int dj = 0; dj < D / 16; ++dj) {
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4_trans(vb + tile_off<D, FP8, TT>(tokV, 2 * dj + (mi >> 1)), r0, r1, r2, r3);
                    mma_bf16_r8(o[2 * dj][0], o[2 * dj][1], pa0[0], pa2[0], r0, r1);
                    mma_bf16_r8(o[2 * dj + 1][0], o[2 * dj + 1][1], pa0[0], pa2[0], r2, r3);
                }
            } else {
                // E4M3 V: lane (n = g, c4) loads d in [DV*n, DV*n + DV) of tokens
                // 2c4, 2c4+1, 8+2c4, 9+2c4 (+16 h16); byte permutes pair tokens per
                // d, and the mma n-index j of n-tile nt stands for d = DV*j + nt.
                constexpr int DV = D / 8;
                constexpr int WORDS = DV / 4;
                // the 16-token halves unrolled: the second half's shared-memory
                // loads may issue while the first half's mma run (the tile
                // still fits the register file: 234 registers, no spills)
#pragma unroll
                for (int h16 = 0; h16 < TT / 16; ++h16) {
                    const uint32_t pl = (TT == 16 || h16 == 0) ? pa0[0] : pa0[TT / 16 - 1];
                    const uint32_t ph = (TT == 16 || h16 == 0) ? pa2[0] : pa2[TT / 16 - 1];
                    uint32_t wa[WORDS], wb[WORDS], wc[WORDS], wd[WORDS];
                    const int t0 = 16 * h16 + 2 * c4;
                    if constexpr (DV == 16) {
                        const uint4 a = lds128(vb + tile_off<D, FP8, TT>(t0, g));
                        const uint4 b = lds128(vb + tile_off<D, FP8, TT>(t0 + 1, g));
                        const uint4 cc = lds128(vb + tile_off<D, FP8, TT>(t0 + 8, g));
                        const uint4 dd = lds128(vb + tile_off<D, FP8, TT>(t0 + 9, g));
                        wa[0] = a.x; wa[1] = a.y; wa[2] = a.z; wa[3] = a.w;
                        wb[0] = b.x; wb[1] = b.y; wb[2] = b.z; wb[3] = b.w;
                        wc[0] = cc.x; wc[1] = cc.y; wc[2] = cc.z; wc[3] = cc.w;
                        wd[0] = dd.x; wd[1] = dd.y; wd[2] = dd.z; wd[3] = dd.w;
                    } else {
                        const uint32_t off8 = (uint32_t)((g & 1) * 8);
                        const uint2 a = lds64(vb + tile_off<D, FP8, TT>(t0, g >> 1) + off8);
                        const uint2 b = lds64(vb + tile_off<D, FP8, TT>(t0 + 1, g >> 1) + off8);
                        const uint2 cc = lds64(vb + tile_off<D, FP8, TT>(t0 + 8, g >> 1) + off8);
                        const uint2 dd = lds64(vb + tile_off<D, FP8, TT>(t0 + 9, g >> 1) + off8);
                        wa[0] = a.x; wa[1] = a.y;
                        wb[0] = b.x; wb[1] = b.y;
                        wc[0] = cc.x; wc[1] = cc.y;
                        wd[0] = dd.x; wd[1] = dd.y;
                    }
#pragma unroll
                    for (int kw = 0; kw < WORDS; ++kw) {
                        const uint32_t x0 = __byte_perm(wa[kw], wb[kw], 0x5140);
                        const uint32_t x1 = __byte_perm(wa[kw], wb[kw], 0x7362);
                        const uint32_t y0 = __byte_perm(wc[kw], wd[kw], 0x5140);
                        const uint32_t y1 = __byte_perm(wc[kw], wd[kw], 0x7362);
                        mma_f16_r8(o[4 * kw][0], o[4 * kw][1], pl, ph, cvt_lo(x0), cvt_lo(y0));
                        mma_f16_r8(o[4 * kw + 1][0], o[4 * kw + 1][1], pl, ph, cvt_hi(x0), cvt_hi(y0));
                        mma_f16_r8(o[4 * kw + 2][0], o[4 * kw + 2][1], pl, ph, cvt_lo(x1), cvt_lo(y1));
                        mma_f16_r8(o[4 * kw + 3][0], o[4 * kw + 3][1], pl, ph, cvt_hi(x1), cvt_hi(y1));
                    }
                }
            }
        }
        __syncwarp();

        // refill this stage with the tile `S` ahead; generic-proxy zero stores
        // above must land before the async-proxy copy that overwrites the buffer
        if (zeroed && lane == 0) fence_proxy_async_smem();
        if (issue_next(s)) ++issued;

        // ---- end of a pair (or of a unit): write out or leave a partial -----------
        if (pair_end) {
            float lsum = l_run + __shfl_xor_sync(kFull, l_run, 1);
            lsum += __shfl_xor_sync(kFull, lsum, 2);
            const long long ts = (long long)prefix[cb] * Hkv + (long long)ckvh * cnt;
            const long long te = ts + cnt;
            const size_t orow = ((size_t)cb * p.Hq + (size_t)ckvh * G + g) * D;
            if (cu0 <= ts && te <= cu1) {
                if (g < G) {
                    const float inv = (FP8 ? vs_cur : 1.f) / lsum;
                    uint32_t* dst = reinterpret_cast<uint32_t*>(p.out + orow);
                    if constexpr (!FP8) {
#pragma unroll
                        for (int nt = 0; nt < NTD; ++nt)
                            dst[(8 * nt + 2 * c4) >> 1] = pack_bf16(o[nt][0] * inv, o[nt][1] * inv);
                    } else {
                        constexpr int DV = D / 8;
#pragma unroll
                        for (int e = 0; e < 2; ++e)
#pragma unroll
                            for (int u = 0; u < DV / 2; ++u)
                                dst[(DV * (2 * c4 + e) + 2 * u) >> 1] =
                                    pack_bf16(o[2 * u][e] * inv, o[2 * u + 1][e] * inv);
                    }
                }
            } else {
                // slot 2U for the pair the unit starts in, 2U + 1 for one that starts inside it
                const int slot = 2 * cU + (cu0 < ts ? 1 : 0);
                const size_t prow = ((size_t)slot * G + g) * D;
                if (g < G) {
                    float* dst = p.part_o + prow;
                    if constexpr (!FP8) {
#pragma unroll
                        for (int nt = 0; nt < NTD; ++nt)
                            *reinterpret_cast<float2*>(dst + 8 * nt + 2 * c4) = make_float2(o[nt][0], o[nt][1]);
                    } else {
                        // the partial is the true sum: o in units of vs_cur
                        constexpr int DV = D / 8;
#pragma unroll
                        for (int e = 0; e < 2; ++e)
#pragma unroll
                            for (int u = 0; u < DV / 2; ++u)
                                *reinterpret_cast<float2*>(dst + DV * (2 * c4 + e) + 2 * u) =
                                    make_float2(o[2 * u][e] * vs_cur, o[2 * u + 1][e] * vs_cur);
                    }
                    if (c4 == 0)
                        *reinterpret_cast<float2*>(p.part_ml + ((size_t)slot * G + g) * 2) =
                            make_float2(m_run, lsum);
                }
            }
        }

        // advance the consumer cursor and the ring position
        if (unit_end) {
            if (k + 1 < issued) {
                cU = pU;
                cu0 = pu0;
                cu1 = pu1;
                c_left = (int)(pu1 - pu0);
                unit_first = true;
                locate(prefix, B, Hkv, cu0, cb, ckvh, ctt, cnt);
            }
        } else {
            --c_left;
            if (++ctt == cnt) {
                ctt = 0;
                if (++ckvh == Hkv) {
                    ckvh = 0;
                    do { ++cb; } while (cb < B && prefix[cb + 1] == prefix[cb]);
                }
                if (cb < B) cnt = prefix[cb + 1] - prefix[cb];
            }
        }
        if (++s == S) {
            s = 0;
            parity ^= 1u;
        }
    }

    // a worker that timed out still owns the loads it issued for tiles
    // k_dead .. issued-1 (one per stage): wait for them, bounded
    if (dead && lane == 0) {
        for (int k = k_dead; k < issued; ++k)
            (void)mbar_wait_bounded(my_bar0 + 8u * (k % S), (uint32_t)((k / S) & 1), kWaitLimitNs / 8);
    }
}

template <int D, bool FP8, int TT>
size_t smem_bytes_for(int stages, int max_batch)
{
    using Gm = Geo<D, FP8, TT>;
    return 1024 + (size_t)kAttnWarps * stages * (Gm::STAGEB + sizeof(StageInfo) + 8) +
           sizeof(int) * (size_t)(max_batch + 1);
}

template <int D, bool FP8, int TT>
cudaError_t prepare_t(int num_sms, int max_batch, AttnLaunch* out)
{
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    const size_t budget = (size_t)optin - 256;   // static shared memory of the kernel
    int stages = kAttnMaxStages;
    while (stages > 2 && smem_bytes_for<D, FP8, TT>(stages, max_batch) > budget) --stages;
    if (smem_bytes_for<D, FP8, TT>(stages, max_batch) > budget) return cudaErrorInvalidConfiguration;
    const size_t bytes = smem_bytes_for<D, FP8, TT>(stages, max_batch);
    // The limit is one setting per kernel for the whole process, shared by
    // every context: set it for the largest batch any context may have, so
    // that creating a context with a smaller batch never lowers it under a
    // context that launches with more (each launch still asks for `bytes`).
    const size_t limit = smem_bytes_for<D, FP8, TT>(stages, kMaxBatch);
    if (limit > budget) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(decode_attn_kernel<D, FP8, kAttnWarps, TT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)limit);
    if (e != cudaSuccess) return e;
    e = combine_prepare(D);
    if (e != cudaSuccess) return e;
    out->ctas = num_sms;
    out->stages = stages;
    out->smem_bytes = bytes;
    out->tile = TT;
    return cudaSuccess;
}

}  // namespace

cudaError_t attn_prepare(int head_dim, bool fp8, int page_size, int num_sms, int max_batch, AttnLaunch* out)
{
    const bool wide = attn_tile(fp8, page_size) == kTileWide;
    if (head_dim == 128) {
        if (!fp8) return prepare_t<128, false, kTile>(num_sms, max_batch, out);
        return wide ? prepare_t<128, true, kTileWide>(num_sms, max_batch, out)
                    : prepare_t<128, true, kTile>(num_sms, max_batch, out);
    }
    if (!fp8) return prepare_t<64, false, kTile>(num_sms, max_batch, out);
    return wide ? prepare_t<64, true, kTileWide>(num_sms, max_batch, out)
                : prepare_t<64, true, kTile>(num_sms, max_batch, out);
}

cudaError_t launch_decode_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                               int head_dim, bool fp8, const AttnLaunch& L, cudaStream_t stream, bool pdl)
{
    const dim3 grid(L.ctas), block(kAttnWarps * 32);
    AttnParams q = p;
    q.stages = L.stages;
    const bool wide = L.tile == kTileWide;
    cudaError_t e;
    if (head_dim == 128) {
        if (!fp8) e = launch_attn_kernel(decode_attn_kernel<128, false, kAttnWarps, kTile>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else if (wide)
            e = launch_attn_kernel(decode_attn_kernel<128, true, kAttnWarps, kTileWide>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else e = launch_attn_kernel(decode_attn_kernel<128, true, kAttnWarps, kTile>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
    } else {
        if (!fp8) e = launch_attn_kernel(decode_attn_kernel<64, false, kAttnWarps, kTile>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else if (wide)
            e = launch_attn_kernel(decode_attn_kernel<64, true, kAttnWarps, kTileWide>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else e = launch_attn_kernel(decode_attn_kernel<64, true, kAttnWarps, kTile>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
    }
    if (e != cudaSuccess) return e;
    q.tile = L.tile;
    q.grid_warps = L.ctas * kAttnWarps;
    const int tail_cap = p.tail_chunks == kTailAuto ? kAutoTailChunks : p.tail_chunks;
    return launch_combine(q, head_dim, (int)max_units(L.ctas * kAttnWarps, tail_cap), L.ctas, stream, true);
}

}  // namespace pkv
