// decode_attn_tokens.cu -- attention of several new tokens per request over
// the paged KV cache: the verification pass of speculative decoding, where a
// draft proposes tokens and the target model checks all of them in one
// forward pass ("Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in
// Production", section "3. Speculative Decoding for Tail Latency";
// "TensorRT-LLM Guide: High-Throughput GPU Inference Engine", section
// "2. Pipelined Speculative Decoding").
//
// What it computes: new token t (0 <= t < q_len) of request b sits at
// position L_b + t and attends tokens 0 .. L_b + t (the cache, the new tokens
// before it and itself), o = softmax(q K^T / sqrt(d)) V, K/V of kv head h / G.
// All q_len x G query rows of a (request, kv head) pair share each K/V tile:
// they are the R = G q_len <= 16 rows of one m16n8k16 mma (row t G + h), so
// the cache is read once per pair whatever q_len is.  Each row has its own
// causal limit (tokens below L_b + t + 1).
//
// The rest is the single-token kernel's design (decode_attn.cu): tiles of 16
// tokens ((request, kv head, tile) flattened and cut into equal contiguous
// warp ranges, a static split), a per-warp ring of TMA tile loads on
// mbarriers fed by a 32-tile page-id lookahead, online softmax in log2 units,
// partial (m, l, o) rows for pairs cut between ranges, merged afterwards by
// the combine kernel (combine.cu).  E4M3 pools as in the single-token kernel:
// codes converted to f16 in registers (K in the byte order of its rows, q
// loaded in the same order; V pairs of tokens permuted per d), the per-(page,
// kv head) scales folded into the scores and into each tile's P V, the mma
// in f16.
//
// Varlen calls (a different number of new tokens per request: chunked
// prefill mixed with decode in one batch, "Scaling TensorRT-LLM: Kernel
// Fusion and Inflight Batching in Production", section "What the Scheduler
// Actually Does"; "TensorRT-LLM Guide", section "1. In-Flight Batching")
// run the same kernel over virtual requests: a plan kernel cuts request b's
// new tokens into blocks of q_len = 16 / G (the last may be shorter), and
// block j becomes a request with L = L_b + j q_len cached tokens (the
// earlier new tokens are already in the pages), its own q / out rows and the
// block table row of b (AttnParams::vmap).
#include "attn_common.cuh"

namespace pkv {
namespace {

using namespace dev;
using namespace attn;

// Query rows of a (request, kv head kvh) pair whose new tokens are q rows
// qrow0, qrow0 + 1, ... as mma A fragments: rows g (a0, a2) and g + 8 (a1,
// a3) of the 16; row r = t G + h is head kvh G + h of new token t, rows
// r >= R are zero.  bf16: a0 = d 16ks+2c..+1, a2 = d 16ks+8+2c..+1.  E4M3
// (f16 operands): the k order inside a k-step follows the byte layout of the
// E4M3 rows, a0 = d 16ks+4c..+1, a2 = d 16ks+4c+2..+3, converted to f16.
template <int D, bool FP8>
__device__ __forceinline__ void load_q_rows(const AttnParams& p, int qrow0, int kvh, int g, int c4, int R,
                                            uint32_t (&qa)[D / 16][4])
{
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int r = g + 8 * half;
        const bool ok = r < R;
        const int t = ok ? r / p.G : 0, h = ok ? r - t * p.G : 0;
        const __nv_bfloat16* qrow = p.q + (((size_t)qrow0 + t) * p.Hq + (size_t)kvh * p.G + h) * D;
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
            if constexpr (!FP8) {
                qa[ks][half] = ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * c4) : 0u;
                qa[ks][2 + half] = ok ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 8 + 2 * c4) : 0u;
            } else {
                const uint2 v = ok ? *reinterpret_cast<const uint2*>(qrow + 16 * ks + 4 * c4) : make_uint2(0u, 0u);
                qa[ks][half] = pack_f16(bf16_lo(v.x), bf16_hi(v.x));
                qa[ks][2 + half] = pack_f16(bf16_lo(v.y), bf16_hi(v.y));
            }
        }
    }
}

// m16n8k16 with f16 A and B (all 16 rows), fp32 accumulation.
__device__ __forceinline__ void mma_f16_16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
        "{%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

template <int D, bool FP8, int WARPS>
__global__ void __launch_bounds__(WARPS * 32, 1)
decode_attn_tokens_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                          const AttnParams p)
{
    using Gm = Geo<D, FP8>;
    constexpr int KSTEPS = D / 16;      // mma k-steps along d for QK^T
    constexpr int NTD = D / 8;          // mma n-tiles along d for P V
    constexpr int NT = WARPS * 32;

    extern __shared__ uint8_t smem_raw[];
    __shared__ int s_warp_tot[WARPS];
    __shared__ int s_bad;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int B = p.vmap ? min(__ldg(p.vcount), p.batch) : p.batch;   // requests, or virtual requests
    const int Hkv = p.Hkv, S = p.stages, QL = p.q_len;
    const int G = p.G, R = G * QL;                   // partial rows per pair
    // (cached tokens before the first new token, new tokens, their first q /
    // out row) of request (or virtual request) v
    auto vinfo = [&](int v, int& L, int& nq, int& qrow0) {
        if (p.vmap) {
            const int4 e = p.vmap[v];
            L = e.w;
            nq = e.z;
            qrow0 = e.y;
        } else {
            L = p.seq_lens[v];
            nq = QL;
            qrow0 = v * QL;
        }
    };

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
    __syncthreads();

    // ---- 1. tiles per request (they cover the last new token's L_b + q_len
    //         tokens) and their exclusive prefix ---------------------------------
    const long long cap = (long long)p.bt_stride * p.P;
    const int per = (B + NT - 1) / NT;
    const int lo = min(B, tid * per), hi = min(B, lo + per);
    int local = 0;
    for (int b = lo; b < hi; ++b) {
        int L, nq, q0;
        vinfo(b, L, nq, q0);
        const bool ok = L >= 0 && (long long)L + nq <= cap;
        const int nt = ok ? (L + nq + kTile - 1) / kTile : 0;
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
    if (B < p.batch) {
        // varlen: the page lookahead searches the prefix over p.batch entries
        // (the plan's capacity); past the last virtual request they hold the
        // total, which no search for a tile below it selects
        const int tot = prefix[B];
        for (int b = B + 1 + tid; b <= p.batch; b += NT) prefix[b] = tot;
        __syncthreads();
    }

    if (s_bad && blockIdx.x == 0) {
        // requests with an impossible length produce zeros and an error bit
        if (tid == 0) atomicOr(p.err, kErrLength);
        for (int b = warp; b < B; b += WARPS) {
            int L, nq, q0;
            vinfo(b, L, nq, q0);
            if (L >= 0 && (long long)L + nq <= cap) continue;
            uint32_t* o32 = reinterpret_cast<uint32_t*>(p.out + (size_t)q0 * p.Hq * D);
            for (int i = lane; i < nq * p.Hq * D / 2; i += 32) o32[i] = 0u;
        }
    }

    // ---- 2. static split: this warp's range --------------------------------------
    const long long T = (long long)prefix[B] * Hkv;
    long long Wl = (long long)gridDim.x * WARPS;
    if (p.workers > 0) Wl = min(Wl, (long long)p.workers);
    else Wl = min(Wl, (T + kMinTilesPerWorker - 1) / kMinTilesPerWorker);
    Wl = max(1LL, min(Wl, max(T, 1LL)));
    const int W = (int)Wl;
    const Split sp = make_split(max(T, 1LL), W, 0);
    if (blockIdx.x == 0) {
        // the combine kernel that follows needs the same split geometry
        if (tid == 0) {
            p.meta[0] = W;
            p.meta[1] = (int)(T & 0xFFFFFFFFll);
            p.meta[2] = (int)(T >> 32);
            p.meta[3] = 0;
        }
        for (int b = tid; b <= B; b += NT) p.meta[4 + b] = prefix[b];
    }
    if (T == 0) return;
    const int w = warp * gridDim.x + blockIdx.x;   // spread workers over SMs first
    if (w >= W) return;
    const long long u0 = sp.ustart(w), u1 = sp.ustart(w + 1);
    const int ntiles = (int)(u1 - u0);

    const uint32_t my_stage0 = stage_area + (uint32_t)(warp * S * Gm::STAGEB);
    StageInfo* const my_info = info_all + warp * S;
    const uint32_t my_bar0 = smem_u32(bar_ptr) + (uint32_t)(warp * S * 8);
    if (lane == 0) {
        for (int s = 0; s < S; ++s) mbar_init(my_bar0 + 8u * s, 1u);
        fence_mbar_init();
    }
    __syncwarp();

    // ---- 3. producer: double-buffered 32-tile lookahead, TMA issue -----------------
    int la_i = 0;
    long long la_fill = u0 + 64;
    Lookahead la_cur = lookahead_fill<FP8>(p, prefix, u0, u1, lane);
    Lookahead la_nxt = lookahead_fill<FP8>(p, prefix, u0 + 32, u1, lane);

    auto issue = [&](int s) {
        if (la_i == 32) {
            la_i = 0;
            la_cur = la_nxt;
            la_nxt = lookahead_fill<FP8>(p, prefix, la_fill, u1, lane);
            la_fill += 32;
        }
        const int src = la_i++;
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
    };

    // q and the slots the RoPE + append kernel writes are read only after it
    // has finished (a no-op unless launched as its programmatic dependent)
    grid_dependency_wait();
    const int pre = min(S, ntiles);
    for (int k = 0; k < pre; ++k) issue(k);
    int issued = pre;

    // ---- 4. consumer ----------------------------------------------------------------
    const int g = lane >> 2;     // mma rows g and g + 8
    const int c4 = lane & 3;
    const int mi = lane >> 3, ri = lane & 7;        // ldmatrix: matrix index, row
    const int tokK = ((mi >> 1) << 3) + ri;         // token row addressed for K
    const int tokV = ((mi & 1) << 3) + ri;          // token row addressed for V (trans)
    // the current pair: its first q / out row, its rows (G x its new tokens)
    int cur_q0 = 0, Rv = R;

    float o[NTD][4];
    uint32_t qa[KSTEPS][4];
    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    int lim[2] = {0, 0};          // tokens visible to rows g and g + 8
    int n_max = 0;                // tokens of the pair's last new token
    bool dead = false;
    int k_dead = 0;
    int s = 0;
    uint32_t parity = 0;

    int cb, ckvh, ctt, cnt;
    locate(prefix, B, Hkv, u0, cb, ckvh, ctt, cnt);

    for (int k = 0; k < ntiles; ++k) {
        if (!dead) {
            const bool ok = __all_sync(kFull, mbar_wait_bounded(my_bar0 + 8u * s, parity, kWaitLimitNs));
            if (!ok) {
                dead = true;
                k_dead = k;
                if (lane == 0) atomicOr(p.err, kErrTimeout);
            }
        }
        if (dead) {
            if (++s == S) {
                s = 0;
                parity ^= 1u;
            }
            continue;
        }
        if (ctt == 0 || k == 0) {
            // start of a (request, kv head) pair or of this range
            int L, nq;
            vinfo(cb, L, nq, cur_q0);
            Rv = G * nq;
            load_q_rows<D, FP8>(p, cur_q0, ckvh, g, c4, Rv, qa);
            const int n0 = L + 1;                // tokens visible to new token 0
            // new token of rows g and g + 8 (rows >= Rv see no token)
            lim[0] = g < Rv ? n0 + g / G : 0;
            lim[1] = g + 8 < Rv ? n0 + (g + 8) / G : 0;
            n_max = n0 + nq - 1;
#pragma unroll
            for (int nt = 0; nt < NTD; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;
            m_run[0] = m_run[1] = -INFINITY;
            l_run[0] = l_run[1] = 0.f;
        }
        const bool pair_end = ctt == cnt - 1 || k == ntiles - 1;

        const StageInfo si = my_info[s];
        bool zeroed = false;
        if (si.valid) {
            const uint32_t kb = my_stage0 + (uint32_t)(s * Gm::STAGEB);
            const uint32_t vb = kb + Gm::TILEB;
            const int tok0 = ctt * kTile;
            const int rows_valid = min(kTile, n_max - tok0);
            if (rows_valid < kTile) {
                // slots past the last new token may hold anything (NaN): zero them in V
                constexpr int CPR = Gm::ROWB / 16;
                const int nch = (kTile - rows_valid) * CPR;
                for (int e = lane; e < nch; e += 32) {
                    const int r = rows_valid + e / CPR, ch = e % CPR;
                    asm volatile("st.shared.v4.u32 [%0], {%1, %1, %1, %1};" ::"r"(vb + tile_off<D, FP8>(r, ch)),
                                 "r"(0u)
                                 : "memory");
                }
                zeroed = true;
                __syncwarp();
            }

            // S = Q K^T: two n-tiles of 8 tokens, rows g (e 0, 1) and g + 8 (e 2, 3), two chains
            float sa[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            float sb[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
            if constexpr (!FP8) {
#pragma unroll
                for (int ks = 0; ks < KSTEPS; ks += 2) {
                    uint32_t r0, r1, r2, r3, r4, r5, r6, r7;
                    ldsm_x4(kb + tile_off<D, FP8>(tokK, 2 * ks + (mi & 1)), r0, r1, r2, r3);
                    ldsm_x4(kb + tile_off<D, FP8>(tokK, 2 * ks + 2 + (mi & 1)), r4, r5, r6, r7);
                    mma_bf16_16(sa[0], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r0, r1);
                    mma_bf16_16(sa[1], qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3], r2, r3);
                    mma_bf16_16(sb[0], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], r4, r5);
                    mma_bf16_16(sb[1], qa[ks + 1][0], qa[ks + 1][1], qa[ks + 1][2], qa[ks + 1][3], r6, r7);
                }
            } else {
                // one 16-byte chunk of an E4M3 row = one k-step: r0 / r1 tokens 0-7,
                // chunks 2s4 / 2s4+1; r2 / r3 tokens 8-15
#pragma unroll
                for (int s4 = 0; s4 < D / 32; ++s4) {
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4(kb + tile_off<D, FP8>(tokK, 2 * s4 + (mi & 1)), r0, r1, r2, r3);
                    mma_f16_16(sa[0], qa[2 * s4][0], qa[2 * s4][1], qa[2 * s4][2], qa[2 * s4][3], cvt_lo(r0),
                               cvt_hi(r0));
                    mma_f16_16(sb[0], qa[2 * s4 + 1][0], qa[2 * s4 + 1][1], qa[2 * s4 + 1][2], qa[2 * s4 + 1][3],
                               cvt_lo(r1), cvt_hi(r1));
                    mma_f16_16(sa[1], qa[2 * s4][0], qa[2 * s4][1], qa[2 * s4][2], qa[2 * s4][3], cvt_lo(r2),
                               cvt_hi(r2));
                    mma_f16_16(sb[1], qa[2 * s4 + 1][0], qa[2 * s4 + 1][1], qa[2 * s4 + 1][2], qa[2 * s4 + 1][3],
                               cvt_lo(r3), cvt_hi(r3));
                }
            }

            // online softmax per row in log2 units; tokens at or past a row's
            // limit are -inf (never 0 * NaN)
            const float slog2 = FP8 ? p.scale_log2 * si.ks : p.scale_log2;
            float sc[2][4];
            float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
            for (int j = 0; j < 2; ++j)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tok = tok0 + 8 * j + 2 * c4 + (e & 1);
                    sc[j][e] = (tok < lim[e >> 1]) ? (sa[j][e] + sb[j][e]) * slog2 : -INFINITY;
                    mx[e >> 1] = fmaxf(mx[e >> 1], sc[j][e]);
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
            // P as the A operand: a0 row g tokens 2c4.., a1 row g+8, a2/a3 tokens 8+2c4..
            // (bf16, or f16 for E4M3 pools), l summed from the rounded values
            uint32_t pa0, pa1, pa2, pa3;
            if constexpr (!FP8) {
                pa0 = pack_bf16(ex2(sc[0][0] - m_ref[0]), ex2(sc[0][1] - m_ref[0]));
                pa1 = pack_bf16(ex2(sc[0][2] - m_ref[1]), ex2(sc[0][3] - m_ref[1]));
                pa2 = pack_bf16(ex2(sc[1][0] - m_ref[0]), ex2(sc[1][1] - m_ref[0]));
                pa3 = pack_bf16(ex2(sc[1][2] - m_ref[1]), ex2(sc[1][3] - m_ref[1]));
                l_run[0] = l_run[0] * alpha[0] + ((bf16_lo(pa0) + bf16_hi(pa0)) + (bf16_lo(pa2) + bf16_hi(pa2)));
                l_run[1] = l_run[1] * alpha[1] + ((bf16_lo(pa1) + bf16_hi(pa1)) + (bf16_lo(pa3) + bf16_hi(pa3)));
            } else {
                pa0 = pack_f16(ex2(sc[0][0] - m_ref[0]), ex2(sc[0][1] - m_ref[0]));
                pa1 = pack_f16(ex2(sc[0][2] - m_ref[1]), ex2(sc[0][3] - m_ref[1]));
                pa2 = pack_f16(ex2(sc[1][0] - m_ref[0]), ex2(sc[1][1] - m_ref[0]));
                pa3 = pack_f16(ex2(sc[1][2] - m_ref[1]), ex2(sc[1][3] - m_ref[1]));
                const float2 f0 = f16x2_to_f32(pa0), f1 = f16x2_to_f32(pa1), f2 = f16x2_to_f32(pa2),
                             f3 = f16x2_to_f32(pa3);
                l_run[0] = l_run[0] * alpha[0] + ((f0.x + f0.y) + (f2.x + f2.y));
                l_run[1] = l_run[1] * alpha[1] + ((f1.x + f1.y) + (f3.x + f3.y));
            }
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
            if constexpr (!FP8) {
#pragma unroll
                for (int dj = 0; dj < D / 16; ++dj) {
                    uint32_t r0, r1, r2, r3;
                    ldsm_x4_trans(vb + tile_off<D, FP8>(tokV, 2 * dj + (mi >> 1)), r0, r1, r2, r3);
                    mma_bf16_16(o[2 * dj], pa0, pa1, pa2, pa3, r0, r1);
                    mma_bf16_16(o[2 * dj + 1], pa0, pa1, pa2, pa3, r2, r3);
                }
            } else {
                // E4M3 V: lane (n = g, c4) loads d in [DV*n, DV*n + DV) of tokens
                // 2c4, 2c4+1, 8+2c4, 9+2c4; byte permutes pair tokens per d, and the
                // mma n-index j of n-tile nt stands for d = DV*j + nt
                constexpr int DV = D / 8;
                constexpr int WORDS = DV / 4;
                uint32_t wa[WORDS], wb[WORDS], wc[WORDS], wd[WORDS];
                const int t0 = 2 * c4;
                if constexpr (DV == 16) {
                    const uint4 a = lds128(vb + tile_off<D, FP8>(t0, g));
                    const uint4 b = lds128(vb + tile_off<D, FP8>(t0 + 1, g));
                    const uint4 cc = lds128(vb + tile_off<D, FP8>(t0 + 8, g));
                    const uint4 dd = lds128(vb + tile_off<D, FP8>(t0 + 9, g));
                    wa[0] = a.x; wa[1] = a.y; wa[2] = a.z; wa[3] = a.w;
                    wb[0] = b.x; wb[1] = b.y; wb[2] = b.z; wb[3] = b.w;
                    wc[0] = cc.x; wc[1] = cc.y; wc[2] = cc.z; wc[3] = cc.w;
                    wd[0] = dd.x; wd[1] = dd.y; wd[2] = dd.z; wd[3] = dd.w;
                } else {
                    const uint32_t off8 = (uint32_t)((g & 1) * 8);
                    const uint2 a = lds64(vb + tile_off<D, FP8>(t0, g >> 1) + off8);
                    const uint2 b = lds64(vb + tile_off<D, FP8>(t0 + 1, g >> 1) + off8);
                    const uint2 cc = lds64(vb + tile_off<D, FP8>(t0 + 8, g >> 1) + off8);
                    const uint2 dd = lds64(vb + tile_off<D, FP8>(t0 + 9, g >> 1) + off8);
                    wa[0] = a.x; wa[1] = a.y;
                    wb[0] = b.x; wb[1] = b.y;
                    wc[0] = cc.x; wc[1] = cc.y;
                    wd[0] = dd.x; wd[1] = dd.y;
                }
                const float vs = si.vs;
#pragma unroll
                for (int kw = 0; kw < WORDS; ++kw) {
                    const uint32_t x0 = __byte_perm(wa[kw], wb[kw], 0x5140);
                    const uint32_t x1 = __byte_perm(wa[kw], wb[kw], 0x7362);
                    const uint32_t y0 = __byte_perm(wc[kw], wd[kw], 0x5140);
                    const uint32_t y1 = __byte_perm(wc[kw], wd[kw], 0x7362);
                    float t[4][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f},
                                     {0.f, 0.f, 0.f, 0.f}};
                    mma_f16_16(t[0], pa0, pa1, pa2, pa3, cvt_lo(x0), cvt_lo(y0));
                    mma_f16_16(t[1], pa0, pa1, pa2, pa3, cvt_hi(x0), cvt_hi(y0));
                    mma_f16_16(t[2], pa0, pa1, pa2, pa3, cvt_lo(x1), cvt_lo(y1));
                    mma_f16_16(t[3], pa0, pa1, pa2, pa3, cvt_hi(x1), cvt_hi(y1));
#pragma unroll
                    for (int e = 0; e < 4; ++e)
#pragma unroll
                        for (int u = 0; u < 4; ++u) o[4 * kw + e][u] = fmaf(t[e][u], vs, o[4 * kw + e][u]);
                }
            }
        }
        __syncwarp();

        // refill this stage with the tile `S` ahead; generic-proxy zero stores
        // above must land before the async-proxy copy that overwrites the buffer
        if (issued < ntiles) {
            if (zeroed && lane == 0) fence_proxy_async_smem();
            issue(s);
            ++issued;
        }

        // ---- end of a pair (or of this range): write out or leave a partial -------
        if (pair_end) {
            float lsum[2];
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                lsum[hf] = l_run[hf] + __shfl_xor_sync(kFull, l_run[hf], 1);
                lsum[hf] += __shfl_xor_sync(kFull, lsum[hf], 2);
            }
            const long long ts = (long long)prefix[cb] * Hkv + (long long)ckvh * cnt;
            const long long te = ts + cnt;
            const bool whole = u0 <= ts && te <= u1;
            const int slot = 2 * w + (u0 < ts ? 1 : 0);
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int r = g + 8 * hf;
                if (r >= Rv) continue;
                if (whole) {
                    const int t = r / G, h = r - t * G;
                    const float inv = 1.f / lsum[hf];
                    uint32_t* dst = reinterpret_cast<uint32_t*>(
                        p.out + (((size_t)cur_q0 + t) * p.Hq + (size_t)ckvh * G + h) * D);
                    if constexpr (!FP8) {
#pragma unroll
                        for (int nt = 0; nt < NTD; ++nt)
                            dst[(8 * nt + 2 * c4) >> 1] = pack_bf16(o[nt][2 * hf] * inv, o[nt][2 * hf + 1] * inv);
                    } else {
                        // n-tile nt, column j = 2c4 + e holds d = DV j + nt
                        constexpr int DV = D / 8;
#pragma unroll
                        for (int e = 0; e < 2; ++e)
#pragma unroll
                            for (int u = 0; u < DV / 2; ++u)
                                dst[(DV * (2 * c4 + e) + 2 * u) >> 1] =
                                    pack_bf16(o[2 * u][2 * hf + e] * inv, o[2 * u + 1][2 * hf + e] * inv);
                    }
                } else {
                    float* dst = p.part_o + ((size_t)slot * R + r) * D;
                    if constexpr (!FP8) {
#pragma unroll
                        for (int nt = 0; nt < NTD; ++nt)
                            *reinterpret_cast<float2*>(dst + 8 * nt + 2 * c4) =
                                make_float2(o[nt][2 * hf], o[nt][2 * hf + 1]);
                    } else {
                        constexpr int DV = D / 8;
#pragma unroll
                        for (int e = 0; e < 2; ++e)
#pragma unroll
                            for (int u = 0; u < DV / 2; ++u)
                                *reinterpret_cast<float2*>(dst + DV * (2 * c4 + e) + 2 * u) =
                                    make_float2(o[2 * u][2 * hf + e], o[2 * u + 1][2 * hf + e]);
                    }
                    if (c4 == 0)
                        *reinterpret_cast<float2*>(p.part_ml + ((size_t)slot * R + r) * 2) =
                            make_float2(m_run[hf], lsum[hf]);
                }
            }
        }

        // advance the consumer cursor and the ring position
        if (++ctt == cnt) {
            ctt = 0;
            if (++ckvh == Hkv) {
                ckvh = 0;
                do { ++cb; } while (cb < B && prefix[cb + 1] == prefix[cb]);
            }
            if (cb < B) cnt = prefix[cb + 1] - prefix[cb];
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

template <int D, bool FP8>
size_t tokens_smem_bytes(int stages, int max_batch)
{
    using Gm = Geo<D, FP8>;
    return 1024 + (size_t)kAttnWarps * stages * (Gm::STAGEB + sizeof(StageInfo) + 8) +
           sizeof(int) * (size_t)(max_batch + 1);
}

template <int D, bool FP8>
cudaError_t prepare_tokens_t(int num_sms, int max_batch, AttnLaunch* out)
{
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    const int stages = kAttnMaxStages;
    const size_t bytes = tokens_smem_bytes<D, FP8>(stages, max_batch);
    // one process-wide limit per kernel: set for the largest batch any
    // context may have (see decode_attn.cu), never lowered by a smaller one
    const size_t limit = tokens_smem_bytes<D, FP8>(stages, kMaxBatch);
    if (bytes > limit || limit > (size_t)optin - 256) return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(decode_attn_tokens_kernel<D, FP8, kAttnWarps>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)limit);
    if (e != cudaSuccess) return e;
    e = combine_prepare(D);
    if (e != cudaSuccess) return e;
    out->ctas = num_sms;
    out->stages = stages;
    out->smem_bytes = bytes;
    out->tile = kTile;
    return cudaSuccess;
}

}  // namespace

namespace {

// One CTA: request b's new tokens (cu_q[b + 1] - cu_q[b] of them) cut into
// blocks of `block`; vmap[v] = {b, first q row, tokens, L_b + offset of the
// block}, v counted in request order (an exclusive scan of the blocks per
// request).  With cmin > 0, a request of at least cmin new tokens is cut
// instead into blocks of cblock tokens listed the same way in cmap (the
// prefill-chunk kernel's work).  More blocks than a map holds, or a negative
// token count, set kErrLength (the surplus is dropped).
__global__ void __launch_bounds__(1024) varlen_plan_kernel(const int32_t* __restrict__ cu_q,
                                                           const int32_t* __restrict__ seq_lens, int batch,
                                                           int block, int vmax, int4* __restrict__ vmap,
                                                           int* __restrict__ vcount, int cmin, int cblock, int cmax,
                                                           int4* __restrict__ cmap, int* __restrict__ ccount,
                                                           int* __restrict__ err)
{
    __shared__ int s_warp[2][32];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, nwarps = blockDim.x >> 5;
    const int per = (batch + (int)blockDim.x - 1) / (int)blockDim.x;
    const int lo = min(batch, tid * per), hi = min(batch, lo + per);
    auto chunked = [&](int q) { return cmin > 0 && q >= cmin; };
    int lv = 0, lc = 0;   // this thread's virtual and chunk blocks
    for (int b = lo; b < hi; ++b) {
        const int q = cu_q[b + 1] - cu_q[b];
        if (q <= 0) continue;
        if (chunked(q)) lc += (q + cblock - 1) / cblock;
        else lv += (q + block - 1) / block;
    }
    int iv = lv, ic = lc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(kFull, iv, o), c = __shfl_up_sync(kFull, ic, o);
        if (lane >= o) {
            iv += v;
            ic += c;
        }
    }
    if (lane == 31) {
        s_warp[0][warp] = iv;
        s_warp[1][warp] = ic;
    }
    __syncthreads();
    int rv = iv - lv, rc = ic - lc;
    for (int w2 = 0; w2 < warp; ++w2) {
        rv += s_warp[0][w2];
        rc += s_warp[1][w2];
    }
    for (int b = lo; b < hi; ++b) {
        const int a = cu_q[b], q = cu_q[b + 1] - a;
        if (q < 0) {
            atomicOr(err, kErrLength);
            continue;
        }
        const long long L = seq_lens[b];
        const bool ch = chunked(q);
        const int blk = ch ? cblock : block;
        for (int j = 0; (long long)j * blk < q; ++j) {
            const long long pos = L + (long long)j * blk;
            const int4 e = make_int4(b, a + j * blk, min(blk, q - j * blk), (L < 0 || pos > 0x7fffffffll) ? -1 : (int)pos);
            if (ch) {
                if (rc < cmax) cmap[rc] = e;
                ++rc;
            } else {
                if (rv < vmax) vmap[rv] = e;
                ++rv;
            }
        }
    }
    if (tid == 0) {
        int tv = 0, tc = 0;
        for (int w2 = 0; w2 < nwarps; ++w2) {
            tv += s_warp[0][w2];
            tc += s_warp[1][w2];
        }
        if (tv > vmax || tc > cmax) atomicOr(err, kErrLength);
        *vcount = min(tv, vmax);
        if (ccount) *ccount = min(tc, cmax);
    }
}

}  // namespace

cudaError_t launch_varlen_plan(const int32_t* cu_q, const int32_t* seq_lens, int batch, int block, int vmax,
                               int4* vmap, int* vcount, int cmin, int cblock, int cmax, int4* cmap, int* ccount,
                               int* err, cudaStream_t stream)
{
    varlen_plan_kernel<<<1, 1024, 0, stream>>>(cu_q, seq_lens, batch, block, vmax, vmap, vcount,
                                               cmap ? cmin : 0, cblock > 0 ? cblock : 1, cmax, cmap, ccount, err);
    return cudaGetLastError();
}

cudaError_t attn_tokens_prepare(int head_dim, bool fp8, int num_sms, int max_batch, AttnLaunch* out)
{
    if (head_dim == 128)
        return fp8 ? prepare_tokens_t<128, true>(num_sms, max_batch, out)
                   : prepare_tokens_t<128, false>(num_sms, max_batch, out);
    return fp8 ? prepare_tokens_t<64, true>(num_sms, max_batch, out) : prepare_tokens_t<64, false>(num_sms, max_batch, out);
}

cudaError_t launch_decode_attn_tokens(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv,
                                      int head_dim, bool fp8, const AttnLaunch& L, cudaStream_t stream, bool pdl)
{
    const dim3 grid(L.ctas), block(kAttnWarps * 32);
    AttnParams q = p;
    q.stages = L.stages;
    q.tail_chunks = 0;
    cudaError_t e;
    if (head_dim == 128) {
        if (fp8) e = launch_attn_kernel(decode_attn_tokens_kernel<128, true, kAttnWarps>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else e = launch_attn_kernel(decode_attn_tokens_kernel<128, false, kAttnWarps>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
    } else {
        if (fp8) e = launch_attn_kernel(decode_attn_tokens_kernel<64, true, kAttnWarps>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
        else e = launch_attn_kernel(decode_attn_tokens_kernel<64, false, kAttnWarps>, grid, block, L.smem_bytes, stream, pdl, tmk, tmv, q);
    }
    if (e != cudaSuccess) return e;
    return launch_combine(q, head_dim, L.ctas * kAttnWarps, L.ctas, stream);
}

}  // namespace pkv
