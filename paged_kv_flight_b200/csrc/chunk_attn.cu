// chunk_attn.cu -- attention of the prefill chunks of a varlen call on the
// Blackwell tensor cores: Q, S, P and O in tensor memory (tcgen05), K / V
// pages by TMA into shared memory.
//
// "Scaling TensorRT-LLM: Kernel Fusion and Inflight Batching in Production",
// section "What the Scheduler Actually Does" (chunked prefill mixed with
// decode in one batch) and section "The Paged KV-Cache" (pages named by a
// per-request block table).  What it computes is the varlen attention's: new
// token t of a request attends keys 0 .. pos_t of the request's cache, pos_t
// its own position (the cache already holds the earlier new tokens and the
// token itself), softmax(q K^T / sqrt(d)) V.
//
// Work item: a block of up to 128 / G new tokens of one request and one kv
// head.  Its 128 query rows r = t G + g (token t of the block, head g of the
// group) are the M = 128 rows of both MMAs, so the block reads its request's
// cache once for all of them.  Q, S, P and O live in tensor memory; shared
// memory holds only a ring of K / V tiles (three stages of 128 keys, as TMA
// lands them with the 128-byte swizzle).  Per tile j:
//   S_j = Q K^T     tcgen05, A = Q from TMEM, B = K (K-major); M 128, N 128
//                   keys, K d; fp32 into TMEM buffer j % 2
//   softmax         eight warps, two per TMEM lane quarter, one per half of the
//                   keys: max of the row over both halves, P = 2^(s - m) in
//                   log2 units as two bf16 terms P_hi + P_lo (about 16
//                   significant bits, so the weights of a row with few keys
//                   carry no bf16-sized error), written over the warp's own S
//                   columns; each half keeps its own running sum (same max)
//   O += P V        tcgen05, A = P from TMEM, B = V (MN-major); M 128, N d,
//                   K 2 x 128: P_hi V then P_lo V over the same V tile; O
//                   stays in TMEM over all tiles
// The reference max m of a row moves only when the row's max passes it by
// more than 2^8 (P <= 2^8 meanwhile); then O and l are rescaled in place.
// With S / P in two buffers and no per-tile fold of O, the softmax of tile
// j + 1 runs while P V of tile j is on the tensor pipe.  Roles:
// warp 0 lane 0 issues the K / V page loads, warp 1 lane 0 the MMAs (S and P
// V each as soon as its inputs are ready), warps 2 .. 9 the softmax and the
// output rows.  Every wait is bounded.
#include "pkv_internal.h"
#include "pkv_device.cuh"
#include "umma.cuh"

namespace pkv {
namespace {

using namespace dev;

constexpr int kCStages = 3;
constexpr int kCSoftWarps = 8;
constexpr int kCThreads = 64 + 32 * kCSoftWarps;
// tensor memory: S / P buffers (2 x 128 columns), O (d), Q (d / 2: two bf16
// per column)
constexpr uint32_t kCCols = 512;
constexpr uint32_t kCOcol = 2 * kChunkKeys;
constexpr uint32_t kCQcol = kCOcol + 128;
constexpr int kCBlk = kChunkRows * 128;       // one 64-element column block of a 128-row tile: 16 KB
constexpr uint64_t kCWaitNs = 500ull * 1000ull * 1000ull;
static_assert(kChunkRows == 128 && kChunkKeys == 128, "the MMA shapes below");

// Shared memory (dynamic, 1024-byte aligned): the ring, per stage K and V,
// [d / 64 blocks][128 keys][128 B] each.
template <int D>
struct ChunkGeo {
    static constexpr int KB = D / 64;
    static constexpr int STB = 2 * KB * kCBlk;
    static constexpr int BYTES = kCStages * STB;
};

__device__ __forceinline__ void sts128(uint32_t addr, uint4 v)
{
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

template <int D>
__global__ void __launch_bounds__(kCThreads, 1)
chunk_attn_kernel(const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv,
                  const AttnParams p)
{
    using Gm = ChunkGeo<D>;
    constexpr int KB = Gm::KB, HD = D / 2;
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t s_full[kCStages], s_empty[kCStages], s_sfull[2], s_pfull, s_ofull, s_ofin, s_drain;
    __shared__ uint32_t s_tmem;
    __shared__ int s_bad, s_fail;
    __shared__ int s_issued, s_landed;         // tiles whose copies went out / were consumed by the MMA
    __shared__ float s_mx[2][2][kChunkRows];   // [tile parity][half of the keys][row] partial maxima
    __shared__ float s_l[2][kChunkRows];       // [half][row] running sums

    const int item = blockIdx.y;
    // the host sizes the grid from the call's token counts; a plan with more
    // blocks than that would leave rows unwritten, so it is reported
    if (blockIdx.x == 0 && item == 0 && threadIdx.x == 0 && __ldg(p.ccount) > (int)gridDim.y)
        atomicOr(p.err, kErrLength);
    if (item >= __ldg(p.ccount)) return;       // CTA-uniform, before any barrier
    const int kvh = blockIdx.x, G = p.G;
    const int4 e = p.cmap[item];
    const int b = e.x, qrow0 = e.y, ntok = e.z, posb = e.w;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const long long n_keys_ll = (long long)posb + ntok;   // keys of the block's last token
    auto out_row = [&](int t, int g) { return p.out + ((size_t)(qrow0 + t) * p.Hq + (size_t)kvh * G + g) * D; };
    if (posb < 0 || ntok <= 0 || n_keys_ll > (long long)p.bt_stride * p.P) {
        // past the block table: the block's rows are zero, the error word says why
        if (tid == 0 && kvh == 0) atomicOr(p.err, kErrLength);
        for (int i = tid; i < ntok * G * (D / 8); i += kCThreads) {
            const int rr = i / (D / 8), c = i - rr * (D / 8);
            reinterpret_cast<uint4*>(out_row(rr / G, rr % G))[c] = make_uint4(0u, 0u, 0u, 0u);
        }
        return;
    }
    const int n_keys = (int)n_keys_ll;
    const int NT = (n_keys + kChunkKeys - 1) / kChunkKeys;
    const int PPT = kChunkKeys / p.P;          // pages per tile

    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t st0 = (raw + 1023u) & ~1023u;
    const uint32_t full0 = smem_u32(&s_full[0]), empty0 = smem_u32(&s_empty[0]);
    const uint32_t sfull0 = smem_u32(&s_sfull[0]), pfull = smem_u32(&s_pfull), ofull = smem_u32(&s_ofull);
    const int32_t* bt = p.block_tables + (size_t)b * p.bt_stride;

    // tile j's pages into stage j % 3: only the pages holding keys < n_keys
    // (the rows past them are never attended; their V rows are zeroed below)
    auto load_tile = [&](int j) {
        const int s = j % kCStages;
        const int keys = min(kChunkKeys, n_keys - j * kChunkKeys);
        const int np = (keys + p.P - 1) / p.P;
        const uint32_t kd = st0 + (uint32_t)(s * Gm::STB), vd = kd + (uint32_t)(KB * kCBlk);
        mbar_arrive_expect_tx(full0 + 8u * s, (uint32_t)(np * p.P * 128 * KB * 2));
        for (int i = 0; i < np; ++i) {
            int page = __ldg(&bt[j * PPT + i]);
            if (page < 0 || page >= p.num_pages) {
                s_bad = 1;
                page = 0;   // an in-range page keeps the copy legal; the rows are zeroed at the end
            }
            const int y = (page * p.Hkv + kvh) * p.P;
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_2d(kd + (uint32_t)(kb * kCBlk + i * p.P * 128), &tmk, 64 * kb, y, full0 + 8u * s);
                tma_load_2d(vd + (uint32_t)(kb * kCBlk + i * p.P * 128), &tmv, 64 * kb, y, full0 + 8u * s);
            }
        }
    };

    if (tid == 0) {
        s_bad = 0;
        s_fail = 0;
        prefetch_tensormap(&tmk);
        prefetch_tensormap(&tmv);
        for (int s = 0; s < kCStages; ++s) {
            mbar_init(full0 + 8u * s, 1u);
            mbar_init(empty0 + 8u * s, 1u);
        }
        mbar_init(sfull0, 1u);
        mbar_init(sfull0 + 8u, 1u);
        mbar_init(pfull, (uint32_t)kCSoftWarps);
        mbar_init(ofull, 1u);
        mbar_init(smem_u32(&s_ofin), 1u);
        mbar_init(smem_u32(&s_drain), 1u);
        fence_mbar_init();
        s_issued = min(kCStages, NT);
        s_landed = 0;
        for (int j = 0; j < kCStages && j < NT; ++j) load_tile(j);
    }
    if (warp == 0) {
        __syncwarp();   // converged for the aligned allocation
        tmem_alloc(smem_u32(&s_tmem), kCCols);
    }
    __syncthreads();   // the allocation's address
    const uint32_t tmem = s_tmem;
    // the softmax warps: row r = 32 (warp % 4) + lane (its TMEM lane), keys
    // and d columns of half h.  First their halves of the Q rows go into
    // tensor memory: d 0 .. D-1 of row r at columns kCQcol + d / 2
    const int sw = warp - 2, quarter = warp & 3, h = sw >> 2;
    const int r = 32 * quarter + lane, t = r / G, g = r - t * G;
    const bool row_ok = t < ntok;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);
    if (warp >= 2) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q + ((size_t)(qrow0 + (row_ok ? t : 0)) * p.Hq +
                                                                 (size_t)kvh * G + g) * D + h * HD);
#pragma unroll
        for (int c0 = 0; c0 < HD / 2; c0 += 16) {   // 16 columns = 32 bf16 = four 16-byte loads
            uint32_t w[16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 v = row_ok ? __ldg(src + c0 / 4 + i) : make_uint4(0u, 0u, 0u, 0u);
                w[4 * i] = v.x;
                w[4 * i + 1] = v.y;
                w[4 * i + 2] = v.z;
                w[4 * i + 3] = v.w;
            }
            tmem_st16(lane_base + kCQcol + (uint32_t)(h * (HD / 2) + c0), w);
        }
        tmem_wait_st();
    }
    tmem_fence_before();
    __syncthreads();   // Q in tensor memory
    tmem_fence_after();

    if (warp == 0) {
        // ---- producer: the rest of the tiles, each once its stage is free
        if (lane == 0) {
            for (int j = kCStages; j < NT; ++j) {
                const int s = j % kCStages;
                if (!mbar_wait_bounded(empty0 + 8u * s, (uint32_t)((j / kCStages - 1) & 1), kCWaitNs)) {
                    s_fail = 1;
                    break;
                }
                load_tile(j);
                s_issued = j + 1;
            }
        }
    } else if (warp == 1) {
        // ---- MMA issue, one thread: S_js once its tile has landed (and its
        // buffer's P V went out: the pipe runs the MMAs in issue order), P V
        // of tile jp once its P is written; whichever is ready first
        if (lane == 0) {
            constexpr uint32_t idS = umma_idesc_bf16<kChunkRows, kChunkKeys>();
            constexpr uint32_t idO = umma_idesc_bf16<kChunkRows, D, true>();
            int js = 0, jp = 0;
            bool ok = true;
            uint64_t t_prog = global_timer_ns();   // the last progress
            for (uint32_t it = 0; jp < NT; ++it) {
                bool moved = false;
                if (js < NT && js <= jp + 1 &&
                    mbar_try_wait(full0 + 8u * (js % kCStages), (uint32_t)((js / kCStages) & 1))) {
                    s_landed = js + 1;
                    tmem_fence_after();
                    const uint32_t kd = st0 + (uint32_t)((js % kCStages) * Gm::STB);
                    const uint32_t dS = tmem + (uint32_t)((js & 1) * kChunkKeys);
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk)   // K steps of 16 along d: 8 Q columns each
                        umma_bf16_ts(dS, tmem + kCQcol + (uint32_t)(8 * kk),
                                     sw128_kmajor_desc(kd + (uint32_t)((kk >> 2) * kCBlk + (kk & 3) * 32)), idS,
                                     kk ? 1u : 0u);
                    umma_commit(sfull0 + 8u * (js & 1));
                    ++js;
                    moved = true;
                }
                if (jp < js && mbar_try_wait(pfull, (uint32_t)(jp & 1))) {
                    tmem_fence_after();
                    const int s = jp % kCStages;
                    const uint32_t vd = st0 + (uint32_t)(s * Gm::STB + KB * kCBlk);
                    const uint32_t pcol = tmem + (uint32_t)((jp & 1) * kChunkKeys);
#pragma unroll
                    for (int kk = 0; kk < 2 * kChunkKeys / 16; ++kk) {   // K steps of 16 keys: P_hi, then P_lo
                        const int k8 = kk & 7;
                        // P of keys 16 k8 .. + 15: half k8 / 4 of the buffer
                        // (64 columns), its quarter (k8 / 2) & 1 (32 columns:
                        // P_hi of 32 keys in 16, then P_lo in 16), 8 columns
                        // per step
                        const uint32_t acol =
                            (uint32_t)((k8 >> 2) * 64 + ((k8 >> 1) & 1) * 32 + (k8 & 1) * 8 + (kk >> 3) * 16);
                        // V: d along N in 64-element blocks kCBlk apart, keys
                        // along K, 8 key rows (1024 B) per swizzle atom
                        umma_bf16_ts(tmem + kCOcol, pcol + acol,
                                     sw128_mnmajor_desc(vd + (uint32_t)(k8 * 2048), (uint32_t)kCBlk, 1024u), idO,
                                     (jp | kk) ? 1u : 0u);
                    }
                    umma_commit(ofull);
                    if (jp == NT - 1) umma_commit(smem_u32(&s_ofin));
                    umma_commit(empty0 + 8u * s);   // K and V of the stage are no longer read
                    ++jp;
                    moved = true;
                }
                if (moved) {
                    t_prog = global_timer_ns();
                } else if ((it & 63u) == 63u && global_timer_ns() - t_prog > kCWaitNs) {
                    ok = false;
                    break;
                }
            }
            if (!ok) {
                // let the MMAs already issued finish before the memory is released
                s_fail = 1;
                umma_commit(smem_u32(&s_drain));
                (void)mbar_wait_bounded(smem_u32(&s_drain), 0u, kCWaitNs);
            }
        }
    } else {
        // ---- softmax and output: row r, half h of the keys and of d
        const int pos = posb + (row_ok ? t : 0);   // row r attends keys 0 .. pos
        const uint32_t ocol = lane_base + kCOcol + (uint32_t)(h * HD);
        float m_run = -INFINITY, l_run = 0.f;
        // a wait's result is made warp-uniform (the TMEM accesses are
        // .aligned); after a timeout the warp does no more TMEM or shared-
        // memory work but still takes its pair barrier once per tile
        auto wait_warp = [&](uint32_t bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait_bounded(bar, parity, kCWaitNs)) != 0;
        };
        bool ok = true;
        for (int j = 0; j < NT; ++j) {
            ok = ok && wait_warp(sfull0 + 8u * (j & 1), (uint32_t)((j >> 1) & 1));
            tmem_fence_after();
            const uint32_t scol = lane_base + (uint32_t)((j & 1) * kChunkKeys + 64 * h);
            const int lim = pos - (j * kChunkKeys + 64 * h);   // keys c <= lim of this half are attended
            // no key of this half is masked for any row of the warp (every
            // tile but the last one or two): no selects
            const bool whole = __all_sync(0xffffffffu, lim >= 63) != 0;
            // the max of this half of the row's S; masked keys are -inf (the
            // select ignores what unloaded rows hold)
            float mx = -INFINITY;
            if (ok) {
                uint32_t sa[32], sb[32];
                tmem_ld32(scol, sa);
                tmem_ld32(scol + 32u, sb);
                tmem_wait_ld();
                if (whole) {
#pragma unroll
                    for (int c = 0; c < 32; ++c) mx = fmaxf(mx, fmaxf(__uint_as_float(sa[c]), __uint_as_float(sb[c])));
                } else {
#pragma unroll
                    for (int c = 0; c < 32; ++c) {
                        if (c <= lim) mx = fmaxf(mx, __uint_as_float(sa[c]));
                        if (c + 32 <= lim) mx = fmaxf(mx, __uint_as_float(sb[c]));
                    }
                }
            }
            mx *= p.scale_log2;   // scale_log2 > 0: the max commutes with it
            // the two warps of this lane quarter (both halves of the rows) swap maxima
            s_mx[j & 1][h][r] = mx;
            asm volatile("bar.sync %0, 64;" ::"r"(1 + quarter) : "memory");
            mx = fmaxf(mx, s_mx[j & 1][h ^ 1][r]);
            if (!ok) continue;
            // The reference max moves only when a row's max passes it by more
            // than 2^8 (P stays <= 2^8: exact in the sums, fine for bf16);
            // then O (this half of d) and l are rescaled in place, once the
            // P V already issued has landed.  Both warps of the quarter see
            // the same maxima, so they take the same decision.
            if (j == 0) {
                m_run = mx;   // finite: tile 0 holds key 0 for every row
            } else if (__any_sync(0xffffffffu, mx > m_run + 8.f)) {
                const float m_new = fmaxf(m_run, mx);
                const float alpha = ex2(m_run - m_new);
                // completions of the P V barrier here are j - 1 or j (S_j's
                // commit covered P V of tile j - 2), so the parity of j - 1
                // names the one this waits for
                ok = wait_warp(ofull, (uint32_t)((j - 1) & 1));
                if (!ok) continue;
                tmem_fence_after();
#pragma unroll
                for (int c0 = 0; c0 < HD; c0 += 32) {
                    uint32_t o[32];
                    tmem_ld32(ocol + (uint32_t)c0, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < 32; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha);
                    tmem_st8(ocol + (uint32_t)c0, *reinterpret_cast<const uint32_t(*)[8]>(&o[0]));
                    tmem_st8(ocol + (uint32_t)c0 + 8u, *reinterpret_cast<const uint32_t(*)[8]>(&o[8]));
                    tmem_st8(ocol + (uint32_t)c0 + 16u, *reinterpret_cast<const uint32_t(*)[8]>(&o[16]));
                    tmem_st8(ocol + (uint32_t)c0 + 24u, *reinterpret_cast<const uint32_t(*)[8]>(&o[24]));
                }
                l_run *= alpha;
                m_run = m_new;
            }
            // P = 2^(s scale - m) as P_hi + P_lo over this half's S columns,
            // 32 keys per pass over the 32 columns that pass has just read:
            // keys c0 + 2i, + 1 in column c0 + i (P_hi) and c0 + 16 + i (P_lo)
            float psum = 0.f;
#pragma unroll
            for (int c0 = 0; c0 < 64; c0 += 32) {
                uint32_t sv[32];
                tmem_ld32(scol + (uint32_t)c0, sv);
                tmem_wait_ld();
#pragma unroll
                for (int k8 = 0; k8 < 2; ++k8) {   // 16 keys per store of 8 columns
                    uint32_t whi[8], wlo[8];
#pragma unroll
                    for (int k2 = 0; k2 < 8; ++k2) {
                        const int i = 8 * k8 + k2, c = c0 + 2 * i;
                        float p0 = ex2(__uint_as_float(sv[2 * i]) * p.scale_log2 - m_run);
                        float p1 = ex2(__uint_as_float(sv[2 * i + 1]) * p.scale_log2 - m_run);
                        if (!whole) {
                            p0 = c <= lim ? p0 : 0.f;
                            p1 = c + 1 <= lim ? p1 : 0.f;
                        }
                        whi[k2] = pack_bf16(p0, p1);
                        wlo[k2] = pack_bf16(p0 - bf16_lo(whi[k2]), p1 - bf16_hi(whi[k2]));   // exact differences
                        psum += p0 + p1;   // P_hi + P_lo equals p to about 2^-17
                    }
                    tmem_st8(scol + (uint32_t)(c0 + 8 * k8), whi);
                    tmem_st8(scol + (uint32_t)(c0 + 16 + 8 * k8), wlo);
                }
            }
            tmem_wait_st();
            l_run += psum;
            if ((j + 1) * kChunkKeys > n_keys) {
                // the last tile: V rows of keys >= n_keys hold unloaded or
                // foreign data; zero them so that 0 x V stays 0, after the
                // stage's copies (already complete) are acquired here too
                ok = wait_warp(full0 + 8u * (j % kCStages), (uint32_t)((j / kCStages) & 1));
                if (!ok) continue;
                const int z0 = n_keys - j * kChunkKeys;
                const uint32_t vd = st0 + (uint32_t)((j % kCStages) * Gm::STB + KB * kCBlk);
                for (int i = 32 * sw + lane; i < (kChunkKeys - z0) * KB * 8; i += 32 * kCSoftWarps) {
                    const int row = z0 + i / (KB * 8), rem = i % (KB * 8);
                    sts128(vd + (uint32_t)((rem >> 3) * kCBlk + row * 128 + (rem & 7) * 16), make_uint4(0u, 0u, 0u, 0u));
                }
                fence_proxy_async_smem();   // the zeroed V rows are read by the async proxy
            }
            tmem_fence_before();   // P and any rescaled O written before the MMA goes on
            __syncwarp();
            if (lane == 0) mbar_arrive(pfull);
        }
        // the last P V (its own barrier: the P V barrier may be two phases on)
        if (ok) ok = wait_warp(smem_u32(&s_ofin), 0u);
        if (!ok) s_fail = 1;
        s_l[h][r] = l_run;
        tmem_fence_after();
        __syncthreads();   // (A) s_l, s_bad and s_fail settled
        const bool zero = s_bad != 0 || s_fail != 0;
        const float inv = 1.f / (l_run + s_l[h ^ 1][r]);
        uint4* dst = reinterpret_cast<uint4*>(out_row(t, g) + h * HD);
#pragma unroll
        for (int c0 = 0; c0 < HD; c0 += 32) {
            uint32_t o[32];
            if (!zero) {
                tmem_ld32(ocol + (uint32_t)c0, o);
                tmem_wait_ld();
            }
#pragma unroll
            for (int c = 0; c < 32; c += 8) {
                const float* f = reinterpret_cast<const float*>(&o[c]);
                if (row_ok)
                    dst[(c0 + c) / 8] = zero ? make_uint4(0u, 0u, 0u, 0u)
                                             : make_uint4(pack_bf16(f[0] * inv, f[1] * inv),
                                                          pack_bf16(f[2] * inv, f[3] * inv),
                                                          pack_bf16(f[4] * inv, f[5] * inv),
                                                          pack_bf16(f[6] * inv, f[7] * inv));
            }
        }
        tmem_fence_before();
        __syncthreads();   // (B) every TMEM read done: the allocation may go
        return;
    }
    // warps 0 and 1 (all lanes) meet the softmax warps at (A) and (B)
    __syncwarp();
    __syncthreads();
    tmem_fence_before();
    __syncthreads();
    if (warp == 0) {
        tmem_fence_after();
        tmem_dealloc(tmem, kCCols);
        if (lane == 0) {
            if (s_fail) {
                // copies that no MMA consumed may still be landing in this
                // CTA's shared memory: wait for them (bounded) before exiting
                atomicOr(p.err, kErrTimeout);
                for (int j = s_landed; j < s_issued; ++j)
                    (void)mbar_wait_bounded(full0 + 8u * (j % kCStages), (uint32_t)((j / kCStages) & 1), kCWaitNs);
            }
            if (s_bad && kvh == 0) atomicOr(p.err, kErrPage);
        }
    }
}

template <int D>
cudaError_t prepare_t()
{
    return cudaFuncSetAttribute(chunk_attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                ChunkGeo<D>::BYTES + 1024);
}

}  // namespace

cudaError_t chunk_attn_prepare(int head_dim)
{
    return head_dim == 128 ? prepare_t<128>() : prepare_t<64>();
}

cudaError_t launch_chunk_attn(const AttnParams& p, const CUtensorMap& tmk, const CUtensorMap& tmv, int head_dim,
                              int max_items, cudaStream_t stream)
{
    if (max_items <= 0) return cudaSuccess;
    const dim3 grid((unsigned)p.Hkv, (unsigned)max_items), block(kCThreads);
    if (head_dim == 128)
        chunk_attn_kernel<128><<<grid, block, ChunkGeo<128>::BYTES + 1024, stream>>>(tmk, tmv, p);
    else
        chunk_attn_kernel<64><<<grid, block, ChunkGeo<64>::BYTES + 1024, stream>>>(tmk, tmv, p);
    return cudaGetLastError();
}

}  // namespace pkv
