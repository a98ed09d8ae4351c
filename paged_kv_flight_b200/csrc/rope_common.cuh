// rope_common.cuh -- one work item of the RoPE + append, shared by the RoPE +
// append kernel (rope_append.cu) and by the phase of the one-token step that
// runs inside the attention kernel (decode_attn.cu), so that both store the
// same bits.
//
// What an item computes ("Scaling TensorRT-LLM: Kernel Fusion and Inflight
// Batching in Production", section "What Gets Fused": RoPE on q and k of the
// new token; section "The Paged KV-Cache": the new k / v land in the slot the
// request's block table names): 8 rotation pairs (x_i, x_{i+d/2}), i = i0 ..
// i0 + 7, of one q row (rotated in place) or one k row (rotated, then written
// to the pool row of the new token's slot, with the same 16 elements of the v
// row copied there).  Rotation in fp64 (rope_rotate) with one final rounding
// to the storage type; E4M3 pools: k divided by the page's k scale in fp64,
// rounded once to fp32 and encoded (satfinite), v divided by the v scale in
// fp32 and encoded ("TensorRT-LLM Guide: High-Throughput GPU Inference
// Engine", section "4. Native FP8 Quantization").
#pragma once

#include "pkv_internal.h"
#include "pkv_device.cuh"

namespace pkv {
namespace rope {

// The raw bf16 inputs of one item: x_i .. x_{i+7}, x_{i+d/2} .. x_{i+d/2+7},
// and for a k row the v elements at the same places.
struct Item {
    uint4 xa, xb, va, vb;
};

// Item (token row bt of q / k_new / v_new, head row r < Hq + Hkv, first pair
// i0): q head r, or k / v of kv head r - Hq.  Rows are 16-byte aligned.
template <int D>
__device__ __forceinline__ Item load_item(const __nv_bfloat16* q, const __nv_bfloat16* k_new,
                                          const __nv_bfloat16* v_new, int Hq, int Hkv, int bt, int r, int i0)
{
    constexpr int HALF = D / 2;
    Item it;
    const bool is_q = r < Hq;
    const __nv_bfloat16* src = is_q ? q + ((size_t)bt * Hq + r) * D : k_new + ((size_t)bt * Hkv + (r - Hq)) * D;
    it.xa = *reinterpret_cast<const uint4*>(src + i0);
    it.xb = *reinterpret_cast<const uint4*>(src + i0 + HALF);
    it.va = it.vb = make_uint4(0, 0, 0, 0);
    if (!is_q) {
        const __nv_bfloat16* vsrc = v_new + ((size_t)bt * Hkv + (r - Hq)) * D;
        it.va = *reinterpret_cast<const uint4*>(vsrc + i0);
        it.vb = *reinterpret_cast<const uint4*>(vsrc + i0 + HALF);
    }
    return it;
}

// Rotates the item by the angles i0 .. i0 + 7 (cosines cs[i0 + k], sines
// sn[i0 + k]) and stores it: a q row back in place; a k row (kv head
// r - Hq) and its v row into pool row prow = (page Hkv + kvh) P + slot.
template <int D, bool FP8>
__device__ __forceinline__ void store_item(const Item& it, __nv_bfloat16* q, void* k_pool, void* v_pool,
                                           const float* k_scale, const float* v_scale, int Hq, int Hkv, int P,
                                           int bt, int r, int i0, int page, int slot, const double* cs,
                                           const double* sn)
{
    constexpr int HALF = D / 2;
    const bool is_q = r < Hq;
    const int kvh = r - Hq;
    const uint32_t wa[4] = {it.xa.x, it.xa.y, it.xa.z, it.xa.w};
    const uint32_t wb[4] = {it.xb.x, it.xb.y, it.xb.z, it.xb.w};
    double ya[8], yb[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const double a = (double)((k & 1) ? dev::bf16_hi(wa[k >> 1]) : dev::bf16_lo(wa[k >> 1]));
        const double bb = (double)((k & 1) ? dev::bf16_hi(wb[k >> 1]) : dev::bf16_lo(wb[k >> 1]));
        dev::rope_rotate(a, bb, cs[i0 + k], sn[i0 + k], &ya[k], &yb[k]);
    }

    const size_t prow = ((size_t)page * Hkv + kvh) * P + slot;   // pool row (k rows only)
    if (is_q || !FP8) {
        uint32_t oa[4], ob[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            oa[k] = (uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(ya[2 * k])) |
                    ((uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(ya[2 * k + 1])) << 16);
            ob[k] = (uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(yb[2 * k])) |
                    ((uint32_t)__bfloat16_as_ushort(dev::bf16_from_f64(yb[2 * k + 1])) << 16);
        }
        __nv_bfloat16* dst = is_q ? q + ((size_t)bt * Hq + r) * D
                                  : reinterpret_cast<__nv_bfloat16*>(k_pool) + prow * D;
        *reinterpret_cast<uint4*>(dst + i0) = make_uint4(oa[0], oa[1], oa[2], oa[3]);
        *reinterpret_cast<uint4*>(dst + i0 + HALF) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
    }
    if (is_q) return;

    if (!FP8) {
        __nv_bfloat16* vdst = reinterpret_cast<__nv_bfloat16*>(v_pool) + prow * D;
        *reinterpret_cast<uint4*>(vdst + i0) = it.va;
        *reinterpret_cast<uint4*>(vdst + i0 + HALF) = it.vb;
    } else {
        const size_t si = (size_t)page * Hkv + kvh;
        const double sk = (double)k_scale[si];
        const float sv = v_scale[si];
        const uint32_t vwa[4] = {it.va.x, it.va.y, it.va.z, it.va.w};
        const uint32_t vwb[4] = {it.vb.x, it.vb.y, it.vb.z, it.vb.w};
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
        uint8_t* kdst = reinterpret_cast<uint8_t*>(k_pool) + prow * D;
        uint8_t* vdst = reinterpret_cast<uint8_t*>(v_pool) + prow * D;
        *reinterpret_cast<uint2*>(kdst + i0) = *reinterpret_cast<const uint2*>(ka);
        *reinterpret_cast<uint2*>(kdst + i0 + HALF) = *reinterpret_cast<const uint2*>(kb);
        *reinterpret_cast<uint2*>(vdst + i0) = *reinterpret_cast<const uint2*>(qa8);
        *reinterpret_cast<uint2*>(vdst + i0 + HALF) = *reinterpret_cast<const uint2*>(qb8);
    }
}

}  // namespace rope
}  // namespace pkv
