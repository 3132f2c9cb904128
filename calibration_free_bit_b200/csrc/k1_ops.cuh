// k1_ops.cuh -- arithmetic and data-movement helpers of the rotate + norm + quantize kernels
// (k1_rotquant.cu, and the quantize stage of the fused step in k3_fused.cu): packed fp32x2
// butterfly arithmetic, the quantizer's saturating FMA and round-down add, shared loads, the
// one-dimensional bulk copy, LSB-first code packing and the codes -> fp16 centroid output.
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video", pseudocode
// block (online per-token part) and RPBH paragraph.
#pragma once

#include <cstdint>

#include "decode4.cuh"

namespace oq {
namespace k1ops {

// Packed fp32x2 arithmetic (sm_100 FADD2/FFMA2 through the CUDA builtins).
__device__ __forceinline__ float2 f2add(float2 a, float2 b) { return __fadd2_rn(a, b); }

__device__ __forceinline__ float2 f2sub(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);     // a - b, one rounding
}

__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// (a + 1.0) rounded toward -inf, for both lanes; returns the fp32 bit patterns.
__device__ __forceinline__ uint2 f2_add_one_rm_bits(float a0, float a1) {
    const float2 r = __fadd2_rd(make_float2(a0, a1), make_float2(1.0f, 1.0f));
    return make_uint2(__float_as_uint(r.x), __float_as_uint(r.y));
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

// One-dimensional bulk copy global -> this CTA's shared memory, completion counted on `bar`.
__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// Top bytes of a, b, c, d as bytes 0..3 of one word.
__device__ __forceinline__ uint32_t top_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    return prmt_b32(prmt_b32(a, b, 0x0073), prmt_b32(c, d, 0x7300), 0x7610);
}

// 32/BITS codes (each in the top byte of D[k]) -> one LSB-first packed word (BITS = 2, 4, 8).
template <int BITS>
__device__ __forceinline__ uint32_t pack_codes(const uint32_t (&D)[32 / BITS]) {
    if constexpr (BITS == 8) {
        return top_bytes(D[0], D[1], D[2], D[3]);
    } else if constexpr (BITS == 4) {
        const uint32_t even = top_bytes(D[0], D[2], D[4], D[6]);
        const uint32_t odd = top_bytes(D[1], D[3], D[5], D[7]);
        return even | (odd << 4);
    } else {
        const uint32_t q0 = top_bytes(D[0], D[4], D[8], D[12]);
        const uint32_t q1 = top_bytes(D[1], D[5], D[9], D[13]);
        const uint32_t q2 = top_bytes(D[2], D[6], D[10], D[14]);
        const uint32_t q3 = top_bytes(D[3], D[7], D[11], D[15]);
        return q0 | (q1 << 2) | (q2 << 4) | (q3 << 6);
    }
}

// Store `NWORDS` 32-bit words of packed codes; alignment follows from the chunk size.
template <int NWORDS>
__device__ __forceinline__ void store_words(uint8_t *dst, const uint32_t (&w)[NWORDS]) {
    if constexpr (NWORDS % 4 == 0) {
#pragma unroll
        for (int i = 0; i < NWORDS; i += 4)
            *reinterpret_cast<uint4 *>(dst + 4 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
    } else if constexpr (NWORDS % 2 == 0) {
#pragma unroll
        for (int i = 0; i < NWORDS; i += 2)
            *reinterpret_cast<uint2 *>(dst + 4 * i) = make_uint2(w[i], w[i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < NWORDS; ++i)
            *reinterpret_cast<uint32_t *>(dst + 4 * i) = w[i];
    }
}

// 32 codes of one token (NW packed words, LSB-first) -> 32 fp16 unit centroids (16 words)
// through the shared byte table `dect` (entry e of a byte: the centroids of the 8/BITS codes
// it holds), stored as two 32-byte pieces (dst 32-byte aligned: rows of d fp16 with d a
// multiple of 16, a thread's 32 positions at a multiple of 32).  BITS = 2, 4, 8.
// 4-bit codes of the (odd-symmetric) codebook use the byte-permute decode instead (no table
// loads): p.dec_src holds its four sources.
template <int BITS>
__device__ __forceinline__ void decode_store(const uint32_t *dect, const uint32_t (&w)[BITS],
                                             uint4 *dst, const uint32_t (&src)[4]) {
    uint32_t o[16];
    if constexpr (BITS == 4) {                       // 8 codes a word -> 4 words of 2 fp16
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t q[4];
            decode8(w[i], src[0], src[1], src[2], src[3], q);
#pragma unroll
            for (int b = 0; b < 4; ++b)
                o[4 * i + b] = q[b];
        }
    } else if constexpr (BITS == 2) {                // a byte = 4 codes = two words
        const uint2 *d2 = reinterpret_cast<const uint2 *>(dect);
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int b = 0; b < 4; ++b) {
                const uint2 v = d2[(w[i] >> (8 * b)) & 0xffu];
                o[8 * i + 2 * b] = v.x;
                o[8 * i + 2 * b + 1] = v.y;
            }
    } else {                                         // a byte = 1 code = one fp16
        const unsigned short *d16 = reinterpret_cast<const unsigned short *>(dect);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            o[2 * i] = (uint32_t)d16[w[i] & 0xffu] | ((uint32_t)d16[(w[i] >> 8) & 0xffu] << 16);
            o[2 * i + 1] =
                (uint32_t)d16[(w[i] >> 16) & 0xffu] | ((uint32_t)d16[w[i] >> 24] << 16);
        }
    }
    // two 32-byte stores (256-bit, sm_100): every lane writes whole 32-byte sectors
#pragma unroll
    for (int k = 0; k < 2; ++k)
        asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};"
                     ::"l"(dst + 2 * k), "r"(o[8 * k]), "r"(o[8 * k + 1]), "r"(o[8 * k + 2]),
                     "r"(o[8 * k + 3]), "r"(o[8 * k + 4]), "r"(o[8 * k + 5]), "r"(o[8 * k + 6]),
                     "r"(o[8 * k + 7]) : "memory");
}

// GELU(x) = x * Phi(x) of a bf16 x (given as fp32 bits, the bf16 in the top half).  For
// 2^-16 <= |x| < 16 every bf16 value has its own entry in the shared-memory table at tab_smem
// (kGeluTableWords fp32 values, each GELU(x) computed in fp64 and rounded to nearest on the
// host): with v = the bf16 bits without the sign (biased exponent and 7-bit mantissa), entry
// sign * 2560 + v - kGeluV0, kGeluV0 = the bits of 2^-16.  Below 2^-16, GELU(x) = x/2 to
// within 2^-17 relative; from 16 up it is x (Phi(16) = 1 - 6e-58), from -16 down 0 (below
// the smallest fp32).
constexpr int kGeluTableWords = 5120;
constexpr uint32_t kGeluV0 = (127u - 16u) << 7;          // 2^-16
constexpr uint32_t kGeluV1 = kGeluV0 + 2559u;            // largest bf16 below 16
__device__ __forceinline__ float gelu_lookup(uint32_t xb, uint32_t tab_smem) {
    const float x = __uint_as_float(xb);
    const uint32_t v = (xb >> 16) & 0x7fffu;
    const uint32_t sgn = xb >> 31;
    const uint32_t vc = min(max(v, kGeluV0), kGeluV1);
    const float t = __uint_as_float(lds32(tab_smem + 4u * (sgn * 2560u + vc - kGeluV0)));
    return v < kGeluV0 ? 0.5f * x : (v > kGeluV1 ? (sgn ? 0.0f : x) : t);
}
}  // namespace k1ops
}  // namespace oq
