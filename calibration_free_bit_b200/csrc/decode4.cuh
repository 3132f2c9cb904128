// decode4.cuh -- 4-bit codes -> fp16 centroids with byte permutes, for a symmetric codebook.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video", pseudocode
// (x_hat = s * codebook[xc], W_hat = diag(row_norms) * codebook[wc]).  The Lloyd-Max codebook
// of the symmetric N(0,1) density satisfies c_i = -c_{15-i}, and so do its fp16 roundings
// (rounding to nearest even is odd-symmetric).  A code c therefore maps to magnitude index
// m = c - 8 (c >= 8) or 7 - c (c < 8) and the sign of (c >= 8).  The low and high bytes of the
// eight fp16 magnitudes |c_8| .. |c_15| sit in four registers; one byte permute per four
// codes selects the low bytes, one the high bytes, two interleave them into fp16 pairs, and
// one more builds the sign bits: about three instructions per code and no shared memory.
#pragma once

#include <cstdint>

namespace oq {

#if defined(__CUDACC__)
__device__ __forceinline__ uint32_t prmt_b32(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

// Eight 4-bit codes (one word, code k in bits 4k..4k+3) -> eight fp16 centroids as four
// packed pairs (pair j = codes 2j, 2j+1; the lower code in the low half).  L0/L1: low bytes of
// the fp16 centroids 8..11 / 12..15; H0/H1: their high bytes (byte k of a word = centroid
// 8+k or 12+k).
__device__ __forceinline__ void decode8(uint32_t w, uint32_t L0, uint32_t L1, uint32_t H0,
                                        uint32_t H1, uint32_t (&o)[4]) {
    const uint32_t nw = ~w;
    const uint32_t t = (nw >> 3) & 0x11111111u;          // 1 where code < 8 (negative)
    const uint32_t m = (w ^ (t * 7u)) & 0x77777777u;     // magnitude index per nibble
    const uint32_t y = nw << 4;                          // bit 7 of byte b <- code 2b's flag
    const uint32_t lo_a = prmt_b32(L0, L1, m & 0xffffu), hi_a = prmt_b32(H0, H1, m & 0xffffu);
    const uint32_t lo_b = prmt_b32(L0, L1, m >> 16), hi_b = prmt_b32(H0, H1, m >> 16);
    // sign of code 2b -> bit 15 (from y, byte b), of code 2b+1 -> bit 31 (from nw, byte b)
    o[0] = prmt_b32(lo_a, hi_a, 0x5140) ^ (prmt_b32(y, nw, 0x4000) & 0x80008000u);
    o[1] = prmt_b32(lo_a, hi_a, 0x7362) ^ (prmt_b32(y, nw, 0x5010) & 0x80008000u);
    o[2] = prmt_b32(lo_b, hi_b, 0x5140) ^ (prmt_b32(y, nw, 0x6020) & 0x80008000u);
    o[3] = prmt_b32(lo_b, hi_b, 0x7362) ^ (prmt_b32(y, nw, 0x7030) & 0x80008000u);
}

#endif  // __CUDACC__

// Host: the four permute sources from a 16-entry fp16 LUT; false unless the LUT is exactly
// odd-symmetric (lut[15-i] == lut[i] ^ 0x8000), the condition decode8 relies on.
inline bool decode8_sources(const uint16_t *lut, uint32_t *L0, uint32_t *L1, uint32_t *H0,
                            uint32_t *H1) {
    for (int i = 0; i < 8; ++i)
        if (lut[15 - i] != (uint16_t)(lut[i] ^ 0x8000u))
            return false;
    auto bytes4 = [&](int i0, bool hi) {
        uint32_t w = 0;
        for (int k = 0; k < 4; ++k)
            w |= (uint32_t)((lut[i0 + k] >> (hi ? 8 : 0)) & 0xffu) << (8 * k);
        return w;
    };
    *L0 = bytes4(8, false);
    *L1 = bytes4(12, false);
    *H0 = bytes4(8, true);
    *H1 = bytes4(12, true);
    return true;
}

}  // namespace oq
