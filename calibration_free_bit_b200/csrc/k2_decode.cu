// k2_decode.cu -- decode prepass of the codebook linear layer: packed b-bit codes -> fp16
// unit-variance centroids, the operands of the tcgen05 GEMM (k2_linear.cu).
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video", pseudocode
// (x_hat = s * codebook[xc], W_hat = diag(row_norms) * codebook[wc]); the packed layout is
// LSB-first per row (code k of a row in bits [k*b, k*b + b) of its byte stream).
#include "decode4.cuh"
#include "oq_internal.h"

namespace oq {
namespace {

// ------------------------------------------------------------------------------------------
// Decode prepass: packed codes -> fp16 unit centroids.  A thread handles groups of 8 codes
// (BITS bytes in, 16 bytes out); consecutive lanes take consecutive groups, so a warp reads
// 32*BITS contiguous bytes and writes 512 contiguous bytes per group round, and each thread
// keeps kDecUnroll independent groups in flight.  The lookup goes through a shared table
// indexed by whole groups of codes (a byte holds 2 codes at b = 4 and 4 codes at b = 2;
// 6 bits hold 2 codes at b = 3), so one shared load yields 2 or 4 fp16 values.
// ------------------------------------------------------------------------------------------
struct DecodeParams {
    const uint8_t *codes;
    uint16_t *out;
    long long groups;           // rows * d / 8
    uint32_t L0, L1, H0, H1;    // decode8 sources (symmetric 4-bit path only)
    uint16_t lut[256];
    // symmetric 4-bit path only: a second tensor decoded by the same launch (groups2 = 0:
    // none), groups g >= groups being its groups g - groups, with its own decode8 sources
    const uint8_t *codes2;
    uint16_t *out2;
    long long groups2;
    uint32_t L0b, L1b, H0b, H1b;
};

constexpr int kDecThreads = 256;
constexpr int kDecUnroll = 8;

template <int BITS>
__device__ __forceinline__ uint4 decode_group(const uint32_t *tab32, uint64_t v) {
    uint32_t o[4];
    if constexpr (BITS == 6) {                        // 6 bytes, 8 codes of 6 bits (fp16 entries)
        const uint16_t *t = reinterpret_cast<const uint16_t *>(tab32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = (uint32_t)t[(v >> (12 * q)) & 63u] |
                   ((uint32_t)t[(v >> (12 * q + 6)) & 63u] << 16);
    } else if constexpr (BITS == 2) {                        // 2 bytes, 4 codes each -> uint2 entries
        const uint2 *t = reinterpret_cast<const uint2 *>(tab32);
        const uint2 a = t[v & 0xffu], b = t[(v >> 8) & 0xffu];
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    } else if constexpr (BITS == 3) {                 // 4 pairs of 6 bits
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = tab32[(v >> (6 * q)) & 63u];
    } else if constexpr (BITS == 4) {                 // 4 bytes, 2 codes each
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = tab32[(v >> (8 * q)) & 0xffu];
    } else {                                          // 8 bytes, 1 code each (fp16 entries)
        const uint16_t *t = reinterpret_cast<const uint16_t *>(tab32);
#pragma unroll
        for (int q = 0; q < 4; ++q)
            o[q] = (uint32_t)t[(v >> (16 * q)) & 0xffu] |
                   ((uint32_t)t[(v >> (16 * q + 8)) & 0xffu] << 16);
    }
    return make_uint4(o[0], o[1], o[2], o[3]);
}

template <int BITS>
__device__ __forceinline__ uint64_t load_group(const uint8_t *codes, long long g) {
    const uint8_t *src = codes + g * BITS;
    if constexpr (BITS == 2)
        return __ldg(reinterpret_cast<const unsigned short *>(src));
    else if constexpr (BITS == 4)
        return __ldg(reinterpret_cast<const unsigned int *>(src));
    else if constexpr (BITS == 8)
        return __ldg(reinterpret_cast<const unsigned long long *>(src));
    else if constexpr (BITS == 6)                     // 6 bytes at an even address
        return (uint64_t)__ldg(reinterpret_cast<const unsigned short *>(src)) |
               ((uint64_t)__ldg(reinterpret_cast<const unsigned short *>(src + 2)) << 16) |
               ((uint64_t)__ldg(reinterpret_cast<const unsigned short *>(src + 4)) << 32);
    else
        return (uint64_t)__ldg(src) | ((uint64_t)__ldg(src + 1) << 8) |
               ((uint64_t)__ldg(src + 2) << 16);
}

// SYM (BITS == 4 only): decode with byte permutes instead of the shared table.
template <int BITS, bool SYM>
__global__ void __launch_bounds__(kDecThreads) k2_decode(const __grid_constant__ DecodeParams p) {
    // b=2: 256 entries of 4 fp16 (uint2); b=3: 64 entries of 2 fp16; b=4: 256 of 2;
    // b=6: 64 of 1; b=8: 256 of 1
    constexpr int PER = BITS == 2 ? 4 : ((BITS == 8 || BITS == 6) ? 1 : 2);   // codes per lookup
    constexpr int IDX_BITS = PER * BITS;
    constexpr int ENTRIES = 1 << IDX_BITS;
    static_assert(!SYM || BITS == 4, "byte-permute decode is 4-bit only");
    __shared__ __align__(16) uint16_t tab[SYM ? 8 : (ENTRIES * PER < 512 ? 512 : ENTRIES * PER)];
    pdl_trigger();
    if constexpr (!SYM) {
        for (int e = threadIdx.x; e < ENTRIES; e += blockDim.x)
#pragma unroll
            for (int i = 0; i < PER; ++i)
                tab[e * PER + i] = p.lut[(e >> (i * BITS)) & ((1 << BITS) - 1)];
        __syncthreads();
    }
    pdl_wait();                                        // codes, out: earlier work done
    const uint32_t *tab32 = reinterpret_cast<const uint32_t *>(tab);
    const long long stride = (long long)gridDim.x * blockDim.x;
    uint4 *out = reinterpret_cast<uint4 *>(p.out);
    uint4 *out2 = reinterpret_cast<uint4 *>(p.out2);
    const long long total = p.groups + (SYM ? p.groups2 : 0);
    for (long long g0 = (long long)blockIdx.x * blockDim.x + threadIdx.x; g0 < total;
         g0 += kDecUnroll * stride) {
        uint64_t v[kDecUnroll];
#pragma unroll
        for (int j = 0; j < kDecUnroll; ++j) {
            const long long g = g0 + j * stride;
            if (SYM && g >= p.groups)
                v[j] = g < total ? load_group<BITS>(p.codes2, g - p.groups) : 0;
            else
                v[j] = g < p.groups ? load_group<BITS>(p.codes, g) : 0;
        }
#pragma unroll
        for (int j = 0; j < kDecUnroll; ++j) {
            const long long g = g0 + j * stride;
            if (g < total) {
                if constexpr (SYM) {
                    uint32_t o[4];
                    if (g < p.groups) {
                        decode8((uint32_t)v[j], p.L0, p.L1, p.H0, p.H1, o);
                        out[g] = make_uint4(o[0], o[1], o[2], o[3]);
                    } else {
                        decode8((uint32_t)v[j], p.L0b, p.L1b, p.H0b, p.H1b, o);
                        out2[g - p.groups] = make_uint4(o[0], o[1], o[2], o[3]);
                    }
                } else {
                    out[g] = decode_group<BITS>(tab32, v[j]);
                }
            }
        }
    }
}

template <int BITS, bool SYM>
cudaError_t decode(const DecodeParams &dp, cudaStream_t st, int num_sms) {
    long long blocks = (dp.groups + (SYM ? dp.groups2 : 0) + kDecThreads - 1) / kDecThreads;
    const long long cap = (long long)num_sms * (2048 / kDecThreads);   // one resident wave
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    return launch_pdl(k2_decode<BITS, SYM>, dim3((unsigned)blocks), dim3(kDecThreads), 0, st, dp);
}

}  // namespace

cudaError_t launch_decode(int bits, const uint8_t *codes, uint16_t *out, long long rows, int d,
                          const uint16_t *lut, cudaStream_t st, int num_sms, std::string *why) {
    DecodeParams dp;
    dp.codes = codes;
    dp.out = out;
    dp.groups = rows * (d / 8);
    dp.codes2 = nullptr;
    dp.out2 = nullptr;
    dp.groups2 = 0;
    dp.L0b = dp.L1b = dp.H0b = dp.H1b = 0;
    for (int i = 0; i < 256; ++i)
        dp.lut[i] = lut[i];
    dp.L0 = dp.L1 = dp.H0 = dp.H1 = 0;
    cudaError_t e;
    switch (bits) {
        case 2: e = decode<2, false>(dp, st, num_sms); break;
        case 3: e = decode<3, false>(dp, st, num_sms); break;
        case 4:
            e = decode8_sources(lut, &dp.L0, &dp.L1, &dp.H0, &dp.H1)
                    ? decode<4, true>(dp, st, num_sms)
                    : decode<4, false>(dp, st, num_sms);
            break;
        case 6: e = decode<6, false>(dp, st, num_sms); break;
        case 8: e = decode<8, false>(dp, st, num_sms); break;
        default: e = cudaErrorInvalidValue;
    }
    if (e != cudaSuccess)
        *why = "decode launch";
    return e;
}

bool launch_decode_pair(int bits_a, const uint8_t *codes_a, uint16_t *out_a, long long rows_a,
                        const uint16_t *lut_a, int bits_b, const uint8_t *codes_b,
                        uint16_t *out_b, long long rows_b, const uint16_t *lut_b, int d,
                        cudaStream_t st, int num_sms, cudaError_t *err, std::string *why) {
    DecodeParams dp;
    if (bits_a != 4 || bits_b != 4 ||
        !decode8_sources(lut_a, &dp.L0, &dp.L1, &dp.H0, &dp.H1) ||
        !decode8_sources(lut_b, &dp.L0b, &dp.L1b, &dp.H0b, &dp.H1b))
        return false;
    dp.codes = codes_a;
    dp.out = out_a;
    dp.groups = rows_a * (d / 8);
    dp.codes2 = codes_b;
    dp.out2 = out_b;
    dp.groups2 = rows_b * (d / 8);
    for (int i = 0; i < 256; ++i)
        dp.lut[i] = 0;
    *err = decode<4, true>(dp, st, num_sms);
    if (*err != cudaSuccess)
        *why = "decode launch";
    return true;
}

}  // namespace oq
