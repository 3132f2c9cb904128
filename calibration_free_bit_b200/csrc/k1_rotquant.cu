// k1_rotquant.cu -- fused RPBH rotate + per-token norm + Lloyd-Max nearest-centroid codes.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video", pseudocode
// block (online per-token part): x_rot = x R^T, s = norm(x_rot),
// codes = nearest_centroid(x_rot / (s + eps), codebook[d, b]); the same kernel with eps = 0
// serves the offline weight step (rows of W, row_norms).  R = blockdiag(H_h/sqrt h) D P is
// the RPBH rotation of the summary's RPBH paragraph, applied as an O(d log h) butterfly.
//
// B200 design (one HBM-bound pass: read 2d bytes per bf16 row, write d*b/8 + 4):
//   * A CTA holds `groups` token PAIRS.  Each pair is staged in shared memory interleaved:
//     32-bit word j = (x_t0[j], x_t1[j]) as two bf16, so one 4-byte gather load serves both
//     tokens and the butterfly runs on packed fp32x2 (add/sub/fma .f32x2, new on sm_100).
//   * A group of d/32 threads owns one pair; thread g holds 32 consecutive rotated positions
//     of one h-block (h/32 threads per block).  The gather offsets and signs (byte offset of
//     perm[i] in the pair buffer | sign << 31) are converted once per CTA into a shared table
//     and read back with 16-byte loads.
//   * Butterfly: 5 in-register stages, then log2(h/32) shuffle stages across the block's
//     threads.  The per-token sum of squares is reduced across the group (segmented warp
//     shuffles + shared memory); s = sqrt(sum z^2 / h) since z is unnormalised.
//   * Nearest centroid by a uniform-grid table (host-built, <= 1 boundary per cell):
//     a = sat(z*K/(s+eps) + 1/2) (one FFMA.SAT), q = floor(a*2^23) via an fp32x2 add with
//     round-down, word = table[q >> F], code = (word + q*G) >> 24.  The table words fold the
//     cell's base code and its boundary, so the decision is exact in the fixed-point q grid
//     (2^-23 of the grid span, < 1.2e-6 sigma).  Bit widths 2/3/4/8 pack LSB-first.
#include <cuda_bf16.h>

#include "oq_internal.h"

namespace oq {
namespace {

__device__ unsigned int g_k1_err;

constexpr int kE = 32;          // rotated positions per thread (per token)
constexpr int kMaxSeg = 18;     // segment slots per group for the norm reduction

__device__ __forceinline__ float2 f2add(float2 a, float2 b) {
    float2 c;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(c.x), "=f"(c.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return c;
}

__device__ __forceinline__ float2 f2sub(float2 a, float2 b) {
    float2 c;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "sub.rn.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "=f"(c.x), "=f"(c.y) : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return c;
}

__device__ __forceinline__ float2 f2fma(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

// (a + 1.0) rounded toward -inf, for both lanes; returns the fp32 bit patterns.
__device__ __forceinline__ uint2 f2_add_one_rm_bits(float a0, float a1) {
    uint2 r;
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %4};\n\t"
        "add.rm.f32x2 rc, ra, rb;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "=r"(r.x), "=r"(r.y) : "f"(a0), "f"(a1), "f"(1.0f));
    return r;
}

__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

__device__ __forceinline__ uint4 ldg_stream(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint2 lds64(uint32_t addr) {
    uint2 v;
    asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
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

template <int BITS, bool IN_F32, int H>
__global__ void __launch_bounds__(512) k1_rotquant(const K1Params p) {
    constexpr int Q = H / kE;                        // threads per h-block
    constexpr bool REPL = (BITS <= 4);               // per-lane table copies (conflict-free)
    constexpr int TSH = REPL ? 7 : 2;                // table row stride: 32 lanes x 4 B, or 4 B
    constexpr int NW = kE * BITS / 32;               // packed code words per token per thread
    constexpr int PAIR_BYTES = IN_F32 ? 8 : 4;

    extern __shared__ __align__(16) unsigned char smem[];
    const int d = p.d;
    const int GT = d / kE;                           // threads per token pair
    const int NG = p.groups;
    const int tid = threadIdx.x;
    const int grp = tid / GT;
    const int g = tid - grp * GT;
    const int lane = tid & 31;
    const int warp_start = tid - lane;
    const int active = min(32, (int)blockDim.x - warp_start);
    const unsigned wmask = active == 32 ? 0xffffffffu : ((1u << active) - 1u);

    // shared memory: [quantizer table][gather entries][segment partials][pair buffers]
    const int table_words = (p.G + 1) * (REPL ? 32 : 1);
    uint32_t *table = reinterpret_cast<uint32_t *>(smem);
    uint32_t *gent = table + ((table_words + 3) & ~3);
    float2 *red = reinterpret_cast<float2 *>(gent + d);
    unsigned char *pairs = reinterpret_cast<unsigned char *>(red + NG * kMaxSeg);
    unsigned char *mypairs = pairs + (size_t)grp * d * PAIR_BYTES;

    for (int i = tid; i < table_words; i += blockDim.x)
        table[i] = p.grid[REPL ? (i >> 5) : i];
    for (int i = tid; i < d; i += blockDim.x) {
        const uint32_t v = p.rp[i];
        gent[i] = ((v & 0x7fffffffu) * PAIR_BYTES) | (v & 0x80000000u);
    }

    // this thread's 32 rotated positions
    const int blk = g / Q, r = g - blk * Q;
    const int pos0 = blk * H + r * kE;
    const uint4 *myent = reinterpret_cast<const uint4 *>(gent + pos0);
    const uint32_t pair_base = smem_u32(mypairs);
    const uint32_t tbl_lane =
        smem_u32(table) + (REPL ? lane * 4 : 0) - ((0x3F800000u >> p.F) << TSH);
    const uint32_t G = (uint32_t)p.G;
    const int F = p.F;

    // segmented-reduction bookkeeping (a warp may hold the tails of two groups)
    const int seg_end = min(active, lane + (GT - g));
    const bool seg_head = (lane == 0) || (g == 0);
    const int seg_slot = (g == 0) ? 0 : (g + 31) / 32;
    const int nslots = 1 + ((grp * GT + GT - 1) / 32 - (grp * GT) / 32);
    const int row_bytes = d * BITS / 8;

    const long long npairs = ((long long)p.T + 1) / 2;
    for (long long base = (long long)blockIdx.x * NG; base < npairs;
         base += (long long)gridDim.x * NG) {
        const long long pr = base + grp;
        const bool valid = pr < npairs;
        const long long t0 = 2 * pr, t1 = 2 * pr + 1;
        const bool has1 = valid && t1 < p.T;

        // ---- stage the pair, interleaved -------------------------------------------------
        if (valid) {
            if constexpr (!IN_F32) {
                const uint4 *x0 = reinterpret_cast<const uint4 *>(
                    static_cast<const __nv_bfloat16 *>(p.x) + t0 * d);
                const uint4 *x1 = reinterpret_cast<const uint4 *>(
                    static_cast<const __nv_bfloat16 *>(p.x) + t1 * d);
#pragma unroll
                for (int k = 0; k < kE / 8; ++k) {
                    const int c = g + k * GT;            // 16-byte chunk: elements 8c..8c+7
                    uint4 a = ldg_stream(x0 + c);
                    uint4 b = has1 ? ldg_stream(x1 + c) : make_uint4(0, 0, 0, 0);
                    uint4 lo, hi;
                    lo.x = prmt(a.x, b.x, 0x5410); lo.y = prmt(a.x, b.x, 0x7632);
                    lo.z = prmt(a.y, b.y, 0x5410); lo.w = prmt(a.y, b.y, 0x7632);
                    hi.x = prmt(a.z, b.z, 0x5410); hi.y = prmt(a.z, b.z, 0x7632);
                    hi.z = prmt(a.w, b.w, 0x5410); hi.w = prmt(a.w, b.w, 0x7632);
                    uint4 *dst = reinterpret_cast<uint4 *>(mypairs) + 2 * c;
                    dst[0] = lo;
                    dst[1] = hi;
                }
            } else {
                const uint4 *x0 = reinterpret_cast<const uint4 *>(
                    static_cast<const float *>(p.x) + t0 * d);
                const uint4 *x1 = reinterpret_cast<const uint4 *>(
                    static_cast<const float *>(p.x) + t1 * d);
#pragma unroll
                for (int k = 0; k < kE / 4; ++k) {
                    const int c = g + k * GT;            // elements 4c..4c+3
                    uint4 a = ldg_stream(x0 + c);
                    uint4 b = has1 ? ldg_stream(x1 + c) : make_uint4(0, 0, 0, 0);
                    uint4 *dst = reinterpret_cast<uint4 *>(mypairs) + 2 * c;
                    dst[0] = make_uint4(a.x, b.x, a.y, b.y);
                    dst[1] = make_uint4(a.z, b.z, a.w, b.w);
                }
            }
        }
        __syncthreads();

        // ---- gather y[i] = sign[i] * x[perm[i]] for both tokens ------------------------------
        float2 v[kE];
        uint32_t ent[4];
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            if ((e & 3) == 0) {
                const uint4 q4 = myent[e >> 2];
                ent[0] = q4.x; ent[1] = q4.y; ent[2] = q4.z; ent[3] = q4.w;
            }
            const uint32_t en = ent[e & 3];
            const uint32_t sg = en & 0x80000000u;
            if constexpr (!IN_F32) {
                const uint32_t w = lds32(pair_base + (en & 0x7fffffffu));
                v[e].x = __uint_as_float((w << 16) + sg);
                v[e].y = __uint_as_float((w ^ en) & 0xffff0000u);
            } else {
                const uint2 w = lds64(pair_base + (en & 0x7fffffffu));
                v[e].x = __uint_as_float(w.x ^ sg);
                v[e].y = __uint_as_float(w.y ^ sg);
            }
        }

        // ---- block Walsh-Hadamard (natural order), unnormalised --------------------------
#pragma unroll
        for (int s = 1; s < kE; s <<= 1) {
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                if ((e & s) == 0) {
                    const float2 a = v[e], b = v[e + s];
                    v[e] = f2add(a, b);
                    v[e + s] = f2sub(a, b);
                }
            }
        }
#pragma unroll
        for (int m = 1; m < Q; m <<= 1) {
            const float sgn = (r & m) ? -1.0f : 1.0f;   // upper lane keeps (partner - own)
            const float2 sg2 = make_float2(sgn, sgn);
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                float2 o;
                o.x = __shfl_xor_sync(wmask, v[e].x, m);
                o.y = __shfl_xor_sync(wmask, v[e].y, m);
                v[e] = f2fma(sg2, v[e], o);
            }
        }

        // ---- per-token sum of squares over the group ---------------------------------------
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < kE; ++e)
            acc = f2fma(v[e], v[e], acc);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float2 o;
            o.x = __shfl_down_sync(wmask, acc.x, off);
            o.y = __shfl_down_sync(wmask, acc.y, off);
            if (lane + off < seg_end) {
                acc.x += o.x;
                acc.y += o.y;
            }
        }
        if (seg_head)
            red[grp * kMaxSeg + seg_slot] = acc;
        __syncthreads();
        float2 ss = red[grp * kMaxSeg];
        for (int i = 1; i < nslots; ++i) {
            const float2 o = red[grp * kMaxSeg + i];
            ss.x += o.x;
            ss.y += o.y;
        }
        const float s0 = sqrtf(ss.x * (1.0f / H));
        const float s1 = sqrtf(ss.y * (1.0f / H));
        const float m0 = (s0 + p.eps > 0.f) ? p.K / (s0 + p.eps) : 0.f;
        const float m1 = (s1 + p.eps > 0.f) ? p.K / (s1 + p.eps) : 0.f;

        // ---- nearest centroid + pack ---------------------------------------------------------
        uint32_t w0[NW], w1[NW];
#pragma unroll
        for (int i = 0; i < NW; ++i) {
            w0[i] = 0;
            w1[i] = 0;
        }
#pragma unroll
        for (int e = 0; e < kE; ++e) {
            const float a0 = fma_sat(v[e].x, m0, 0.5f);
            const float a1 = fma_sat(v[e].y, m1, 0.5f);
            const uint2 qb = f2_add_one_rm_bits(a0, a1);
            const uint32_t t0w = lds32(tbl_lane + ((qb.x >> F) << TSH));
            const uint32_t t1w = lds32(tbl_lane + ((qb.y >> F) << TSH));
            const uint32_t c0 = (qb.x * G + t0w) >> 24;
            const uint32_t c1 = (qb.y * G + t1w) >> 24;
            const int bit = e * BITS;
            const int wi = bit >> 5, sh = bit & 31;
            w0[wi] |= c0 << sh;
            w1[wi] |= c1 << sh;
            if (sh + BITS > 32) {
                w0[wi + 1] |= c0 >> (32 - sh);
                w1[wi + 1] |= c1 >> (32 - sh);
            }
        }
        if (valid) {
            uint8_t *dst0 = p.codes + t0 * row_bytes + pos0 * BITS / 8;
            store_words<NW>(dst0, w0);
            if (g == 0)
                p.norms[t0] = s0;
            if (has1) {
                store_words<NW>(dst0 + row_bytes, w1);
                if (g == 0)
                    p.norms[t1] = s1;
            }
        }
    }
}

template <int BITS, bool F32>
cudaError_t launch_h(const K1Params &p, int h, dim3 grid, int threads, size_t smem,
                     cudaStream_t st, std::string *why) {
    auto go = [&](auto kern) -> cudaError_t {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)smem);
        if (e != cudaSuccess) {
            *why = "cudaFuncSetAttribute(k1)";
            return e;
        }
        kern<<<grid, threads, smem, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            *why = "k1 launch";
        return e;
    };
    switch (h) {
        case 32: return go(k1_rotquant<BITS, F32, 32>);
        case 64: return go(k1_rotquant<BITS, F32, 64>);
        case 128: return go(k1_rotquant<BITS, F32, 128>);
        case 256: return go(k1_rotquant<BITS, F32, 256>);
        case 512: return go(k1_rotquant<BITS, F32, 512>);
        case 1024: return go(k1_rotquant<BITS, F32, 1024>);
        default: *why = "unsupported h"; return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_k1(const K1Params &p_in, int bits, int h, int in_f32, cudaStream_t st,
                      int num_sms, std::string *why) {
    K1Params p = p_in;
    const int GT = p.d / kE;
    int NG = 256 / GT;
    if (NG < 1)
        NG = 1;
    const long long npairs = ((long long)p.T + 1) / 2;
    if (NG > npairs)
        NG = (int)npairs;
    const size_t pair_bytes = (size_t)p.d * (in_f32 ? 8 : 4);
    while (NG > 1 && NG * pair_bytes > 96 * 1024)
        --NG;
    p.groups = NG;
    const int threads = NG * GT;
    const int table_words = (p.G + 1) * (bits <= 4 ? 32 : 1);
    const size_t smem = (size_t)((table_words + 3) & ~3) * 4 + (size_t)p.d * 4 +
                        sizeof(float2) * NG * kMaxSeg + NG * pair_bytes;
    const long long ctas_needed = (npairs + NG - 1) / NG;
    const int resident = (threads <= 256 ? 3 : (threads <= 512 ? 1 : 1));
    long long grid = (long long)num_sms * resident * 4;
    if (grid > ctas_needed)
        grid = ctas_needed;
    if (grid < 1)
        grid = 1;
    const dim3 g((unsigned)grid);
    switch (bits * 2 + (in_f32 ? 1 : 0)) {
        case 4: return launch_h<2, false>(p, h, g, threads, smem, st, why);
        case 5: return launch_h<2, true>(p, h, g, threads, smem, st, why);
        case 6: return launch_h<3, false>(p, h, g, threads, smem, st, why);
        case 7: return launch_h<3, true>(p, h, g, threads, smem, st, why);
        case 8: return launch_h<4, false>(p, h, g, threads, smem, st, why);
        case 9: return launch_h<4, true>(p, h, g, threads, smem, st, why);
        case 16: return launch_h<8, false>(p, h, g, threads, smem, st, why);
        case 17: return launch_h<8, true>(p, h, g, threads, smem, st, why);
        default: *why = "unsupported bit width"; return cudaErrorInvalidValue;
    }
}

cudaError_t read_and_clear_k1_error(unsigned *out, cudaStream_t st) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_k1_err, sizeof(unsigned), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_k1_err, &zero, sizeof(unsigned), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace oq
