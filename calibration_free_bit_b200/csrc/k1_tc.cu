// k1_tc.cu -- rotate + norm + quantize with the block Walsh-Hadamard on the tensor cores.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video": RPBH paragraph
// (uniform permutation, random sign flips, block-diagonal Walsh-Hadamard), pseudocode online
// part (x_rot = x R^T; s = norm(x_rot); codes = nearest_centroid(x_rot / (s + eps))).
//
// For bf16 rows the block transform is a small dense contraction, so it runs as tcgen05.mma.
// Per 128 rotated positions (a "chunk") the transform is D[c, t] = sum_p Hb[c, p] Y[t, p],
// where Y is the gathered, sign-flipped input (y[i] = sign[i] * x[perm[i]]) and
// Hb = blockdiag(H_h) for h <= 128 (H_h the Sylvester matrix, entries +-1, exact in bf16).
// Every chunk multiplies the same Hb, so one MMA serves a "segment" of SEG = 8 chunks of a tile
// of 8 tokens: its B operand stacks the segment's (chunk, token) rows along N (N = 64), and
// its accumulator holds column 8 * chunk + token.  Products of bf16 +-1 and bf16 inputs are
// exact and accumulate in fp32.  h = 256 = H_2 (x) H_128: the two 128-chunks of a block come
// out of the MMA as u = H y_a and v = H y_b, and the epilogue forms u + v and u - v.
//
// The norm comes from the staged input rows: s = ||R x|| = ||x|| because R is orthogonal (the
// summary's rotation-cancellation paragraph), so the quantizer knows s before the rotated
// values exist and each segment is quantized as soon as its MMA completes.
//
// Warp roles (one CTA per SM, persistent over tiles of 8 tokens):
//   warp 0      bulk-copies the 8 rows of a tile into one of two staging buffers
//   warp 1      owns tensor memory; one thread issues the MMAs (8 per segment, K = 128)
//   warps 2-3   norms: s_t = ||x_t|| from the staged rows (fixed-order fp32 sums)
//   warps 4-7   gather: per segment, 8 pieces of 16 bytes (8 positions of one token) per
//               thread, written into the K-major, 128-byte-swizzled B operand
//   warps 8-15  epilogue: tensor memory -> quantize -> code bytes in shared memory ([position]
//               [token], 8 bytes a position); at the end of a tile they transpose, pack
//               (LSB-first) and store them
// Hb sits in tensor memory (columns 0..63, the A operand of the .ts MMA form); segment
// accumulators use a ring of 6 x 64 columns after it.  Every mbarrier wait is bounded (about
// 2 s of SM clock); a wait that gives up sets a bit in the device error word and the CTA
// winds down.
#include <cuda.h>

#include <mutex>

#include "oq_internal.h"
#include "sm100_common.cuh"

namespace oq {
namespace {

using namespace sm100;

__device__ unsigned int g_k1tc_err;

enum : unsigned {
    TC_ERR_STAGE = 1u << 0,     // staging copy or its release
    TC_ERR_RING = 1u << 1,      // gather ring / MMA hand-off
    TC_ERR_ACC = 1u << 2,       // accumulator hand-off
    TC_ERR_NORM = 1u << 3,      // norm hand-off
    TC_ERR_CODES = 1u << 4,     // code-tile hand-off
};

constexpr int NT = 8;            // tokens per tile
constexpr int SEG = 8;           // chunks per segment (one MMA group)
constexpr int SEG_N = NT * SEG;  // MMA N of a full segment: 64
constexpr int RING = 3;          // B operand ring of segments (gather -> MMA)
constexpr int TSLOTS = 6;        // accumulator ring of segments (MMA -> epilogue)
constexpr int H_COLS = 64;       // Hb: 128 x 128 bf16 = 64 TMEM columns
constexpr int TMEM_COLS = 512;
constexpr int B_ATOM = SEG * 1024;   // one 64-wide K atom of a segment: 8 groups of 8 rows
constexpr int B_SEG = 2 * B_ATOM;    // K = 128: two atoms, 16 KB
constexpr int kNormWarps = 2, kGatherWarps = 4, kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kNormWarps + kGatherWarps + kEpiWarps);   // 512
constexpr int kNumBars = 2 * 4 + 2 * RING + 2 * TSLOTS + 2 * 2 + 2;
static_assert(H_COLS + TSLOTS * SEG_N <= TMEM_COLS, "tensor memory budget");

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B (K-major), M = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
           ((uint32_t)(128 >> 4) << 24);
}



__device__ __forceinline__ float fma_sat(float a, float b, float c) {
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// (a + 1.0) rounded toward -inf, two values; returns the fp32 bit patterns.
__device__ __forceinline__ uint2 add_one_rm_bits(float a0, float a1) {
    const float2 r = __fadd2_rd(make_float2(a0, a1), make_float2(1.0f, 1.0f));
    return make_uint2(__float_as_uint(r.x), __float_as_uint(r.y));
}

__device__ __forceinline__ void bulk_copy(uint32_t dst, const void *src, uint32_t bytes,
                                          uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

// 32x32b.x8: 8 consecutive TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld8_nowait(uint32_t taddr, uint32_t (&r)[8]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Store BITS words of packed codes (32 codes) at dst; alignment 4 * (BITS & -BITS) bytes.
template <int BITS>
__device__ __forceinline__ void store_packed(uint8_t *dst, const uint32_t (&w)[BITS]) {
    if constexpr (BITS % 4 == 0) {
#pragma unroll
        for (int i = 0; i < BITS; i += 4)
            *reinterpret_cast<uint4 *>(dst + 4 * i) = make_uint4(w[i], w[i + 1], w[i + 2], w[i + 3]);
    } else if constexpr (BITS % 2 == 0) {
#pragma unroll
        for (int i = 0; i < BITS; i += 2)
            *reinterpret_cast<uint2 *>(dst + 4 * i) = make_uint2(w[i], w[i + 1]);
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i)
            *reinterpret_cast<uint32_t *>(dst + 4 * i) = w[i];
    }
}

// 32 codes, one per byte (b[k] = bytes 4k..4k+3 = codes 4k..4k+3) -> BITS words, LSB-first.
template <int BITS>
__device__ __forceinline__ void pack32(const uint32_t (&b)[8], uint32_t (&w)[BITS]) {
    if constexpr (BITS == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            w[i] = b[i];
    } else if constexpr (BITS == 4) {
        // byte 0 of (x | x >> 4) = c0 | c1 << 4, byte 2 = c2 | c3 << 4
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t lo = b[2 * i] | (b[2 * i] >> 4), hi = b[2 * i + 1] | (b[2 * i + 1] >> 4);
            w[i] = prmt(lo, hi, 0x6420);
        }
    } else if constexpr (BITS == 2) {
        // byte 0 of u = x | x >> 6 | (x | x >> 6) >> 12 holds c0 | c1 << 2 | c2 << 4 | c3 << 6
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            uint32_t q[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const uint32_t u = b[4 * i + k] | (b[4 * i + k] >> 6);
                q[k] = u | (u >> 12);
            }
            w[i] = prmt(prmt(q[0], q[1], 0x0040), prmt(q[2], q[3], 0x0040), 0x5410);
        }
    } else {
#pragma unroll
        for (int i = 0; i < BITS; ++i)
            w[i] = 0;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
            const uint32_t c = (b[k >> 2] >> (8 * (k & 3))) & 0xffu;
            const int bit = k * BITS, wi = bit >> 5, sh = bit & 31;
            w[wi] |= c << sh;
            if (sh + BITS > 32)
                w[wi + 1] |= c >> (32 - sh);
        }
    }
}

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1) k1_tc(const K1TcParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *basep = smem_raw + (base - raw);
    const int d = p.d;
    const int nchunk = d / 128;
    const int nseg = (nchunk + SEG - 1) / SEG;
    const uint32_t RS = 2u * d + 16u;                    // staged row stride (bank spread)
    // [B ring][staging x2][code tiles x2][entries][table][norm scales][barriers][tmem slot]
    const uint32_t sB = base;
    const uint32_t sStage = sB + RING * B_SEG;
    const uint32_t sCodes = sStage + 2 * NT * RS;
    const uint32_t sEnt = sCodes + 2 * NT * (uint32_t)d;
    const uint32_t sTbl = sEnt + 2u * d;
    const uint32_t sScale = sTbl + 4u * p.tbl_words;     // [2][NT] float
    const uint32_t bars = (sScale + 2 * NT * 4 + 7u) & ~7u;
    auto stage_full = [&](int b) { return bars + 8u * b; };
    auto stage_free = [&](int b) { return bars + 8u * (2 + b); };
    auto norm_ready = [&](int b) { return bars + 8u * (4 + b); };
    auto norm_free = [&](int b) { return bars + 8u * (6 + b); };
    auto bfull = [&](int r) { return bars + 8u * (8 + r); };
    auto bempty = [&](int r) { return bars + 8u * (8 + RING + r); };
    auto tfull = [&](int s) { return bars + 8u * (8 + 2 * RING + s); };
    auto tempty = [&](int s) { return bars + 8u * (8 + 2 * RING + TSLOTS + s); };
    auto codes_done = [&](int b) { return bars + 8u * (8 + 2 * RING + 2 * TSLOTS + b); };
    auto codes_free = [&](int b) { return bars + 8u * (8 + 2 * RING + 2 * TSLOTS + 2 + b); };
    const uint32_t setup_bar = bars + 8u * (kNumBars - 2);
    const uint32_t drain_bar = bars + 8u * (kNumBars - 1);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(basep + (bars + 8u * kNumBars - base));
    float *scale_s = reinterpret_cast<float *>(basep + (sScale - base));
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long ntiles = ((long long)p.T + NT - 1) / NT;
    // chunks in segment g, and the MMA N (a multiple of 16: an odd count gets one zero group)
    auto seg_chunks = [&](int g) { return min(SEG, nchunk - g * SEG); };

    if (threadIdx.x == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(stage_full(b), 1);
            mbar_init(stage_free(b), kNormWarps + kGatherWarps);
            mbar_init(norm_ready(b), kNormWarps);
            mbar_init(norm_free(b), kEpiWarps);
            mbar_init(codes_done(b), kEpiWarps);
            mbar_init(codes_free(b), kEpiWarps);
        }
        for (int r = 0; r < RING; ++r) {
            mbar_init(bfull(r), kGatherWarps);
            mbar_init(bempty(r), 1);
        }
        for (int s = 0; s < TSLOTS; ++s) {
            mbar_init(tfull(s), 1);
            mbar_init(tempty(s), kEpiWarps);
        }
        mbar_init(setup_bar, 1);
        mbar_init(drain_bar, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
        // rotation entries and quantizer table: two bulk copies
        mbar_expect_tx(setup_bar, 2u * d + 4u * p.tbl_words);
        bulk_copy(sEnt, p.ent, 2u * d, setup_bar);
        bulk_copy(sTbl, p.tbl_img, 4u * p.tbl_words, setup_bar);
    }
    // the B ring starts at zero, so a padding group (odd chunk count) is finite
    for (uint32_t i = threadIdx.x; i < RING * B_SEG / 16; i += blockDim.x)
        *reinterpret_cast<uint4 *>(basep + (sB - base) + 16u * i) = make_uint4(0, 0, 0, 0);
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(TMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp >= 8 && warp < 12) {
        // Hb row r = 32 (warp % 4) + lane into columns 0..63: column j holds K = 2j (low half)
        // and 2j + 1 (high half); entry (r, k) = (-1)^popcount(r & k & (hb - 1)) inside a
        // diagonal block (the Sylvester entry of the in-block indices), 0 outside
        const int r = (warp & 3) * 32 + lane;
        const int hb = p.h < 128 ? p.h : 128;
        uint32_t v[32];
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                uint32_t wv = 0;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int k = 2 * (half * 32 + j) + e;
                    uint32_t hv = 0;
                    if (r / hb == k / hb)
                        hv = (__popc(r & k & (hb - 1)) & 1) ? 0xBF80u : 0x3F80u;   // bf16 -1 / +1
                    wv |= hv << (16 * e);
                }
                v[j] = wv;
            }
            tmem_st32(tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)(half * 32), v);
        }
        tmem_st_wait();
    }
    // the B-ring zeros (generic proxy) must be visible to the tensor core
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };
    auto give_up = [&](unsigned bit) {
        atomicOr(&g_k1tc_err, bit);
        atomicExch(&abort_flag, 1);
    };
    if (!mbar_wait(setup_bar, 0))
        give_up(TC_ERR_STAGE);

    if (warp == 0) {
        // ---------------- producer: staging rows ----------------
        if (lane == 0) {
            int k = 0;
            for (long long ti = blockIdx.x; ti < ntiles && !aborted(); ti += gridDim.x, ++k) {
                const int b = k & 1;
                if (k >= 2 && !mbar_wait(stage_free(b), ((k >> 1) & 1) ^ 1)) {
                    give_up(TC_ERR_STAGE);
                    break;
                }
                const long long t0 = ti * NT;
                const int nv = (int)min((long long)NT, p.T - t0);
                mbar_expect_tx(stage_full(b), (uint32_t)nv * 2u * d);
                for (int t = 0; t < nv; ++t)
                    bulk_copy(sStage + (uint32_t)(b * NT + t) * RS, p.x + (t0 + t) * 2 * d,
                              2u * d, stage_full(b));
            }
            // let the copies in flight land before the CTA can exit
            for (int j = k > 2 ? k - 2 : 0; j < k; ++j)
                mbar_wait(stage_full(j & 1), (j >> 1) & 1);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer: one group of 8 MMAs (K = 128) per segment -------------
        if (lane == 0) {
            uint32_t q = 0;                                  // segment counter
            for (long long ti = blockIdx.x; ti < ntiles && !aborted(); ti += gridDim.x) {
                bool ok = true;
                for (int g = 0; g < nseg; ++g, ++q) {
                    const int r = q % RING, s = q % TSLOTS;
                    if (!mbar_wait(bfull(r), (q / RING) & 1)) {
                        give_up(TC_ERR_RING);
                        ok = false;
                        break;
                    }
                    if (q >= TSLOTS && !mbar_wait(tempty(s), ((q / TSLOTS) & 1) ^ 1)) {
                        give_up(TC_ERR_ACC);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int n = NT * ((seg_chunks(g) + 1) & ~1);   // multiple of 16
                    const uint32_t idesc = idesc_bf16(n);
                    const uint32_t d_tmem = tmem + (uint32_t)(H_COLS + s * SEG_N);
                    const uint32_t bseg = sB + (uint32_t)r * B_SEG;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)   // K = 128 in steps of 16
                        mma_ts(d_tmem, tmem + (uint32_t)(8 * kk),
                               sw128_desc(bseg + (uint32_t)(kk >> 2) * B_ATOM) +
                                   (uint64_t)(2 * (kk & 3)),
                               idesc, kk != 0);
                    mma_commit(bempty(r));
                    mma_commit(tfull(s));
                }
                if (!ok)
                    break;
            }
            mma_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0))
                atomicOr(&g_k1tc_err, TC_ERR_ACC);
        }
    } else if (warp < 2 + kNormWarps) {
        // ---------------- norms: s_t = ||x_t|| in fixed order ----------------
        const int nw = warp - 2;
        int k = 0;
        for (long long ti = blockIdx.x; ti < ntiles; ti += gridDim.x, ++k) {
            const int b = k & 1;
            const bool ok_in = mbar_wait(stage_full(b), (k >> 1) & 1);
            const bool ok_out = k < 2 || mbar_wait(norm_free(b), ((k >> 1) & 1) ^ 1);
            if (!__all_sync(0xffffffffu, ok_in && ok_out && !aborted())) {
                if (lane == 0 && !(ok_in && ok_out))
                    give_up(TC_ERR_NORM);
                break;
            }
            // this warp's tokens nw, nw + 2, nw + 4, nw + 6 together: two fp32x2 partial sums per
            // token (16 independent chains per thread), fixed order, then a shuffle tree
            const long long t0 = ti * NT;
            constexpr int TPW = NT / kNormWarps;               // tokens per norm warp
            float2 acc[TPW][2];
#pragma unroll
            for (int j = 0; j < TPW; ++j)
                acc[j][0] = acc[j][1] = make_float2(0.f, 0.f);
            const unsigned char *rows = basep + (sStage - base) + (size_t)(b * NT + nw) * RS;
            for (int i = lane; i < d / 8; i += 32) {
#pragma unroll
                for (int j = 0; j < TPW; ++j) {
                    const uint4 v = *reinterpret_cast<const uint4 *>(
                        rows + (size_t)j * kNormWarps * RS + 16 * i);
                    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                    for (int k2 = 0; k2 < 4; ++k2) {
                        const float2 f = make_float2(__uint_as_float(w[k2] << 16),
                                                     __uint_as_float(w[k2] & 0xffff0000u));
                        acc[j][k2 & 1] = __ffma2_rn(f, f, acc[j][k2 & 1]);
                    }
                }
            }
#pragma unroll
            for (int j = 0; j < TPW; ++j) {
                const int t = nw + j * kNormWarps;
                float ss = (acc[j][0].x + acc[j][0].y) + (acc[j][1].x + acc[j][1].y);
#pragma unroll
                for (int m = 16; m >= 1; m >>= 1)
                    ss += __shfl_xor_sync(0xffffffffu, ss, m);
                if (t0 + t >= p.T)
                    ss = 0.f;                                   // rows past T: unused
                if (lane == 0) {
                    const float sn = sqrtf(ss);
                    scale_s[b * NT + t] = (sn + p.eps > 0.f) ? p.K / (sn + p.eps) : 0.f;
                    if (t0 + t < p.T)
                        p.norms[t0 + t] = sn;
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(norm_ready(b));
                mbar_arrive(stage_free(b));
            }
        }
    } else if (warp < 2 + kNormWarps + kGatherWarps) {
        // ---------------- gather: Y[t, i] = sign[i] * x_t[perm[i]] into the B operand --------
        // thread: token n = lane & 7 and piece pc = (warp - 4) * 4 + lane / 8 (positions
        // 8 pc .. 8 pc + 7 of a chunk) of every chunk of the segment.  Row n of chunk j's
        // 8-row group of K atom pc / 8 gets the piece at 16-byte column (pc % 8) ^ n (the
        // 128-byte swizzle).
        const int gw = warp - 2 - kNormWarps;
        const int n = lane & 7, pc = gw * 4 + (lane >> 3);
        const uint32_t dst_off = (uint32_t)(pc >> 3) * B_ATOM + (uint32_t)n * 128u +
                                 (uint32_t)(((pc & 7) ^ n) << 4);
        const unsigned char *entp = basep + (sEnt - base) + 16u * (uint32_t)pc;
        uint32_t q = 0;
        int k = 0;
        bool stop = false;
        for (long long ti = blockIdx.x; ti < ntiles && !stop; ti += gridDim.x, ++k) {
            const int b = k & 1;
            const bool ok = mbar_wait(stage_full(b), (k >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (lane == 0 && !ok)
                    give_up(TC_ERR_STAGE);
                break;
            }
            const unsigned short *rowp = reinterpret_cast<const unsigned short *>(
                basep + (sStage - base) + (size_t)(b * NT + n) * RS);
            for (int g = 0; g < nseg; ++g, ++q) {
                const int r = q % RING;
                if (q >= RING) {
                    const bool okr = mbar_wait(bempty(r), ((q / RING) & 1) ^ 1);
                    if (!__all_sync(0xffffffffu, okr)) {
                        if (lane == 0)
                            give_up(TC_ERR_RING);
                        stop = true;
                        break;
                    }
                }
                const int cnt = seg_chunks(g);
                unsigned char *dstp = basep + (sB - base) + r * B_SEG + dst_off;
#pragma unroll
                for (int j = 0; j < SEG; ++j) {
                    if (j >= cnt)                                  // warp-uniform
                        break;
                    const int c = g * SEG + j;
                    const uint4 e4 = *reinterpret_cast<const uint4 *>(entp + 256u * c);
                    const uint32_t ew[4] = {e4.x, e4.y, e4.z, e4.w};
                    uint32_t o[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t e0 = ew[i] & 0xffffu, e1 = ew[i] >> 16;
                        const uint32_t v0 = rowp[e0 & 0x7fffu];
                        const uint32_t v1 = rowp[e1 & 0x7fffu];
                        o[i] = ((v0 | (v1 << 16)) ^ ((e0 | (e1 << 16)) & 0x80008000u));
                    }
                    *reinterpret_cast<uint4 *>(dstp + j * 1024) = make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(bfull(r));
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(stage_free(b));
        }
    } else {
        // ---------------- epilogue: TMEM -> quantize -> code bytes -> packed rows ----------
        // warp e = warp - 8: TMEM lane quarter e % 4 (rotated positions 32 (e % 4) + lane of a
        // chunk) and chunk parity e / 4 of each segment (h = 256: chunk-pair parity); the
        // accumulator column of (chunk j of the segment, token t) is 8 j + t.
        const int e = warp - 2 - kNormWarps - kGatherWarps;
        const int quarter = e & 3, par = e >> 2;
        const int pos = quarter * 32 + lane;
        constexpr bool REPL = (BITS <= 4);
        constexpr int TSH = REPL ? 7 : 2;
        // table word for fp32 bits q: tbl[(q >> F) << TSH], the per-lane copy when replicated
        const unsigned char *tbl_lane = basep + (sTbl - base) + (REPL ? lane * 4 : 0) -
                                        ((0x3F800000u >> p.F) << TSH);
        const uint32_t G = (uint32_t)p.G;
        const int F = p.F;
        const int row_bytes = d * BITS / 8;
        const bool pairs = p.h == 256;
        // slot of position `pos` in the code tile: bits 0..4 XOR the group-of-32 index, so the
        // packer's lanes (one group each, same offset) hit different banks
        auto swz = [](int pos) { return (pos & ~31) | ((pos & 31) ^ ((pos >> 5) & 15)); };
        // code of each of 8 token values (D = q G + table[q >> F]; the code is its top byte),
        // two tokens per packed round-down add; returns the 8 codes as bytes of two words
        // (token t in byte t % 4 of word t / 4)
        auto codes8 = [&](const float (&z)[NT], const float (&m)[NT]) -> uint2 {
            uint32_t D[NT];
#pragma unroll
            for (int t = 0; t < NT; t += 2) {
                const uint2 qb = add_one_rm_bits(fma_sat(z[t], m[t], 0.5f),
                                                 fma_sat(z[t + 1], m[t + 1], 0.5f));
                D[t] = qb.x * G + *reinterpret_cast<const uint32_t *>(tbl_lane + ((qb.x >> F) << TSH));
                D[t + 1] = qb.y * G + *reinterpret_cast<const uint32_t *>(tbl_lane + ((qb.y >> F) << TSH));
            }
            return make_uint2(prmt(prmt(D[0], D[1], 0x0073), prmt(D[2], D[3], 0x7300), 0x7610),
                              prmt(prmt(D[4], D[5], 0x0073), prmt(D[6], D[7], 0x7300), 0x7610));
        };
        uint32_t q = 0;
        int k = 0;
        bool stop = false;
        for (long long ti = blockIdx.x; ti < ntiles && !stop; ti += gridDim.x, ++k) {
            const int b = k & 1;
            bool ok = mbar_wait(norm_ready(b), (k >> 1) & 1);
            ok = ok && (k < 2 || mbar_wait(codes_free(b), ((k >> 1) & 1) ^ 1));
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (lane == 0 && !ok)
                    give_up(TC_ERR_NORM);
                break;
            }
            float m[NT];
#pragma unroll
            for (int j = 0; j < NT; ++j)
                m[j] = scale_s[b * NT + j];
            __syncwarp();
            if (lane == 0)
                mbar_arrive(norm_free(b));
            unsigned char *ctile = basep + (sCodes - base) + (size_t)b * NT * d;
            for (int g = 0; g < nseg; ++g, ++q) {
                const int s = q % TSLOTS;
                const bool okc = mbar_wait(tfull(s), (q / TSLOTS) & 1);
                if (!__all_sync(0xffffffffu, okc)) {
                    if (lane == 0)
                        give_up(TC_ERR_ACC);
                    stop = true;
                    break;
                }
                tc_fence_after();
                const int cnt = seg_chunks(g);
                const uint32_t t_base =
                    tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(H_COLS + s * SEG_N);
                // this warp's chunks of the segment: j_i = par + 2 i (pairs: j_i = 2 par + 4 i,
                // with partner j_i + 1); indices are compile-time so the values stay in registers
                uint32_t acc[4][8], acc2[2][8];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = pairs ? 2 * par + 4 * i : par + 2 * i;
                    if ((!pairs || i < 2) && j < cnt) {               // warp-uniform
                        tmem_ld8_nowait(t_base + (uint32_t)(8 * j), acc[i]);
                        if (pairs && i < 2)
                            tmem_ld8_nowait(t_base + (uint32_t)(8 * (j + 1)), acc2[i & 1]);
                    }
                }
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(tempty(s));
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int j = pairs ? 2 * par + 4 * i : par + 2 * i;
                    if (!((!pairs || i < 2) && j < cnt))
                        continue;
                    const int c = g * SEG + j;
                    // code tile layout [position][token]: 8 bytes per rotated position, the
                    // position swizzled within its group of 32 (see swz) for the packer's reads
                    uint2 *dst = reinterpret_cast<uint2 *>(ctile) + swz(c * 128 + pos);
                    float z[NT];
                    if (!pairs) {
#pragma unroll
                        for (int t = 0; t < NT; ++t)
                            z[t] = __uint_as_float(acc[i][t]);
                        dst[0] = codes8(z, m);
                    } else if (i < 2) {
                        float z2[NT];
#pragma unroll
                        for (int t = 0; t < NT; ++t) {
                            const float u = __uint_as_float(acc[i][t]);
                            const float v = __uint_as_float(acc2[i & 1][t]);
                            z[t] = u + v;
                            z2[t] = u - v;
                        }
                        dst[0] = codes8(z, m);
                        reinterpret_cast<uint2 *>(ctile)[swz((c + 1) * 128 + pos)] = codes8(z2, m);
                    }
                }
            }
            if (stop)
                break;
            // every code byte of the tile is in shared memory once all epilogue warps arrive
            __syncwarp();
            if (lane == 0)
                mbar_arrive(codes_done(b));
            if (!__all_sync(0xffffffffu, mbar_wait(codes_done(b), (k >> 1) & 1))) {
                if (lane == 0)
                    give_up(TC_ERR_CODES);
                break;
            }
            // pack: task = (token half th, 32 consecutive positions).  The 32 positions' words
            // for tokens 4 th .. 4 th + 3 (one word per position, token t in byte t % 4) are
            // transposed 4 x 4 bytes at a time into 8 words per token (byte k = position
            // 4 w + k), the layout pack32 takes.
            const long long t0 = ti * NT;
            const int groups = d / 32;
            const uint32_t *cw = reinterpret_cast<const uint32_t *>(ctile);
            for (int task = e * 32 + lane; task < 2 * groups; task += kEpiWarps * 32) {
                const int gi = task >> 1, th = task & 1;
                uint32_t col[4][8];                       // [token][word]
#pragma unroll
                for (int w = 0; w < 8; ++w) {
                    uint32_t a4[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k)
                        a4[k] = cw[swz(gi * 32 + 4 * w + k) * 2 + th];
                    // bytes: a4[k] = (t0, t1, t2, t3) of position 4 w + k
                    const uint32_t lo01 = prmt(a4[0], a4[1], 0x5140), hi01 = prmt(a4[0], a4[1], 0x7362);
                    const uint32_t lo23 = prmt(a4[2], a4[3], 0x5140), hi23 = prmt(a4[2], a4[3], 0x7362);
                    col[0][w] = prmt(lo01, lo23, 0x5410);
                    col[1][w] = prmt(lo01, lo23, 0x7632);
                    col[2][w] = prmt(hi01, hi23, 0x5410);
                    col[3][w] = prmt(hi01, hi23, 0x7632);
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int t = 4 * th + j;
                    if (t0 + t >= p.T)
                        continue;
                    uint32_t w[BITS];
                    pack32<BITS>(col[j], w);
                    store_packed<BITS>(p.codes + (t0 + t) * row_bytes + gi * 4 * BITS, w);
                }
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(codes_free(b));
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(TMEM_COLS) : "memory");
    }
}

}  // namespace

size_t k1_tc_smem(int d, int tbl_words) {
    const size_t rs = 2 * (size_t)d + 16;
    size_t b = 1024 + (size_t)RING * B_SEG + 2 * NT * rs + 2 * NT * (size_t)d + 2 * (size_t)d +
               4 * (size_t)tbl_words + 2 * NT * 4 + 8;
    b += 8 * (size_t)kNumBars + 16;
    return b;
}

// dynamic shared memory a CTA may take: 227 KB minus room for the kernel's static variables
constexpr size_t kMaxDynSmem = 227 * 1024 - 256;

bool k1_tc_supported(int d, int h, int bits, int tbl_words) {
    return d >= 128 && d % 128 == 0 && d <= 8192 && (h == 32 || h == 64 || h == 128 || h == 256) &&
           (bits == 2 || bits == 3 || bits == 4 || bits == 6 || bits == 8) &&
           k1_tc_smem(d, tbl_words) <= kMaxDynSmem;
}

cudaError_t launch_k1_tc(const K1TcParams &p, int bits, cudaStream_t st, int num_sms,
                         std::string *why) {
    const size_t smem = k1_tc_smem(p.d, p.tbl_words);
    auto go = [&](auto kern) -> cudaError_t {
        // per device and instantiation: the largest dynamic shared memory set so far
        static std::mutex mu;
        static size_t set_to[kMaxDevices][9] = {};
        int dev = 0;
        cudaError_t e = cudaGetDevice(&dev);
        if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices))
            e = cudaErrorInvalidDevice;
        if (e == cudaSuccess) {
            std::lock_guard<std::mutex> lk(mu);
            if (set_to[dev][bits] < smem) {
                e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
                if (e == cudaSuccess)
                    set_to[dev][bits] = smem;
            }
        }
        if (e != cudaSuccess) {
            *why = "cudaFuncSetAttribute(k1_tc)";
            return e;
        }
        const long long ntiles = ((long long)p.T + NT - 1) / NT;
        const int grid = (int)(ntiles < num_sms ? ntiles : num_sms);
        kern<<<grid, kThreads, smem, st>>>(p);
        e = cudaGetLastError();
        if (e != cudaSuccess)
            *why = "k1_tc launch";
        return e;
    };
    switch (bits) {
        case 2: return go(k1_tc<2>);
        case 3: return go(k1_tc<3>);
        case 4: return go(k1_tc<4>);
        case 6: return go(k1_tc<6>);
        case 8: return go(k1_tc<8>);
        default: *why = "unsupported bit width"; return cudaErrorInvalidValue;
    }
}

cudaError_t read_and_clear_k1tc_error(unsigned *out, cudaStream_t st) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_k1tc_err, sizeof(unsigned), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_k1tc_err, &zero, sizeof(unsigned), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace oq
