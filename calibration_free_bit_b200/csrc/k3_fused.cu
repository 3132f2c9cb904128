// k3_fused.cu -- the online step y = W_hat x_hat in one persistent kernel: the rotate +
// norm + quantize stage and the codebook GEMM run side by side on every SM.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video": pseudocode
// block, online per-token part (x_rot = x R^T, s = norm(x_rot), codes of x_rot / (s + eps)),
// and rotation-cancellation paragraph (the codes of R x and of R w meet directly, y = s rn
// sum_k Ca[xc] Cw[wc]); its speed-caveat paragraph names a fused kernel as the missing piece.
//
// B200 design.  The GEMM of the step leaves most of an SM's issue slots idle (one thread
// issues the tcgen05 MMAs, one the TMA loads; four epilogue warps drain each accumulator),
// while the quantize stage is bound by issue and latency.  Every CTA therefore holds both:
//   * warps 0..5: the CTA-pair GEMM of k2_linear.cu (256 x 256 tiles, cta_group::2, a 4-stage
//     TMA ring, two TMEM accumulators, TMA-store epilogue), with tiles taken in row-block order
//     from a global counter by the pair's leader and passed to both CTAs through a small ring
//     of tile ids in shared memory;
//   * warps 6..: one or two groups of d/32 threads running the quantize stage of
//     k1_rotquant.cu on token pairs taken from a global counter, writing each code's fp16
//     unit centroid into the GEMM's A operand and the norms s, and publishing, per block of
//     256 rows, how many rows are done (release add at GPU scope after a proxy fence);
//   * first of all, the GEMM warps decode the 2- or 4-bit weight codes into the fp16 B operand
//     (a static share a warp, one proxy fence and one count a warp; the producers wait for the
//     count once), and then, as ramp groups of d/32 threads with their buffers in the stage
//     ring, quantize a few token pairs each before they take up their GEMM roles.
// A GEMM producer loads a tile's A rows only once their block's count is complete (acquire
// load, then a proxy fence before the TMA); the epilogue acquires the same count before it
// reads s.  The quantize groups never wait on the GEMM, and any CTA's group can take any
// pair, so every wait ends however many CTAs are resident.  Weight codes of other widths are
// decoded into fp16 B by the decode prepass on the same stream before the kernel.
// Every wait is bounded; a wait that gives up sets a bit in the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>
#include <type_traits>

#include "decode4.cuh"
#include "k1_ops.cuh"
#include "oq_internal.h"
#include "sm100_common.cuh"

namespace oq {
namespace {

using namespace sm100;
using namespace k1ops;

__device__ unsigned int g_k3_err;

enum : unsigned {
    K3_ERR_STAGE = 1u << 0,       // a GEMM stage or accumulator wait gave up
    K3_ERR_ROWS = 1u << 1,        // a wait for quantized rows gave up
    K3_ERR_TILE = 1u << 2,        // a wait for a tile id or its release gave up
    K3_ERR_COPY = 1u << 3,        // a quantize-stage bulk copy did not complete
    K3_ERR_ARMED = 1u << 4,       // the armed test wait (oq_debug_arm_wait_timeout) gave up
};

constexpr int kE = 32;                  // rotated positions per quantize thread
constexpr int kMaxSeg = 18;             // warps of a quantize group (d <= 4096: 4)
constexpr int kBK = 64;                 // k-block of the GEMM
constexpr int kS = 4;                   // GEMM stages
constexpr int kTileRing = 4;            // slots of the tile-id ring
constexpr int kAB = 128 * kBK * 2;      // this CTA's 128 rows of A (or B) per k-block: 16 KB
constexpr int kOut = 32 * 32 * 4;       // one epilogue staging chunk
constexpr int kEpi = 4;
constexpr int kGemmThreads = 32 * (2 + kEpi);
constexpr int kMaxGroups = 2;                        // quantize groups per CTA
constexpr int kMaxThreads = kGemmThreads + kMaxGroups * 128;   // groups of d/32 <= 128
constexpr uint32_t kIdesc = idesc_f16(256, 256);
constexpr long long kWaitCycles = 4000000000ll;


__device__ __forceinline__ unsigned ld_acquire(const unsigned *p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void red_release_add(unsigned *p, unsigned v) {
    asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

constexpr int kDecBatch = 16;            // weight-code words a lane holds at once

// The GEMM warps' first task: warp wi of nw decodes its static share of the 2- or 4-bit weight
// codes into the fp16 B operand, kDecBatch words a lane per batch with all of a batch's loads
// issued before its stores, then one proxy fence and one release count (for the TMA reads of
// B).
__device__ __forceinline__ void decode_weight_share(const FusedStepParams &p, int lane,
                                                    long long wi, long long nw) {
    const long long per = (p.wdec_words + nw - 1) / nw;
    const long long lo = wi * per;
    const long long hi = min(p.wdec_words, lo + per);
    for (long long b = lo; b < hi; b += 32 * kDecBatch) {
        uint32_t wv[kDecBatch];
#pragma unroll
        for (int j = 0; j < kDecBatch; ++j) {
            const long long i = b + j * 32 + lane;
            wv[j] = i < hi ? __ldg(p.wcodes + i) : 0u;
        }
#pragma unroll
        for (int j = 0; j < kDecBatch; ++j) {
            const long long i = b + j * 32 + lane;
            if (i >= hi)
                continue;
            if (p.wdec_bits == 4) {
                uint32_t o[4];
                decode8(wv[j], p.wdec_src[0], p.wdec_src[1], p.wdec_src[2], p.wdec_src[3], o);
                p.b16[i] = make_uint4(o[0], o[1], o[2], o[3]);
            } else {                                   // 2-bit: a byte = 4 centroids
                const uint2 q0 = __ldg(p.wdec_tab + (wv[j] & 0xffu));
                const uint2 q1 = __ldg(p.wdec_tab + ((wv[j] >> 8) & 0xffu));
                const uint2 q2 = __ldg(p.wdec_tab + ((wv[j] >> 16) & 0xffu));
                const uint2 q3 = __ldg(p.wdec_tab + (wv[j] >> 24));
                p.b16[2 * i] = make_uint4(q0.x, q0.y, q1.x, q1.y);
                p.b16[2 * i + 1] = make_uint4(q2.x, q2.y, q3.x, q3.y);
            }
        }
    }
    fence_proxy_async_global();
    __syncwarp();
    if (lane == 0)
        red_release_add(p.ctr + 3, 1u);
}

// Wait until all nw decoding warps have counted themselves (no wait when the weights were
// decoded before the launch); false after the wait limit.
__device__ __forceinline__ bool wait_weights(const FusedStepParams &p, unsigned nw) {
    if (p.wdec_words == 0 || ld_acquire(p.ctr + 3) >= nw)
        return true;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(256);
        if (ld_acquire(p.ctr + 3) >= nw)
            return true;
        if (clock64() - t0 > kWaitCycles)
            return false;
    }
}

// Wait until the rows of 256-row block b are all quantized; false after the wait limit.
__device__ __forceinline__ bool wait_rows(const FusedStepParams &p, int b) {
    const unsigned need = (unsigned)min(256, p.T - 256 * b);
    const unsigned *c = p.ctr + 4 + b;
    if (ld_acquire(c) >= need)
        return true;
    const long long t0 = clock64();
    for (;;) {
        __nanosleep(256);
        if (ld_acquire(c) >= need)
            return true;
        if (clock64() - t0 > kWaitCycles)
            return false;
    }
}

// One quantize group's working memory: norm partials (two rounds), barriers ([0] the row
// stage, [1] the table images (the first permanent group's), [2] the armed test wait), pair
// scheduling words, the raw rows of a pair and the interleaved pair.
struct QGroup {
    float2 *red;
    unsigned long long *bars;
    int *sched;
    unsigned char *raw;
    unsigned char *pairs;
};
constexpr size_t kQSmallBytes = sizeof(float2) * 2 * kMaxSeg + 8 * 4 + 4 * 8;

// The quantize stage of one group of GT = d/32 threads (g = 0 .. GT-1, named barrier bar_id):
// token pairs from the global counter -> fp16 A rows and s, each finished pair's rows counted
// in its 256-row block (proxy fence, then release add).  At most max_rounds pairs; on its last
// round the group takes no further pair, so no copy is in flight when it returns.
template <int BITS, int H>
__device__ __forceinline__ void quantize_rounds(const FusedStepParams &p, const QGroup &q, int g,
                                                int GT, int bar_id, const uint32_t *table,
                                                const uint32_t *gent, const uint32_t *dect,
                                                uint32_t setup_bar, int max_rounds) {
    constexpr int Q = H / kE;                        // threads per h-block
    constexpr int TSH = BITS <= 4 ? 7 : 2;           // per-lane table copies for <= 4 bits
    constexpr int NW = kE * BITS / 32;
    const int lane = (int)threadIdx.x & 31;
    const int d = p.d;
    const uint32_t row_in = (uint32_t)d * 2;
    const long long npairs = ((long long)p.T + 1) / 2;
    auto group_sync = [&]() {
        asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(GT) : "memory");
    };
    const uint32_t row_bar = smem_u32(&q.bars[0]);
    const int r = g % Q;
    const int pos0 = g * kE;
    const uint4 *myent = reinterpret_cast<const uint4 *>(gent + g * kK1EntStride);
    const uint32_t tbl_lane = smem_u32(table) + (BITS <= 4 ? lane * 4 : 0) -
                              ((0x3F800000u >> p.F) << TSH);
    const uint32_t G = (uint32_t)p.G;
    const int F = p.F;
    const int seg_end = min(32, lane + (GT - g));
    const bool seg_head = lane == 0;
    const int seg_slot = g >> 5;
    const int nslots = (GT + 31) >> 5;
    // the two rows of pair pr into the raw stage (the group's first thread issues)
    auto issue = [&](long long pr) {
        if (g != 0 || pr >= npairs)
            return;
        const long long t0 = 2 * pr;
        const bool two = t0 + 1 < p.T;
        mbar_expect_tx(row_bar, two ? 2 * row_in : row_in);
        bulk_copy(smem_u32(q.raw), p.x + t0 * row_in, row_in, row_bar);
        if (two)
            bulk_copy(smem_u32(q.raw) + row_in, p.x + (t0 + 1) * row_in, row_in, row_bar);
    };
    if (g == 0) {
        const int first = max_rounds > 0 ? (int)atomicAdd(p.ctr + 0, 1u) : (int)npairs;
        q.sched[0] = first;
        issue(first);
    }
    if (!mbar_wait(setup_bar, 0))
        atomicOr(&g_k3_err, K3_ERR_COPY);
    group_sync();
    long long pr = q.sched[0];
    // Rows of a round are published one round later: the proxy fence that must precede
    // the count then finds the stores long done instead of waiting for them.
    int pend_block = -1;
    unsigned pend_rows = 0;
    for (int round = 0; pr < npairs; ++round) {
        bool valid = true;
        if (!mbar_wait(row_bar, (uint32_t)round & 1u)) {
            atomicOr(&g_k3_err, K3_ERR_COPY);
            valid = false;
        }
        const long long t0 = 2 * pr, t1 = t0 + 1;
        const bool has1 = valid && t1 < p.T;
        // ---- interleave the staged rows into the pair buffer ----
        if (valid) {
            const uint4 *r0 = reinterpret_cast<const uint4 *>(q.raw);
            const uint4 *r1 = reinterpret_cast<const uint4 *>(q.raw + row_in);
            uint4 *slots = reinterpret_cast<uint4 *>(q.pairs);
            const uint4 sl = myent[kE / 4];
            const uint32_t slw[4] = {sl.x, sl.y, sl.z, sl.w};
#pragma unroll
            for (int k = 0; k < kE / 8; ++k) {
                const int c = g + k * GT;
                const uint4 a = r0[c], b = r1[c];
                slots[slw[k] & 0xffffu] =
                    make_uint4(prmt_b32(a.x, b.x, 0x5410), prmt_b32(a.x, b.x, 0x7632),
                               prmt_b32(a.y, b.y, 0x5410), prmt_b32(a.y, b.y, 0x7632));
                slots[slw[k] >> 16] =
                    make_uint4(prmt_b32(a.z, b.z, 0x5410), prmt_b32(a.z, b.z, 0x7632),
                               prmt_b32(a.w, b.w, 0x5410), prmt_b32(a.w, b.w, 0x7632));
            }
        }
        group_sync();
        if (pend_rows)
            fence_proxy_async_global();            // the previous round's rows
        // the raw stage is free: take the next pair (none after the last allowed round) and
        // start its copy
        if (g == 0) {
            const int nx = round + 1 < max_rounds ? (int)atomicAdd(p.ctr + 0, 1u) : (int)npairs;
            q.sched[1 + (round & 1)] = nx;
            issue(nx);
        }
        // ---- gather y[i] = sign[i] x[perm[i]] for both tokens ----
        float2 v[kE];
        {
            const uint32_t base0 = smem_u32(q.pairs);
#pragma unroll
            for (int e4 = 0; e4 < kE / 4; ++e4) {
                const uint4 q4 = myent[e4];
                const uint32_t en4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t en = en4[i];
                    const uint32_t sg = en & 0x80000000u;
                    const uint32_t w = lds32(base0 + (en & 0x7fffffffu));
                    v[4 * e4 + i].x = __uint_as_float((w << 16) + sg);
                    v[4 * e4 + i].y = __uint_as_float((w ^ en) & 0xffff0000u);
                }
            }
        }
        // ---- block Walsh-Hadamard (natural order), unnormalised ----
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
            const float sgn = (r & m) ? -1.0f : 1.0f;
            const float2 sg2 = make_float2(sgn, sgn);
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                float2 o;
                o.x = __shfl_xor_sync(0xffffffffu, v[e].x, m);
                o.y = __shfl_xor_sync(0xffffffffu, v[e].y, m);
                v[e] = f2fma(sg2, v[e], o);
            }
        }
        // ---- per-token sum of squares over the group ----
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < kE; ++e)
            acc = f2fma(v[e], v[e], acc);
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            float2 o;
            o.x = __shfl_down_sync(0xffffffffu, acc.x, off);
            o.y = __shfl_down_sync(0xffffffffu, acc.y, off);
            if (lane + off < seg_end) {
                acc.x += o.x;
                acc.y += o.y;
            }
        }
        if (seg_head)
            q.red[(round & 1) * kMaxSeg + seg_slot] = acc;
        group_sync();
        if (g == 0 && pend_rows)
            red_release_add(p.ctr + 4 + pend_block, pend_rows);
        const float2 *myred = q.red + (round & 1) * kMaxSeg;
        const long long nxt = q.sched[1 + (round & 1)];
        float2 ss = myred[0];
        for (int i = 1; i < nslots; ++i) {
            const float2 o = myred[i];
            ss.x += o.x;
            ss.y += o.y;
        }
        const float s0 = sqrtf(ss.x * (1.0f / H));
        const float s1 = sqrtf(ss.y * (1.0f / H));
        const float m0 = (s0 + p.eps > 0.f) ? p.K / (s0 + p.eps) : 0.f;
        const float m1 = (s1 + p.eps > 0.f) ? p.K / (s1 + p.eps) : 0.f;
        // ---- nearest centroid, packed codes in registers ----
        uint32_t w0[NW], w1[NW];
        {
            constexpr int PER = 32 / BITS;
#pragma unroll
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t d0[PER], d1[PER];
#pragma unroll
                for (int k = 0; k < PER; ++k) {
                    const float2 vv = v[wi * PER + k];
                    const float a0 = fma_sat(vv.x, m0, 0.5f);
                    const float a1 = fma_sat(vv.y, m1, 0.5f);
                    const uint2 qb = f2_add_one_rm_bits(a0, a1);
                    d0[k] = qb.x * G + lds32(tbl_lane + ((qb.x >> F) << TSH));
                    d1[k] = qb.y * G + lds32(tbl_lane + ((qb.y >> F) << TSH));
                }
                w0[wi] = pack_codes<BITS>(d0);
                w1[wi] = pack_codes<BITS>(d1);
            }
        }
        // ---- fp16 centroids into the A operand, norms, then publish the rows ----
        if (valid) {
            uint4 *a0 = reinterpret_cast<uint4 *>(p.a16 + t0 * d + pos0);
            decode_store<BITS>(dect, w0, a0, p.dec_src);
            if (has1)
                decode_store<BITS>(dect, w1, a0 + d / 8, p.dec_src);
            if (g == 0) {
                p.s[t0] = s0;
                if (has1)
                    p.s[t1] = s1;
            }
        }
        pend_block = (int)(t0 / 256);
        pend_rows = valid ? (has1 ? 2u : 1u) : 0u;
        if (round == 0 && pend_rows) {
            // the first rows open the GEMM's first tiles: publish them at once
            fence_proxy_async_global();
            group_sync();
            if (g == 0)
                red_release_add(p.ctr + 4 + pend_block, pend_rows);
            pend_rows = 0;
        }
        pr = nxt;
    }
    if (pend_rows) {                             // the last round's rows
        fence_proxy_async_global();
        group_sync();
        if (g == 0)
            red_release_add(p.ctr + 4 + pend_block, pend_rows);
    }
}

// one epilogue staging chunk per warp (the stores of a tile overlap the next tile's mainloop
// through the second TMEM accumulator, so a second staging buffer buys little here and its
// 16 KB go to a second quantize group)
__host__ __device__ constexpr size_t gemm_bytes() {
    return (size_t)kS * 2 * kAB + (size_t)kEpi * kOut;
}

// shared memory: [GEMM stages + staging: 1 KB aligned][GEMM barriers][scalars, ring, norms]
// [quantize: table | entries | decode table | partials | barriers | sched | raw rows | pairs]
constexpr int kGemmBars = 2 * kS + 5 + 2 * kTileRing + 1;   // + the ramp barrier
constexpr size_t kBarsBytes = (8 * kGemmBars + 15) & ~(size_t)15;
// scalars: TMEM base and abort flag (16 bytes), the tile-id ring, then the epilogue's
// row-norm chunks (read as float4: 16-byte aligned), then the small regions of the ramp
// groups (their rows and pairs live in the GEMM's stage ring until the ramp ends)
constexpr int kMaxRamp = kGemmThreads / 32;
constexpr size_t kRnOffset = 16 + ((4 * kTileRing + 15) & ~(size_t)15);
constexpr size_t kRampOffset = kRnOffset + kEpi * 64 * 4;
constexpr size_t kMiscBytes = kRampOffset + kMaxRamp * kQSmallBytes;
static_assert(kBarsBytes % 16 == 0 && kRnOffset % 16 == 0 && kRampOffset % 16 == 0 &&
              kQSmallBytes % 16 == 0 && kMiscBytes % 16 == 0, "16-byte aligned regions");

// Ramp groups: before their GEMM roles, the GEMM warps form groups of d/32 threads that
// quantize a few token pairs each (the GEMM's first wave needs many row blocks at once), with
// their rows and pairs in the stage ring (8d bytes a group).
__host__ __device__ inline int ramp_groups(int d, int ramp_rounds) {
    const int gt = d / kE;
    if (ramp_rounds <= 0 || gt > kGemmThreads)
        return 0;
    const int by_threads = kGemmThreads / gt;
    const int by_ring = (int)(((size_t)kS * 2 * kAB) / ((size_t)8 * d));
    return by_threads < by_ring ? by_threads : by_ring;
}

// per group: norm partials (two rounds), 4 barriers, 8 scheduling words, raw rows, pairs
size_t quant_group_bytes(int d) {
    return sizeof(float2) * 2 * kMaxSeg + 8 * 4 + 4 * 8 + (size_t)2 * d * 2 + (size_t)d * 4;
}

size_t quant_bytes(const FusedStepParams &p, int groups) {
    return 4 * (size_t)(p.tbl_words + p.ent_words + p.dec_words) +
           (size_t)groups * quant_group_bytes(p.d);
}

size_t fused_smem(const FusedStepParams &p, int groups) {
    // up to 1023 bytes of alignment, the GEMM region, its barriers, the scalars, the quantize
    // region (the kernel's layout, in that order)
    return 1024 + gemm_bytes() + kBarsBytes + kMiscBytes + quant_bytes(p, groups) + 64;
}

template <int BITS, int H, bool BF16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kMaxThreads, 1)
    k3_fused(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
             const __grid_constant__ CUtensorMap tmY, const FusedStepParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_addr = smem_u32(smem_raw);
    const uint32_t base = (raw_addr + 1023u) & ~1023u;
    unsigned char *basep = smem_raw + (base - raw_addr);
    const uint32_t sA = base, sB = base + kS * kAB;
    const uint32_t sOut = sB + kS * kAB;
    const uint32_t bars = sOut + kEpi * kOut;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (kS + s); };
    auto tfull_bar = [&](int a) { return bars + 8u * (2 * kS + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (2 * kS + 2 + a); };
    const uint32_t drain_bar = bars + 8u * (2 * kS + 4);
    auto idfull_bar = [&](int r) { return bars + 8u * (2 * kS + 5 + r); };
    auto idempty_bar = [&](int r) { return bars + 8u * (2 * kS + 5 + kTileRing + r); };
    const uint32_t ramp_bar = bars + 8u * (2 * kS + 5 + 2 * kTileRing);
    unsigned char *miscp = basep + (bars + (uint32_t)kBarsBytes - base);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(miscp);
    int *abort_flag = reinterpret_cast<int *>(miscp + 4);
    int *ring = reinterpret_cast<int *>(miscp + 16);
    const uint32_t ring_addr = smem_u32(ring);
    float *rn_s = reinterpret_cast<float *>(miscp + kRnOffset);
    unsigned char *rampsmall = miscp + kRampOffset;
    unsigned char *qbase = miscp + kMiscBytes;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int n_tiles = (p.N + 255) / 256;
    const int num_tiles = ((p.T + 255) / 256) * n_tiles;
    const int num_kb = p.d / kBK;
    const int GT = p.d / kE;
    const int NQ = ((int)blockDim.x - kGemmThreads) / GT;     // quantize groups
    const int qgrp = threadIdx.x >= kGemmThreads ? ((int)threadIdx.x - kGemmThreads) / GT : 0;
    const int NR = ramp_groups(p.d, p.ramp_rounds);           // ramp groups
    auto ramp_group = [&](int rg) {
        unsigned char *sm = rampsmall + (size_t)rg * kQSmallBytes;
        float2 *rred = reinterpret_cast<float2 *>(sm);
        unsigned long long *rbars = reinterpret_cast<unsigned long long *>(rred + 2 * kMaxSeg);
        int *rsched = reinterpret_cast<int *>(rbars + 4);
        unsigned char *rraw = basep + (sA - base) + (size_t)rg * 8 * p.d;
        return QGroup{rred, rbars, rsched, rraw, rraw + (size_t)4 * p.d};
    };

    // quantize-stage shared memory: shared tables, then one region per group
    uint32_t *table = reinterpret_cast<uint32_t *>(qbase);
    uint32_t *gent = table + p.tbl_words;
    uint32_t *dect = gent + p.ent_words;
    unsigned char *qg = reinterpret_cast<unsigned char *>(dect + p.dec_words) +
                        (size_t)qgrp * (sizeof(float2) * 2 * kMaxSeg + 8 * 4 + 4 * 8 +
                                        (size_t)2 * p.d * 2 + (size_t)p.d * 4);
    float2 *red = reinterpret_cast<float2 *>(qg);
    unsigned long long *qbars = reinterpret_cast<unsigned long long *>(red + 2 * kMaxSeg);
    int *qsched = reinterpret_cast<int *>(qbars + 4);
    unsigned char *qraw = reinterpret_cast<unsigned char *>(qsched + 8);
    unsigned char *qpairs = qraw + (size_t)2 * p.d * 2;
    // the table images land once per CTA, on group 0's setup barrier
    unsigned long long *qbars0 = reinterpret_cast<unsigned long long *>(
        reinterpret_cast<unsigned char *>(dect + p.dec_words) + sizeof(float2) * 2 * kMaxSeg);
    const uint32_t setup_bar = smem_u32(&qbars0[1]);

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < kS; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 2 * kEpi);
        }
        mbar_init(drain_bar, 1);
        for (int r = 0; r < kTileRing; ++r) {
            mbar_init(idfull_bar(r), 1);
            // releases of a tile id: the leader's MMA thread and epilogue warps, the peer's
            // producer and epilogue warps
            mbar_init(idempty_bar(r), 1 + kEpi + 1 + kEpi);
        }
        for (int q = 0; q < NQ; ++q) {
            unsigned long long *b = reinterpret_cast<unsigned long long *>(
                reinterpret_cast<unsigned char *>(dect + p.dec_words) +
                (size_t)q * (sizeof(float2) * 2 * kMaxSeg + 8 * 4 + 4 * 8 +
                             (size_t)2 * p.d * 2 + (size_t)p.d * 4) +
                sizeof(float2) * 2 * kMaxSeg);
            mbar_init(smem_u32(&b[0]), 1);         // the group's row stage
            mbar_init(smem_u32(&b[1]), 1);         // table images (group 0's)
            mbar_init(smem_u32(&b[2]), 2);         // armed test wait (group 0's)
        }
        for (int q = 0; q < NR; ++q)
            mbar_init(smem_u32(&ramp_group(q).bars[0]), 1);   // a ramp group's row stage
        mbar_init(ramp_bar, NR > 0 ? NR : 1);               // every ramp group is done
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        *abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(512) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                 // x, the fp16 weight operand, rn and the counters are ready
    auto aborted = [&]() { return *(volatile int *)abort_flag != 0; };
    auto give_up = [&](unsigned bit) {
        atomicOr(&g_k3_err, bit);
        atomicExch(abort_flag, 1);
    };

    // ---------------- ramp (the GEMM warps, before their roles) ----------------
    // Every GEMM warp decodes a share of the 2/4-bit weight codes.  The warps of the ramp
    // groups then quantize up to ramp_rounds token pairs a group with their rows and pairs in
    // the stage ring, order their shared-memory accesses before the async proxy's, and count
    // their group on ramp_bar; the producers wait for it before their first TMA load.
    if (warp < 2 + kEpi) {
        if (p.wdec_words > 0)
            decode_weight_share(p, lane, (long long)blockIdx.x * (2 + kEpi) + warp,
                                (long long)gridDim.x * (2 + kEpi));
        if ((int)threadIdx.x < NR * GT) {
            const int rg = (int)threadIdx.x / GT, g = (int)threadIdx.x - rg * GT;
            const int bar_id = 1 + kMaxGroups + rg;
            quantize_rounds<BITS, H>(p, ramp_group(rg), g, GT, bar_id, table, gent, dect,
                                     setup_bar, p.ramp_rounds);
            fence_async_smem();
            asm volatile("bar.sync %0, %1;" ::"r"(bar_id), "r"(GT) : "memory");
            if (g == 0)
                mbar_arrive(ramp_bar);
        }
    }

    if (warp == 0) {
        // ---------------- tile scheduler (leader) and TMA producer (both CTAs) -------------
        if (lane == 0) {
            uint32_t it = 0;
            if (NR > 0 && !mbar_wait(ramp_bar, 0))
                give_up(K3_ERR_STAGE);             // the ring may still be in use: load nothing
            for (int i = 0;; ++i) {
                const int r = i % kTileRing;
                const uint32_t par = (uint32_t)(i / kTileRing) & 1u;
                int tile;
                if (rank == 0) {
                    if (i >= kTileRing && !mbar_wait(idempty_bar(r), par ^ 1u)) {
                        give_up(K3_ERR_TILE);
                        tile = num_tiles;
                    } else {
                        tile = aborted() ? num_tiles : (int)atomicAdd(p.ctr + 1, 1u);
                    }
                    if (tile > num_tiles)
                        tile = num_tiles;
                    // publish the id in both CTAs' rings
                    ring[r] = tile;
                    asm volatile("st.shared::cluster.u32 [%0], %1;"
                                 ::"r"(mapa_shared(ring_addr + 4u * r, 1)), "r"(tile) : "memory");
                    mbar_arrive(idfull_bar(r));
                    mbar_arrive_cluster(mapa_shared(idfull_bar(r), 1));
                } else {
                    if (!mbar_wait(idfull_bar(r), par)) {
                        give_up(K3_ERR_TILE);
                        break;
                    }
                    tile = ring[r];
                    mbar_arrive_remote(mapa_shared(idempty_bar(r), 0));
                }
                if (tile >= num_tiles)
                    break;
                const int mb = tile / n_tiles;
                const int m0 = mb * 256 + (int)rank * 128;
                const int n0 = (tile % n_tiles) * 256 + (int)rank * 128;
                if ((i == 0 && !wait_weights(p, gridDim.x * (2 + kEpi))) || !wait_rows(p, mb)) {
                    give_up(K3_ERR_ROWS);
                    break;
                }
                fence_proxy_async_global();           // rows written by generic stores
                bool stop = false;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % kS;
                    if (it >= kS && !mbar_wait(empty_bar(s), ((it / kS) & 1) ^ 1)) {
                        give_up(K3_ERR_STAGE);
                        stop = true;
                        break;
                    }
                    if (aborted()) {
                        stop = true;
                        break;
                    }
                    if (rank == 0)
                        mbar_expect_tx(full_bar(s), 4 * kAB);
                    const uint32_t fb = mapa_shared(full_bar(s), 0);
                    tma_load_2d_pair(sA + s * kAB, &tmA, kb * kBK, m0, fb);
                    tma_load_2d_pair(sB + s * kAB, &tmB, kb * kBK, n0, fb);
                }
                if (stop)
                    break;
            }
            if (aborted() && rank == 0) {
                const uint32_t from = it > (uint32_t)kS ? it - kS : 0;
                for (uint32_t j = from; j < it; ++j)
                    mbar_wait(full_bar(j % kS), (j / kS) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader) ----------------
        if (lane == 0 && rank == 0) {
            uint32_t it = 0;
            for (int i = 0;; ++i) {
                const int r = i % kTileRing;
                if (!mbar_wait(idfull_bar(r), (uint32_t)(i / kTileRing) & 1u)) {
                    give_up(K3_ERR_TILE);
                    break;
                }
                const int tile = ring[r];
                mbar_arrive(idempty_bar(r));
                if (tile >= num_tiles || aborted())
                    break;
                const int acc = i & 1;
                if (i >= 2 && !mbar_wait(tempty_bar(acc), ((i >> 1) & 1) ^ 1)) {
                    give_up(K3_ERR_STAGE);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * 256);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % kS;
                    if (!mbar_wait(full_bar(s), (it / kS) & 1)) {
                        give_up(K3_ERR_STAGE);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sw128_desc(sA + s * kAB);
                    const uint64_t db = sw128_desc(sB + s * kAB);
#pragma unroll
                    for (int kk = 0; kk < kBK / 16; ++kk)
                        mma_ss_pair(d_tmem, da + 2 * kk, db + 2 * kk, kIdesc, (kb | kk) != 0);
                    mma_commit_pair_mc(empty_bar(s), 0x3);
                }
                if (!ok)
                    break;
                mma_commit_pair_mc(tfull_bar(acc), 0x3);
            }
            mma_commit_pair_mc(drain_bar, 0x1);
            if (!mbar_wait(drain_bar, 0))
                atomicOr(&g_k3_err, K3_ERR_STAGE);
        }
    } else if (warp < 2 + kEpi) {
        // ---------------- epilogue (both CTAs) ----------------
        const int q = warp & 3;
        float *rn_w = rn_s + (warp - 2) * 64;
        const uint32_t out0 = sOut + (uint32_t)((warp - 2) * kOut);
        unsigned char *out0p = basep + (out0 - base);
        uint32_t u = 0;
        for (int i = 0;; ++i) {
            const int r = i % kTileRing;
            const bool got = mbar_wait(idfull_bar(r), (uint32_t)(i / kTileRing) & 1u);
            if (!__all_sync(0xffffffffu, got)) {
                if (lane == 0)
                    give_up(K3_ERR_TILE);
                break;
            }
            const int tile = ring[r];
            __syncwarp();
            if (lane == 0) {
                if (rank == 0)
                    mbar_arrive(idempty_bar(r));
                else
                    mbar_arrive_remote(mapa_shared(idempty_bar(r), 0));
            }
            if (tile >= num_tiles)
                break;
            const int acc = i & 1;
            const int mb = tile / n_tiles;
            const int m0 = mb * 256 + (int)rank * 128;
            const int n0 = (tile % n_tiles) * 256;
            // acquire the block's row count (every lane) before reading its norms
            if (!__all_sync(0xffffffffu, wait_rows(p, mb))) {
                if (lane == 0)
                    give_up(K3_ERR_ROWS);
                break;
            }
            const int row = m0 + q * 32 + lane;
            const float srow = (row < p.T) ? p.s[row] * p.inv_d : 0.f;
            float rnv[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const int col = n0 + c * 32 + lane;
                rnv[c] = (col < p.N) ? p.rn[col] : 0.f;
            }
            const bool ok = mbar_wait(tfull_bar(acc), (i >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (!ok)
                    give_up(K3_ERR_STAGE);
                break;
            }
            tc_fence_after();
            const uint32_t t_base = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * 256);
            const bool rows_in = m0 + q * 32 < p.T;
            constexpr int kCW = BF16 ? 64 : 32;
#pragma unroll
            for (int c = 0; c < 256 / kCW; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_base + (uint32_t)(c * kCW), r0);
                if constexpr (BF16)
                    tmem_ld32(t_base + (uint32_t)(c * kCW + 32), r1);
                if (!rows_in || n0 + c * kCW >= p.N)
                    continue;
                const uint32_t b = 0;
                if (lane == 0)
                    bulk_wait_read<0>();               // the previous chunk's store has read it
                __syncwarp();
                if constexpr (BF16) {
                    rn_w[lane] = rnv[2 * c];
                    rn_w[32 + lane] = rnv[2 * c + 1];
                } else {
                    rn_w[lane] = rnv[c];
                }
                __syncwarp();
                if constexpr (BF16)
                    store_chunk_bf16(&tmY, out0p + b * kOut, out0 + b * kOut, r0, r1, srow,
                                     rn_w, lane, n0 + c * kCW, m0 + q * 32);
                else
                    store_chunk(&tmY, out0p + b * kOut, out0 + b * kOut, r0, srow, rn_w, lane,
                                n0 + c * kCW, m0 + q * 32);
                ++u;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
        }
        if (lane == 0)
            bulk_wait_all();
    } else {
        // ---------------- permanent quantize group ----------------
        const int g = (int)threadIdx.x - kGemmThreads - qgrp * GT;   // 0 .. GT-1
        if (g == 0 && qgrp == 0) {
            mbar_expect_tx(setup_bar, 4u * (p.tbl_words + p.ent_words + p.dec_words));
            bulk_copy(smem_u32(table), p.tbl_img, 4u * p.tbl_words, setup_bar);
            bulk_copy(smem_u32(gent), p.ent_img, 4u * p.ent_words, setup_bar);
            if (p.dec_words > 0)
                bulk_copy(smem_u32(dect), p.dec_img, 4u * p.dec_words, setup_bar);
        }
        const QGroup qgp{red, qbars, qsched, qraw, qpairs};
        quantize_rounds<BITS, H>(p, qgp, g, GT, 1 + qgrp, table, gent, dect, setup_bar,
                                 0x7fffffff);
        if (p.test_wait_cycles > 0 && blockIdx.x == 0 && g == 0 && qgrp == 0) {
            const uint32_t tb = smem_u32(&qbars[2]);
            mbar_arrive(tb);
            if (!mbar_wait(tb, 0, p.test_wait_cycles))
                atomicOr(&g_k3_err, K3_ERR_ARMED);
        }
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(512) : "memory");
    }
}

// Zeroes the fused step's progress counters once the stream's earlier work is done, as a
// programmatic-launch kernel: it can be resident beside the previous kernel's tail, and the
// fused kernel launched after it sets up while it runs (a memset node would break the chain).
__global__ void __launch_bounds__(256) k3_zero_counters(unsigned *ctr, int n) {
    pdl_trigger();
    pdl_wait();
    for (int i = (int)threadIdx.x; i < n; i += (int)blockDim.x)
        ctr[i] = 0u;
}

}  // namespace

// ------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------
namespace {

template <int BITS, int H, bool BF16>
cudaError_t launch_t(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &my,
                     const FusedStepParams &p, int groups, int pairs, size_t smem,
                     cudaStream_t st, std::string *why) {
    auto kern = k3_fused<BITS, H, BF16>;
    static std::mutex mu;
    static size_t set_to[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices))
        e = cudaErrorInvalidDevice;
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lk(mu);
        if (set_to[dev] < smem) {
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)smem);
            if (e == cudaSuccess)
                set_to[dev] = smem;
        }
    }
    if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(k3_fused)";
        return e;
    }
    const int threads = kGemmThreads + groups * (p.d / kE);
    if (pairs < 1) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(threads, 1, 1);
        cfg.dynamicSmemBytes = smem;
        int n = 0;
        e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
        if (e != cudaSuccess || n < 1) {
            *why = "k3_fused: no CTA pair fits on this device";
            return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        }
        pairs = n;
    }
    const int tiles = ((p.N + 255) / 256) * ((p.T + 255) / 256);
    if (pairs > tiles)
        pairs = tiles;
    e = launch_pdl(kern, dim3(2 * pairs), dim3(threads), smem, st, ma, mb, my, p);
    if (e != cudaSuccess)
        *why = "k3_fused launch";
    return e;
}

}  // namespace

bool fused_step_supported(int d, int h, int bits, bool bf16_in) {
    return bf16_in && (d == 1024 || d == 2048 || d == 3072 || d == 4096) &&
           (h == 64 || h == 128 || h == 256) && (bits == 2 || bits == 4 || bits == 8);
}

cudaError_t launch_zero_counters(unsigned *ctr, int n, cudaStream_t st) {
    return launch_pdl(k3_zero_counters, dim3(1), dim3(256), 0, st, ctr, n);
}

size_t fused_step_counter_words(int T, int N) {
    (void)N;
    return 4 + ((size_t)T + 255) / 256;
}

cudaError_t launch_fused_step(const FusedStepParams &p, int bits, int h, bool y_bf16,
                              const uint16_t *B16, void *y, cudaStream_t st, std::string *why) {
    if (!fused_step_supported(p.d, h, bits, true)) {
        *why = "k3_fused: unsupported shape";
        return cudaErrorInvalidValue;
    }
    // two quantize groups per CTA when they fit beside the GEMM, else one
    int groups = kMaxGroups;
    while (groups > 1 && fused_smem(p, groups) > 227 * 1024)
        --groups;
    const size_t smem = fused_smem(p, groups);
    if (smem > 227 * 1024) {
        *why = "k3_fused: shared memory exceeds the per-CTA limit";
        return cudaErrorInvalidConfiguration;
    }
    CUtensorMap ma, mb, my;
    if (!make_operand_map(&ma, p.a16, p.T, p.d) || !make_operand_map(&mb, B16, p.N, p.d) ||
        !make_out_map(&my, y, p.T, p.N, y_bf16)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int pairs = 0;                   // as many as fit (occupancy query at launch)
    auto pick_h = [&](auto bits_tag, auto bf16_tag) -> cudaError_t {
        constexpr int B = decltype(bits_tag)::value;
        constexpr bool Y16 = decltype(bf16_tag)::value;
        switch (h) {
            case 64: return launch_t<B, 64, Y16>(ma, mb, my, p, groups, pairs, smem, st, why);
            case 128: return launch_t<B, 128, Y16>(ma, mb, my, p, groups, pairs, smem, st, why);
            case 256: return launch_t<B, 256, Y16>(ma, mb, my, p, groups, pairs, smem, st, why);
            default: *why = "k3_fused: h"; return cudaErrorInvalidValue;
        }
    };
    auto pick_bits = [&](auto bf16_tag) -> cudaError_t {
        switch (bits) {
            case 2: return pick_h(std::integral_constant<int, 2>{}, bf16_tag);
            case 4: return pick_h(std::integral_constant<int, 4>{}, bf16_tag);
            case 8: return pick_h(std::integral_constant<int, 8>{}, bf16_tag);
            default: *why = "k3_fused: bit width"; return cudaErrorInvalidValue;
        }
    };
    return y_bf16 ? pick_bits(std::true_type{}) : pick_bits(std::false_type{});
}

cudaError_t read_and_clear_k3_error(unsigned *out, cudaStream_t st) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_k3_err, sizeof(unsigned), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_k3_err, &zero, sizeof(unsigned), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace oq
