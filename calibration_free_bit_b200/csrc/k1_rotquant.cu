// k1_rotquant.cu -- fused RPBH rotate + per-token norm + Lloyd-Max nearest-centroid codes.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video", pseudocode
// block (online per-token part): x_rot = x R^T, s = norm(x_rot),
// codes = nearest_centroid(x_rot / (s + eps), codebook[d, b]); the same kernel with eps = 0
// serves the offline weight step (rows of W, row_norms).  R = blockdiag(H_h/sqrt h) D P is
// the RPBH rotation of the summary's RPBH paragraph, applied as an O(d log h) butterfly.
//
// B200 design (one HBM-bound pass: read 2d bytes per bf16 row, write d*b/8 + 4):
//   * Thread groups of d/32 threads; a group works on one token PAIR at a time, whose two
//     rows stream into shared memory with bulk copies (completing on an mbarrier) one pair
//     ahead of the compute.  bf16 rows whose groups are whole warps, or can be padded to
//     whole warps with at most one lane in eight idle: one CTA per SM, an equal contiguous
//     share of the pairs per CTA, each group on its own named barrier taking its next pair
//     from a shared counter.  Otherwise several smaller CTAs per SM step through the pairs in
//     lockstep rounds.
//   * bf16 rows are interleaved into 32-bit words (x_t0[j], x_t1[j]), so one 4-byte gather
//     load serves both tokens and the butterfly runs on packed fp32x2 (add/sub/fma .f32x2,
//     new on sm_100).  Each half of an 8-element chunk goes to a 16-byte slot the host
//     chose: the eight stores of a quarter-warp cover all banks, and the slots' bank groups
//     are arranged so that the 32 lanes of a random gather meet on fewer banks.
//   * Thread g holds the 32 consecutive rotated positions g*32 .. g*32+31 (h/32 threads per
//     h-block).  Its gather offsets and signs (pair-buffer byte offset of perm[i] | sign<<31)
//     are converted once per CTA into a shared table, padded to 36 words per thread so the
//     16-byte entry loads of a warp are bank-conflict free.
//   * Butterfly: 5 in-register stages, then log2(h/32) shuffle stages across the block's
//     threads.  The per-token sum of squares is reduced across the group (segmented warp
//     shuffles + shared memory); s = sqrt(sum z^2 / h) since z is unnormalised.
//   * Nearest centroid by a uniform-grid table (host-built, <= 1 boundary per cell):
//     a = sat(z*K/(s+eps) + 1/2) (one FFMA.SAT), q = floor(a*2^23) via an fp32x2 add with
//     round-down, word = table[q >> F], code = (word + q*G) >> 24.  The table words fold the
//     cell's base code and its boundary, so the decision is exact in the fixed-point q grid
//     (2^-23 of the grid span, < 1.2e-6 sigma).  Bit widths 2/3/4/6/8 pack LSB-first.
//   * fp16 output (the one-call path): each code's fp16 unit centroid instead of the packed
//     codes (the GEMM's A operand, 32-byte stores); with it, the groups that run out of pairs
//     can decode the layer's 2- or 4-bit weight codes into the GEMM's B operand (each CTA an
//     equal share).
//   * Fused GELU (bf16 rows): GELU of each gathered element from a shared table of all bf16
//     values (k1_ops.cuh, gelu_lookup).
//   * Every mbarrier wait is bounded (about 2 s of SM clock); a wait that gives up sets a bit
//     in the device error word (read by oq_check) and the round's outputs are not written.
#include <cuda_bf16.h>

#include <map>
#include <set>
#include <tuple>

#include <type_traits>

#include "decode4.cuh"
#include "k1_ops.cuh"
#include "oq_internal.h"

namespace oq {
namespace {

using namespace k1ops;

__device__ unsigned int g_k1_err;

constexpr int kE = 32;                // rotated positions per thread (per token)
constexpr int kSmallH = 16;           // template tag of the block sizes 2, 4, 8, 16
constexpr int kMaxSeg = 18;           // segment slots per group for the norm reduction
constexpr int kEntStride = kK1EntStride;   // padded entry rows (conflict-free 16 B loads)
static_assert(kEntStride == kE + 4, "entry image layout");

enum : unsigned {
    K1_ERR_COPY_WAIT = 1u,        // a bulk copy of rows or tables did not complete in time
    K1_ERR_ARMED_WAIT = 2u,       // the armed test wait (oq_debug_arm_wait_timeout) gave up
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t r;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(sel));
    return r;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// A waiting thread may sleep in try_wait up to this long (it wakes when the phase completes).
constexpr unsigned kSuspendHintNs = 200000;

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(bar), "r"(parity), "n"(kSuspendHintNs) : "memory");
    return done != 0;
}

// Wait for the phase of the given parity; false after `limit` SM cycles (by default 4e9,
// about 2 s at the boost clock; the caller records an error).  The first test reads no clock.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity,
                                          long long limit = 4000000000ll) {
    if (mbar_try(bar, parity))
        return true;
    const long long t0 = clock64();
    for (;;) {
        if (mbar_try(bar, parity))
            return true;
        if (clock64() - t0 > limit)
            return false;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

// Per CTA: NG groups of d/32 threads, each group owns one token pair per round.  bf16 input:
// the NEXT round's two rows stream into a raw buffer while the current round computes from
// the interleaved pair buffer.  fp32 input: rows are gathered straight from `stages` raw
// buffers (2 when shared memory allows, else 1).
// GELU (bf16 input only): the kernel quantizes R * GELU(x) instead of R * x; GELU is applied
// to each gathered element before its sign flip (it is elementwise, so it commutes with P).
// A16 (bf16 input, BITS = 2, 4, 8): instead of the packed codes, the kernel writes each code's
// fp16 unit centroid to p.a16 [T, d] (the GEMM's A operand; the codes stay on chip).
// NAMED (bf16 input, groups of whole warps, padded to them where k1_named allows): each group
// synchronises on its own named barrier and takes pairs from a shared counter; the kernel then
// reserves all 16 barriers of the SM's CTA slot, so it is launched one CTA per SM.  Otherwise the CTA synchronises as a whole and
// its groups step through the CTA's pairs in lockstep.
// H = kSmallH stands for every block size below 32 (2, 4, 8, 16): a thread's 32 positions
// then hold 32/h whole blocks, the butterfly stops after log2(h) in-register stages (h read
// from p.h) and no shuffle stage runs.
template <int BITS, bool IN_F32, int H, bool GELU = false, bool A16 = false, bool NAMED = false>
__global__ void __maxnreg__(96) k1_rotquant(const K1Params p) {
    static_assert(!(GELU && IN_F32), "fused GELU is bf16-only");
    static_assert(!(NAMED && IN_F32), "named-barrier groups are bf16-only");
    static_assert(!A16 || (!IN_F32 && (BITS == 2 || BITS == 4 || BITS == 8)), "A16 output");
    static_assert(H >= kE || (H == kSmallH && !A16), "small blocks: one variant, codes out");
    constexpr int Q = H >= kE ? H / kE : 1;          // threads per h-block
    const int hrt = H >= kE ? H : p.h;               // the block size (run time below 32)
    constexpr bool REPL = (BITS <= 4);               // per-lane table copies (conflict-free)
    constexpr int TSH = REPL ? 7 : 2;                // table row stride: 32 lanes x 4 B, or 4 B
    constexpr int NW = kE * BITS / 32;               // packed code words per token per thread
    constexpr int IN_BYTES = IN_F32 ? 4 : 2;

    extern __shared__ __align__(16) unsigned char smem[];
    const int d = p.d;
    const int GT = d / kE;                           // position-owning threads per token pair
    // threads per group: NAMED groups are padded to whole warps, and their padding lanes own
    // no positions (they run the group's steps on a duplicate entry row, take no part in the
    // norm and store nothing)
    const int GTP = NAMED ? ((GT + 31) & ~31) : GT;
    const int NG = p.groups;
    const int nstage = IN_F32 ? p.stages : 1;        // raw row buffers per group
    const int tid = threadIdx.x;
    const int grp = tid / GTP;
    const int g = tid - grp * GTP;
    const bool owns = g < GT;
    const int lane = tid & 31;
    const int warp_start = tid - lane;
    const int active = min(32, (int)blockDim.x - warp_start);
    const unsigned wmask = active == 32 ? 0xffffffffu : ((1u << active) - 1u);
    const uint32_t row_in = (uint32_t)d * IN_BYTES;  // bytes of one input row
    // NAMED: a group waits only for its own threads (named barrier 1 + grp, GTP threads)
    auto group_sync = [&]() {
        if constexpr (NAMED)
            asm volatile("bar.sync %0, %1;" ::"r"(1 + grp), "r"(GTP) : "memory");
        else
            __syncthreads();
    };

    // shared memory: [table][entries][decode table][partials][mbarriers][raw rows][pairs]
    uint32_t *table = reinterpret_cast<uint32_t *>(smem);
    uint32_t *gent = table + p.tbl_words;
    uint32_t *dect = gent + p.ent_words;             // A16 only (dec_words = 0 otherwise)
    uint32_t *wdect = dect + p.dec_words;            // fused 2-bit weight decode table
    const float *gtab = reinterpret_cast<const float *>(wdect + p.wdec_words);   // GELU only
    float2 *red = reinterpret_cast<float2 *>(wdect + p.wdec_words + p.gelu_words);
    unsigned long long *bars = reinterpret_cast<unsigned long long *>(red + 2 * NG * kMaxSeg);
    // [0] next pair, [1 + grp] a group's next pair, [16] next decode chunk, [17 + grp] a
    // group's decode chunk
    int *sched = reinterpret_cast<int *>(bars + 2 * NG + 2);
    unsigned char *raw = reinterpret_cast<unsigned char *>(sched + 32);
    unsigned char *myraw = raw + (size_t)grp * nstage * 2 * row_in;
    unsigned char *pairs = raw + (size_t)NG * nstage * 2 * row_in;
    unsigned char *mypairs = pairs + (size_t)grp * d * 4;
    const uint32_t setup_bar = smem_u32(&bars[2 * NG]);

    pdl_trigger();
    if (tid == 0) {
        for (int b = 0; b < 2 * NG + 1; ++b)
            mbar_init(smem_u32(&bars[b]), 1);
        mbar_init(smem_u32(&bars[2 * NG + 1]), 2);   // the armed test wait's barrier
        sched[0] = NG;                               // pairs lo .. lo + NG - 1 start the groups
        sched[16] = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (tid == 0) {
        // host-built table, entry and decode images: bulk copies
        mbar_expect_tx(setup_bar, 4u * (p.tbl_words + p.ent_words + p.dec_words +
                                        p.wdec_words + p.gelu_words));
        bulk_copy(smem_u32(table), p.tbl_img, 4u * p.tbl_words, setup_bar);
        bulk_copy(smem_u32(gent), p.ent_img, 4u * p.ent_words, setup_bar);
        if (p.dec_words > 0)
            bulk_copy(smem_u32(dect), p.dec_img, 4u * p.dec_words, setup_bar);
        if (p.wdec_words > 0)
            bulk_copy(smem_u32(wdect), p.wdec_img, 4u * p.wdec_words, setup_bar);
        if (p.gelu_words > 0)
            bulk_copy(smem_u32(gtab), p.gelu_img, 4u * p.gelu_words, setup_bar);
    }

    // this thread's 32 rotated positions: pos0 + e with pos0 = g * 32; r = its index inside
    // the h-block (0 when a block fits inside one thread)
    const int r = g % Q;
    const int pos0 = g * kE;
    const uint4 *myent = reinterpret_cast<const uint4 *>(gent + min(g, GT - 1) * kEntStride);
    const uint32_t tbl_lane =
        smem_u32(table) + (REPL ? lane * 4 : 0) - ((0x3F800000u >> p.F) << TSH);
    const uint32_t G = (uint32_t)p.G;
    const int F = p.F;

    const int seg_end = min(active, lane + (GT - g));
    const bool seg_head = (lane == 0) || (g == 0);
    const int seg_slot = (g == 0) ? 0 : (g + 31) / 32;
    const int nslots = NAMED ? (GT + 31) / 32 : 1 + ((grp * GT + GT - 1) / 32 - (grp * GT) / 32);
    const int row_bytes = d * BITS / 8;
    const long long npairs = ((long long)p.T + 1) / 2;
    // The group's pairs are lo + my for my < cnt.  NAMED: the CTA owns an equal contiguous
    // share of all pairs and its groups take them from a shared counter (a group that finishes
    // early takes the next one).  Otherwise all groups of all CTAs step through the pairs in
    // lockstep rounds of gridDim.x * NG, and a CTA leaves once its next round is empty.
    constexpr bool dyn = NAMED;
    const long long lo = dyn ? (long long)blockIdx.x * npairs / gridDim.x
                             : (long long)blockIdx.x * NG;
    const int cnt = (int)(dyn ? ((long long)blockIdx.x + 1) * npairs / gridDim.x - lo
                              : npairs - lo);
    const int step = dyn ? NG : (int)gridDim.x * NG;
    const unsigned char *xb = static_cast<const unsigned char *>(p.x);

    // the two rows of pair lo + i into raw stage `s` (one thread per group issues)
    auto issue = [&](int i, int s) {
        if (g != 0 || i >= cnt)
            return;
        const long long t0 = 2 * (lo + i);
        const bool two = t0 + 1 < p.T;
        const uint32_t bar = smem_u32(&bars[2 * grp + s]);
        const uint32_t dst = smem_u32(myraw + (size_t)s * 2 * row_in);
        mbar_expect_tx(bar, two ? 2 * row_in : row_in);
        bulk_copy(dst, xb + t0 * row_in, row_in, bar);
        if (two)
            bulk_copy(dst + row_in, xb + (t0 + 1) * row_in, row_in, bar);
    };

    pdl_wait();                                        // x, codes, norms: earlier work done
    issue(grp, 0);
    if (!mbar_wait(setup_bar, 0))
        atomicOr(&g_k1_err, K1_ERR_COPY_WAIT);

    int my = grp;                                      // the pair in hand: lo + my
    for (int round = 0;; ++round) {
        if (dyn ? my >= cnt : my - grp >= cnt)
            break;                                     // uniform across the group / the CTA
        const long long pr = lo + my;
        bool valid = my < cnt;
        const long long t0 = 2 * pr, t1 = 2 * pr + 1;
        const int stage = round % nstage;
        const uint32_t parity = (uint32_t)(round / nstage) & 1u;

        if (valid && !mbar_wait(smem_u32(&bars[2 * grp + stage]), parity)) {
            atomicOr(&g_k1_err, K1_ERR_COPY_WAIT);
            valid = false;
        }
        const bool has1 = valid && t1 < p.T;
        const unsigned char *cur = myraw + (size_t)stage * 2 * row_in;

        if constexpr (!IN_F32) {
            // ---- interleave the staged rows into the pair buffer ---------------------------
            if (valid && owns) {
                const uint4 *r0 = reinterpret_cast<const uint4 *>(cur);
                const uint4 *r1 = reinterpret_cast<const uint4 *>(cur + row_in);
                uint4 *slots = reinterpret_cast<uint4 *>(mypairs);
                // the 16-byte slots of this thread's eight half-chunks (host-chosen so that
                // the random gather below spreads over the banks)
                const uint4 sl = myent[kE / 4];
                const uint32_t slw[4] = {sl.x, sl.y, sl.z, sl.w};
#pragma unroll
                for (int k = 0; k < kE / 8; ++k) {
                    const int c = g + k * GT;              // elements 8c..8c+7
                    const uint4 a = r0[c], b = r1[c];
                    slots[slw[k] & 0xffffu] =
                        make_uint4(prmt(a.x, b.x, 0x5410), prmt(a.x, b.x, 0x7632),
                                   prmt(a.y, b.y, 0x5410), prmt(a.y, b.y, 0x7632));
                    slots[slw[k] >> 16] =
                        make_uint4(prmt(a.z, b.z, 0x5410), prmt(a.z, b.z, 0x7632),
                                   prmt(a.w, b.w, 0x5410), prmt(a.w, b.w, 0x7632));
                }
            }
            group_sync();
            if (dyn) {                                     // raw is free: fetch the next pair
                if (g == 0) {
                    const int nx = atomicAdd(&sched[0], 1);
                    sched[1 + grp] = nx;
                    issue(nx, 0);
                }
            } else {
                issue(my + step, 0);
            }
        } else {
            if (nstage > 1)
                issue(my + step, (round + 1) % nstage);    // the other stage is free
        }

        // ---- gather y[i] = sign[i] * x[perm[i]] for both tokens ------------------------------
        float2 v[kE];
        {
            const uint32_t base0 = IN_F32 ? smem_u32(cur) : smem_u32(mypairs);
#pragma unroll
            for (int e4 = 0; e4 < kE / 4; ++e4) {
                const uint4 q4 = myent[e4];
                const uint32_t en4[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int e = 4 * e4 + i;
                    const uint32_t en = en4[i];
                    const uint32_t sg = en & 0x80000000u;
                    const uint32_t off = en & 0x7fffffffu;
                    if constexpr (GELU) {
                        const uint32_t w = lds32(base0 + off);
                        const float a = gelu_lookup(w << 16, smem_u32(gtab));
                        const float b = gelu_lookup(w & 0xffff0000u, smem_u32(gtab));
                        v[e].x = __uint_as_float(__float_as_uint(a) ^ sg);
                        v[e].y = __uint_as_float(__float_as_uint(b) ^ sg);
                    } else if constexpr (!IN_F32) {
                        const uint32_t w = lds32(base0 + off);
                        v[e].x = __uint_as_float((w << 16) + sg);
                        v[e].y = __uint_as_float((w ^ en) & 0xffff0000u);
                    } else {
                        v[e].x = __uint_as_float(lds32(base0 + off) ^ sg);
                        v[e].y = __uint_as_float(lds32(base0 + row_in + off) ^ sg);
                    }
                }
            }
        }

        // ---- block Walsh-Hadamard (natural order), unnormalised --------------------------
#pragma unroll
        for (int s = 1; s < kE; s <<= 1) {
            if (H < kE && s >= hrt)
                break;                                 // blocks of h < 32 end here
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
            red[((round & 1) * NG + grp) * kMaxSeg + seg_slot] = acc;
        group_sync();
        if constexpr (IN_F32) {
            if (nstage == 1)
                issue(my + step, 0);                       // gathers are done: refill
        }
        // partials alternate between two buffers by round: a round's writes never meet the
        // previous round's reads, which the barrier of that round separates
        const float2 *myred = red + ((round & 1) * NG + grp) * kMaxSeg;
        // the group's next pair (its leader wrote the index before the barrier above)
        const int nxt = dyn ? sched[1 + grp] : my + step;
        float2 ss = myred[0];
        for (int i = 1; i < nslots; ++i) {
            const float2 o = myred[i];
            ss.x += o.x;
            ss.y += o.y;
        }
        const float inv_h = H >= kE ? 1.0f / H : 1.0f / (float)hrt;   // exact: h = 2^k
        const float s0 = sqrtf(ss.x * inv_h);
        const float s1 = sqrtf(ss.y * inv_h);
        const float m0 = (s0 + p.eps > 0.f) ? p.K / (s0 + p.eps) : 0.f;
        const float m1 = (s1 + p.eps > 0.f) ? p.K / (s1 + p.eps) : 0.f;

        // ---- nearest centroid + pack ---------------------------------------------------------
        uint32_t w0[NW], w1[NW];
        // The code of element e is the top byte of D = q*G + table[q >> F].
        auto code_word = [&](float vx, float vy, uint32_t &d0, uint32_t &d1) {
            const float a0 = fma_sat(vx, m0, 0.5f);
            const float a1 = fma_sat(vy, m1, 0.5f);
            const uint2 qb = f2_add_one_rm_bits(a0, a1);
            d0 = qb.x * G + lds32(tbl_lane + ((qb.x >> F) << TSH));
            d1 = qb.y * G + lds32(tbl_lane + ((qb.y >> F) << TSH));
        };
        if constexpr (BITS == 3 || BITS == 6) {
#pragma unroll
            for (int i = 0; i < NW; ++i) {
                w0[i] = 0;
                w1[i] = 0;
            }
#pragma unroll
            for (int e = 0; e < kE; ++e) {
                uint32_t d0, d1;
                code_word(v[e].x, v[e].y, d0, d1);
                const uint32_t c0 = d0 >> 24, c1 = d1 >> 24;
                const int bit = e * BITS;
                const int wi = bit >> 5, sh = bit & 31;
                w0[wi] |= c0 << sh;
                w1[wi] |= c1 << sh;
                if (sh + BITS > 32) {
                    w0[wi + 1] |= c0 >> (32 - sh);
                    w1[wi + 1] |= c1 >> (32 - sh);
                }
            }
        } else {
            // byte permutes gather the top bytes; 2- and 4-bit codes are then merged into
            // nibbles / bit pairs with shifted adds (the bytes' upper bits are zero)
            constexpr int PER = 32 / BITS;                 // codes per output word
#pragma unroll
            for (int wi = 0; wi < NW; ++wi) {
                uint32_t d0[PER], d1[PER];
#pragma unroll
                for (int k = 0; k < PER; ++k)
                    code_word(v[wi * PER + k].x, v[wi * PER + k].y, d0[k], d1[k]);
                w0[wi] = pack_codes<BITS>(d0);
                w1[wi] = pack_codes<BITS>(d1);
            }
        }
        if (valid && owns) {
            if constexpr (A16) {
                uint4 *a0 = reinterpret_cast<uint4 *>(p.a16 + t0 * d + pos0);
                const uint32_t src[4] = {p.dec_src[0], p.dec_src[1], p.dec_src[2], p.dec_src[3]};
                decode_store<BITS>(dect, w0, a0, src);
                if (has1)
                    decode_store<BITS>(dect, w1, a0 + d / 8, src);
            } else {
                uint8_t *dst0 = p.codes + t0 * row_bytes + pos0 * BITS / 8;
                store_words<NW>(dst0, w0);
                if (has1)
                    store_words<NW>(dst0 + row_bytes, w1);
            }
            if (g == 0)
                p.norms[t0] = s0;
            if (has1 && g == 0)
                p.norms[t1] = s1;
        }
        my = nxt;
    }

    if constexpr (NAMED) {
        // ---- fused weight decode: this CTA's share of the code words, in chunks of GTP * 8 --
        if (p.wdec_groups > 0) {
            const long long dlo = (long long)blockIdx.x * p.wdec_groups / gridDim.x;
            const long long dcnt = ((long long)blockIdx.x + 1) * p.wdec_groups / gridDim.x - dlo;
            const uint32_t *wc = p.wdec_codes + dlo;
            uint4 *wo = p.wdec_out + (p.wdec_bits == 4 ? dlo : 2 * dlo);
            constexpr int kU = 8;                          // code words per thread and chunk
            for (;;) {
                if (g == 0)
                    sched[17 + grp] = atomicAdd(&sched[16], 1);
                group_sync();
                const long long c0 = (long long)sched[17 + grp] * GTP * kU;
                group_sync();                              // read before the next claim
                if (c0 >= dcnt)
                    break;
                uint32_t wv[kU];
#pragma unroll
                for (int j = 0; j < kU; ++j) {
                    const long long i = c0 + g + (long long)j * GTP;
                    wv[j] = i < dcnt ? __ldg(wc + i) : 0u;
                }
#pragma unroll
                for (int j = 0; j < kU; ++j) {
                    const long long i = c0 + g + (long long)j * GTP;
                    if (i < dcnt) {
                        if (p.wdec_bits == 4) {
                            uint32_t o[4];
                            decode8(wv[j], p.wdec_src[0], p.wdec_src[1], p.wdec_src[2],
                                    p.wdec_src[3], o);
                            wo[i] = make_uint4(o[0], o[1], o[2], o[3]);
                        } else {                           // 2-bit: a byte = 4 centroids
                            const uint2 *t2 = reinterpret_cast<const uint2 *>(wdect);
                            const uint2 q0 = t2[wv[j] & 0xffu], q1 = t2[(wv[j] >> 8) & 0xffu];
                            const uint2 q2 = t2[(wv[j] >> 16) & 0xffu], q3 = t2[wv[j] >> 24];
                            wo[2 * i] = make_uint4(q0.x, q0.y, q1.x, q1.y);
                            wo[2 * i + 1] = make_uint4(q2.x, q2.y, q3.x, q3.y);
                        }
                    }
                }
            }
        }
    }

    // ---- armed test of the bounded waits (oq_debug_arm_wait_timeout): after all of its work,
    // one thread waits on a barrier that expects two arrivals and gets one, gives up after
    // p.test_wait_cycles and records it, exactly as a stalled copy's wait would.  No copy
    // targets this barrier, so nothing is in flight when the CTA exits.
    if (p.test_wait_cycles > 0 && blockIdx.x == 0 && tid == 0) {
        const uint32_t tb = smem_u32(&bars[2 * NG + 1]);
        mbar_arrive(tb);
        if (!mbar_wait(tb, 0, p.test_wait_cycles))
            atomicOr(&g_k1_err, K1_ERR_ARMED_WAIT);
    }
}

// Shared-memory attributes are set once per kernel and device, and occupancy is cached per
// (kernel, device, block size, shared memory), to keep the per-call host cost low.
cudaError_t k1_prepare(const void *kern, int threads, size_t smem, int *per_sm) {
    struct Key {
        const void *k;
        int dev, threads;
        size_t smem;
        bool operator<(const Key &o) const {
            return std::tie(k, dev, threads, smem) < std::tie(o.k, o.dev, o.threads, o.smem);
        }
    };
    static std::mutex mu;
    static std::map<Key, int> occ;
    static std::set<std::pair<const void *, int>> attr_done;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    std::lock_guard<std::mutex> lk(mu);
    if (!attr_done.count({kern, dev})) {
        e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess)
            return e;
        attr_done.insert({kern, dev});
    }
    const Key key{kern, dev, threads, smem};
    auto it = occ.find(key);
    if (it == occ.end()) {
        int n = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kern, threads, smem);
        if (e != cudaSuccess)
            return e;
        it = occ.emplace(key, n).first;
    }
    *per_sm = it->second;
    return cudaSuccess;
}

template <int BITS, bool F32, bool GELU = false, bool A16 = false>
cudaError_t launch_h(const K1Params &p, int h, long long ctas_needed, int threads, size_t smem,
                     int num_sms, cudaStream_t st, std::string *why, bool named) {
    auto go = [&](auto kern) -> cudaError_t {
        int per_sm = 0;
        cudaError_t e = k1_prepare((const void *)kern, threads, smem, &per_sm);
        if (e != cudaSuccess || per_sm < 1) {
            *why = "k1 attributes / occupancy";
            return e != cudaSuccess ? e : cudaErrorInvalidConfiguration;
        }
        long long grid = (long long)num_sms * per_sm;
        if (grid > ctas_needed)
            grid = ctas_needed;
        e = launch_pdl(kern, dim3((unsigned)grid), dim3(threads), smem, st, p);
        if (e != cudaSuccess)
            *why = "k1 launch";
        return e;
    };
    // the named-barrier form exists for bf16 input only (F32 picks the same kernel twice)
    auto pick = [&](auto kn, auto kl) { return named ? go(kn) : go(kl); };
    if constexpr (A16) {            // the fp16-output variants are built for h <= 256
        switch (h) {
            case 32: return pick(k1_rotquant<BITS, F32, 32, GELU, true, !F32>, k1_rotquant<BITS, F32, 32, GELU, true>);
            case 64: return pick(k1_rotquant<BITS, F32, 64, GELU, true, !F32>, k1_rotquant<BITS, F32, 64, GELU, true>);
            case 128: return pick(k1_rotquant<BITS, F32, 128, GELU, true, !F32>, k1_rotquant<BITS, F32, 128, GELU, true>);
            case 256: return pick(k1_rotquant<BITS, F32, 256, GELU, true, !F32>, k1_rotquant<BITS, F32, 256, GELU, true>);
            default: *why = "unsupported h for fp16 output"; return cudaErrorInvalidValue;
        }
    } else {
        switch (h) {
            case 2:
            case 4:
            case 8:
            case 16: return pick(k1_rotquant<BITS, F32, kSmallH, GELU, false, !F32>, k1_rotquant<BITS, F32, kSmallH, GELU>);
            case 32: return pick(k1_rotquant<BITS, F32, 32, GELU, false, !F32>, k1_rotquant<BITS, F32, 32, GELU>);
            case 64: return pick(k1_rotquant<BITS, F32, 64, GELU, false, !F32>, k1_rotquant<BITS, F32, 64, GELU>);
            case 128: return pick(k1_rotquant<BITS, F32, 128, GELU, false, !F32>, k1_rotquant<BITS, F32, 128, GELU>);
            case 256: return pick(k1_rotquant<BITS, F32, 256, GELU, false, !F32>, k1_rotquant<BITS, F32, 256, GELU>);
            case 512: return pick(k1_rotquant<BITS, F32, 512, GELU, false, !F32>, k1_rotquant<BITS, F32, 512, GELU>);
            case 1024: return pick(k1_rotquant<BITS, F32, 1024, GELU, false, !F32>, k1_rotquant<BITS, F32, 1024, GELU>);
            default: *why = "unsupported h"; return cudaErrorInvalidValue;
        }
    }
}

size_t k1_smem(const K1Params &p, int in_f32, int NG, int stages) {
    const size_t row_in = (size_t)p.d * (in_f32 ? 4 : 2);
    size_t b = 4 * (size_t)(p.tbl_words + p.ent_words + p.dec_words + p.wdec_words +
                            p.gelu_words);
    b += sizeof(float2) * 2 * NG * kMaxSeg;                // norm partials, two buffers
    b += 8 * (size_t)(2 * NG + 2);                         // mbarriers
    b += 4 * 32;                                           // pair and decode scheduling words
    b += (size_t)NG * stages * 2 * row_in;                 // raw rows
    if (!in_f32)
        b += (size_t)NG * p.d * 4;                         // interleaved pairs
    return b;
}

}  // namespace

cudaError_t launch_k1(const K1Params &p_in, int bits, int h, int in_f32, cudaStream_t st,
                      int num_sms, std::string *why) {
    K1Params p = p_in;
    const int GT = p.d / kE;
    const long long npairs = ((long long)p.T + 1) / 2;
    int stages = in_f32 ? 2 : 1;
    if (in_f32 && k1_smem(p, in_f32, 1, 2) > 200 * 1024)
        stages = 1;
    long long ctas_needed;
    int NG;
    const bool named = k1_named(p.d, !in_f32);
    const int GTP = named ? k1_group_threads(p.d) : GT;   // threads per group
    if (p.wdec_groups > 0 && !named) {
        *why = "fused weight decode needs the named-barrier K1 (bf16 rows, whole-warp groups)";
        return cudaErrorInvalidValue;
    }
    if (named) {
        // Groups of whole warps: one CTA per SM with as many groups as the register file
        // holds (96 registers a thread; at most 15 named barriers and 1024 threads), each CTA
        // an equal share of the pairs.  The group count is the smallest that takes the share
        // in the same number of rounds, so the rounds stay full.
        // With a fused weight decode every SM takes a share of the decode with all the groups
        // it holds, whatever the number of pairs.
        const bool wdec = p.wdec_groups > 0;
        ctas_needed = wdec ? num_sms : std::min<long long>(num_sms, npairs);
        const long long share = (npairs + ctas_needed - 1) / ctas_needed;
        // registers: each of the SM's four 16K-register partitions holds 5 warps of 96
        constexpr int kWarpsPerSm = 4 * ((65536 / 4) / (96 * 32));
        int ng_max = std::min(std::min(15, 1024 / GTP), kWarpsPerSm * 32 / GTP);
        while (ng_max > 1 && k1_smem(p, in_f32, ng_max, stages) > 220 * 1024)
            --ng_max;
        if (wdec) {
            NG = ng_max;
        } else {
            ng_max = (int)std::max(1LL, std::min<long long>(ng_max, share));
            const long long rounds = (share + ng_max - 1) / ng_max;
            NG = (int)((share + rounds - 1) / rounds);
        }
    } else {
        // Groups that share warps run in lockstep: several smaller CTAs per SM.
        NG = 256 / GT;
        if (NG < 1)
            NG = 1;
        if (NG > npairs)
            NG = (int)npairs;
        while (NG > 1 && k1_smem(p, in_f32, NG, stages) > 72 * 1024)
            --NG;
        ctas_needed = (npairs + NG - 1) / NG;
    }
    const size_t smem = k1_smem(p, in_f32, NG, stages);
    if (smem > 227 * 1024) {
        *why = "k1 shared memory exceeds the per-CTA limit";
        return cudaErrorInvalidConfiguration;
    }
    p.groups = NG;
    p.stages = stages;
    const int threads = NG * GTP;
    if (p.a16) {
        if (in_f32) {
            *why = "fp16 centroid output takes bf16 input";
            return cudaErrorInvalidValue;
        }
        auto go16 = [&](auto gelu_tag) -> cudaError_t {
            constexpr bool GL = decltype(gelu_tag)::value;
            switch (bits) {
                case 2: return launch_h<2, false, GL, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
                case 4: return launch_h<4, false, GL, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
                case 8: return launch_h<8, false, GL, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
                default: *why = "fp16 centroid output: bit width"; return cudaErrorInvalidValue;
            }
        };
        return p.gelu ? go16(std::true_type{}) : go16(std::false_type{});
    }
    if (p.gelu) {
        if (in_f32) {
            *why = "fused GELU takes bf16 input";
            return cudaErrorInvalidValue;
        }
        switch (bits) {
            case 2: return launch_h<2, false, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
            case 3: return launch_h<3, false, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
            case 4: return launch_h<4, false, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
            case 6: return launch_h<6, false, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
            case 8: return launch_h<8, false, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
            default: *why = "unsupported bit width"; return cudaErrorInvalidValue;
        }
    }
    switch (bits * 2 + (in_f32 ? 1 : 0)) {
        case 4: return launch_h<2, false>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 5: return launch_h<2, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 6: return launch_h<3, false>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 7: return launch_h<3, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 8: return launch_h<4, false>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 9: return launch_h<4, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 12: return launch_h<6, false>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 13: return launch_h<6, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 16: return launch_h<8, false>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
        case 17: return launch_h<8, true>(p, h, ctas_needed, threads, smem, num_sms, st, why, named);
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
