// k2_linear.cu -- codebook linear layer on sm_100a: y = (s_t rn_o / d) * sum_k Ca[xc] Cw[wc].
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video":
// rotation-cancellation paragraph (W R^T R x = W x, so codes of R x and of R w meet directly)
// and the pseudocode's x_hat = s * codebook[xc], W_hat = diag(row_norms) * codebook[wc]; its
// speed-caveat paragraph notes that non-uniform centroids cannot feed integer tensor cores,
// which is why the codes are decoded to fp16 unit centroids before the MMA.
//
// Path: (1) decode prepass (k2_decode.cu): packed codes -> fp16 unit-variance centroids, for
// the activation codes and the weight codes, into stream-ordered workspace; (2) this file's
// hand-written persistent tcgen05 GEMM: TMA (128B swizzle) brings fp16 K-major tiles into a 4-stage
// shared-memory ring, one elected thread issues tcgen05.mma kind::f16 (M=128, N=256, K=16)
// into one of two TMEM fp32 accumulators (2 x 256 columns), and 4 epilogue warps read the
// other accumulator back with tcgen05.ld, apply the s_t * rn_o / d scale and hand 32 x 32
// chunks to TMA tensor stores.  sigma^2 = 1/d is folded into the epilogue so the fp16 values
// are unit-variance (best fp16 precision).  Every mbarrier wait is bounded by
// SM clock cycles (about 2 s); a wait that gives up sets a bit in the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdlib>
#include <mutex>

#include "decode4.cuh"
#include "oq_internal.h"
#include "sm100_common.cuh"

namespace oq {
namespace {

using namespace sm100;

__device__ unsigned int g_k2_err;

// Fixed workspace for oq_linear_noalloc: the fp16 operand buffers live here instead of in
// memory the library allocates.  Every GPU that loads the library holds this array until the
// process exits.  Host code must not use the symbol as an address (it is a host-side stand-in);
// noalloc_workspace() looks the device address up once per device.
constexpr size_t kNoAllocWorkspaceBytes = 64ull << 20;
// beyond the operands: the split-K partials of a small-T call (at most 74 work units of one
// 256 x 256 fp32 tile each, 18.5 MiB)
constexpr size_t kNoAllocSplitBytes = 20ull << 20;
static __device__ __align__(256) unsigned char
    g_noalloc_workspace[kNoAllocWorkspaceBytes + kNoAllocSplitBytes];

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;               // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;               // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;

enum : unsigned {
    ERR_WAIT_FULL = 1u << 0,
    ERR_WAIT_EMPTY = 1u << 1,
    ERR_WAIT_ACCUM = 1u << 2,
    ERR_ARMED_WAIT = 1u << 3,     // the armed test wait (oq_debug_arm_wait_timeout) gave up
};

// ------------------------------------------------------------------------------------------
// Persistent tcgen05 GEMM.  The B operand (fp16 weight centroids from the prepass) always
// comes in by TMA.  The A operand either comes in by TMA as well (fp16 activation centroids
// from the prepass), or, for 4-bit activation codes of a symmetric codebook (ACODES), four
// decoder warps read the packed codes and write the fp16 A tile into the same shared-memory
// ring, in the layout TMA would have produced.
// ------------------------------------------------------------------------------------------
constexpr uint32_t kIdesc = idesc_f16(BM, BN);

struct GemmParams {
    const float *s;
    const float *rn;
    uint32_t L0, L1, H0, H1;    // ACODES: decode8 sources of the activation codebook
    int M, N, K;
    float inv_d;
    long long test_wait_cycles; // > 0: the armed test wait (oq_debug_arm_wait_timeout)
    int ksplit;                 // pair kernel: k-ranges per tile (1: none), kb_per k-blocks
    int kb_per;                 // each; partials in rows part * m_pad + row of tmP
    int m_pad;
    void *y;                    // k2_splitk_reduce: the output
};

// The armed test of the bounded waits: after all of the kernel's work, one thread waits on a
// barrier that expects two arrivals and gets one, gives up after `cycles` and records it in
// the error word, exactly as a stalled pipeline wait would.  Nothing targets this barrier.
__device__ __forceinline__ void armed_test_wait(uint32_t bar, long long cycles) {
    mbar_arrive(bar);
    if (!mbar_wait(bar, 0, cycles))
        atomicOr(&g_k2_err, ERR_ARMED_WAIT);
}

constexpr int kEpiWarps = 4;         // warps 2..5
constexpr int kDecWarps = 8;         // ACODES: warps 6..13, two per TMEM lane quarter
constexpr int kAccCols = BN;         // one fp32 accumulator: 256 TMEM columns
constexpr int kTmemCols = 2 * kAccCols;
constexpr int kStageOut = 32 * 32 * 4;                        // one 32 x 32 fp32 output chunk
constexpr int kCodeStageBytes = BM * BK / 2;                  // ACODES: 128 rows x 32 bytes
constexpr int kNumBars = 3 * STAGES + 5;

// ACODES keeps one output staging buffer per epilogue warp (room for the code stages).
template <bool ACODES>
__host__ __device__ constexpr int out_bufs() { return ACODES ? 1 : 2; }

template <bool ACODES>
__host__ __device__ constexpr size_t gemm_smem() {
    return 1024 + (size_t)STAGES * (STAGE_BYTES + (ACODES ? kCodeStageBytes : 0)) +
           (size_t)kEpiWarps * out_bufs<ACODES>() * kStageOut + 8 * kNumBars + 8 +
           kEpiWarps * 64 * sizeof(float) + 64;
}
static_assert(gemm_smem<false>() <= 227 * 1024 && gemm_smem<true>() <= 227 * 1024,
              "shared memory budget");

template <bool ACODES>
__host__ __device__ constexpr int gemm_threads() { return 32 * (2 + kEpiWarps + (ACODES ? kDecWarps : 0)); }

// Persistent, warp-specialised tcgen05 GEMM.  Warp 0 lane 0: TMA producer over a 4-stage
// shared-memory ring.  Warp 1: TMEM owner; its lane 0 issues the MMAs.  Warps 2..5: epilogue
// (TMEM lane quarter = warp % 4), each with 4 KB output staging buffers that TMA tensor
// stores drain to global memory.  ACODES: tmA maps the packed codes (uint8 [M, K/2], 32 x 128
// byte boxes), TMA brings each stage's code tile in with its B tile, and warps 6..9 decode the
// codes of rows (warp % 4) * 32 + lane into the stage's A tile (warps 6..9 the first 32 codes
// of each row and k-block, warps 10..13 the last 32).  Two 256-column accumulators alternate between
// tiles, so the epilogue of one tile overlaps the mainloop of the next.  Tiles are walked
// n-fastest so consecutive CTAs share the same 128-row A block in L2.  BF16: y is bf16
// (32 x 64 chunks) instead of fp32 (32 x 32 chunks).
template <bool BF16, bool ACODES>
__global__ void __launch_bounds__(gemm_threads<ACODES>(), 1)
    k2_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ CUtensorMap tmY, const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;                 // 1 KB aligned tiles
    unsigned char *basep = smem_raw + (base - raw);
    constexpr int kOutBufs = out_bufs<ACODES>();
    const uint32_t sA = base, sB = base + STAGES * A_STAGE_BYTES;
    const uint32_t sC = sB + STAGES * B_STAGE_BYTES;              // ACODES: code stages
    const uint32_t sOut = sC + (ACODES ? STAGES * kCodeStageBytes : 0);   // [4][bufs][4 KB]
    const uint32_t bars = sOut + kEpiWarps * kOutBufs * kStageOut;
    auto full_bar = [&](int s) { return bars + 8u * s; };                   // TMA bytes
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };       // MMA done
    auto afull_bar = [&](int s) { return bars + 8u * (2 * STAGES + s); };   // ACODES: A
    auto tfull_bar = [&](int a) { return bars + 8u * (3 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (3 * STAGES + 2 + a); };
    const uint32_t drain_bar = bars + 8u * (3 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(basep + (drain_bar + 8u - base));
    float *rn_s = reinterpret_cast<float *>(basep + (drain_bar + 16u - base));   // [4][64]
    __shared__ int abort_flag;
    __shared__ __align__(8) unsigned long long test_bar;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = ((p.M + BM - 1) / BM) * n_tiles;
    const int num_kb = p.K / BK;

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
            mbar_init(afull_bar(s), kDecWarps);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        mbar_init(smem_u32(&test_bar), 2);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                         // operands, s, rn and y: earlier work of the stream done
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };
    auto give_up = [&](unsigned bit) {
        atomicOr(&g_k2_err, bit);
        atomicExch(&abort_flag, 1);
    };

    if (warp == 0) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !aborted(); tile += gridDim.x) {
                const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * BN;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (it >= STAGES &&
                        !mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1)) {
                        give_up(ERR_WAIT_EMPTY);
                        break;
                    }
                    if (aborted())
                        break;
                    if constexpr (ACODES) {
                        mbar_expect_tx(full_bar(s), B_STAGE_BYTES + kCodeStageBytes);
                        tma_load_2d(sC + s * kCodeStageBytes, &tmA, kb * (BK / 2), m0,
                                    full_bar(s));
                    } else {
                        mbar_expect_tx(full_bar(s), STAGE_BYTES);
                        tma_load_2d(sA + s * A_STAGE_BYTES, &tmA, kb * BK, m0, full_bar(s));
                    }
                    tma_load_2d(sB + s * B_STAGE_BYTES, &tmB, kb * BK, n0, full_bar(s));
                }
            }
            if (aborted()) {
                // let the loads already issued land before the CTA can exit
                const uint32_t from = it > (uint32_t)STAGES ? it - STAGES : 0;
                for (uint32_t j = from; j < it; ++j)
                    mbar_wait(full_bar(j % STAGES), (j / STAGES) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            int i = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !aborted();
                 tile += gridDim.x, ++i) {
                const int acc = i & 1;
                if (i >= 2 && !mbar_wait(tempty_bar(acc), ((i >> 1) & 1) ^ 1)) {
                    give_up(ERR_WAIT_EMPTY);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kAccCols);
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!mbar_wait(full_bar(s), (it / STAGES) & 1) ||
                        (ACODES && !mbar_wait(afull_bar(s), (it / STAGES) & 1))) {
                        give_up(ERR_WAIT_FULL);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sw128_desc(sA + s * A_STAGE_BYTES);
                    const uint64_t db = sw128_desc(sB + s * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)   // 16 fp16 = 32 bytes = 2 desc units
                        mma_ss(d_tmem, da + 2 * kk, db + 2 * kk, kIdesc, (kb | kk) != 0);
                    mma_commit(empty_bar(s));
                }
                if (!ok)
                    break;
                mma_commit(tfull_bar(acc));
            }
            // every MMA issued above has completed once this barrier flips
            mma_commit(drain_bar);
            if (!mbar_wait(drain_bar, 0))
                atomicOr(&g_k2_err, ERR_WAIT_ACCUM);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ---------------- epilogue: TMEM -> registers -> scale -> smem -> TMA store -------
        // No cross-warp barrier: one warp giving up a wait cannot strand the others.
        const int q = warp & 3;                               // TMEM lane quarter
        float *rn_w = rn_s + (warp - 2) * 64;
        const uint32_t out0 = sOut + (uint32_t)((warp - 2) * kOutBufs * kStageOut);
        unsigned char *out0p = basep + (out0 - base);
        uint32_t u = 0;                                       // chunks stored so far
        int i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int acc = i & 1;
            const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * BN;
            const int row = m0 + q * 32 + lane;
            const float srow = (row < p.M) ? p.s[row] * p.inv_d : 0.f;
            float rnv[BN / 32];                               // rn of column c*32 + lane
#pragma unroll
            for (int c = 0; c < BN / 32; ++c) {
                const int col = n0 + c * 32 + lane;
                rnv[c] = (col < p.N) ? p.rn[col] : 0.f;
            }
            const bool ok = mbar_wait(tfull_bar(acc), (i >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (!ok)
                    give_up(ERR_WAIT_ACCUM);
                break;
            }
            tc_fence_after();
            const uint32_t t_base =
                tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols);
            const bool rows_in = m0 + q * 32 < p.M;
            constexpr int kCW = BF16 ? 64 : 32;               // columns per stored chunk
#pragma unroll
            for (int c = 0; c < BN / kCW; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_base + (uint32_t)(c * kCW), r0);
                if constexpr (BF16)
                    tmem_ld32(t_base + (uint32_t)(c * kCW + 32), r1);
                if (!rows_in || n0 + c * kCW >= p.N)
                    continue;                                 // box wholly outside y
                const uint32_t b = kOutBufs == 2 ? (u & 1) : 0;
                if (lane == 0)
                    bulk_wait_read<kOutBufs - 1>();           // the store that used buffer b
                __syncwarp();
                if constexpr (BF16) {
                    rn_w[lane] = rnv[2 * c];
                    rn_w[32 + lane] = rnv[2 * c + 1];
                } else {
                    rn_w[lane] = rnv[c];
                }
                __syncwarp();
                if constexpr (BF16)
                    store_chunk_bf16(&tmY, out0p + b * kStageOut, out0 + b * kStageOut, r0, r1,
                                     srow, rn_w, lane, n0 + c * kCW, m0 + q * 32);
                else
                    store_chunk(&tmY, out0p + b * kStageOut, out0 + b * kStageOut, r0, srow,
                                rn_w, lane, n0 + c * kCW, m0 + q * 32);
                ++u;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
        }
        if (lane == 0)
            bulk_wait_all();
    } else if constexpr (ACODES) {
        // ---------------- activation decoders: 4-bit codes -> fp16 A stages ----------------
        // Thread = row r of the 128-row tile and one half of its 64 codes per k-block: it reads
        // 16 bytes of codes from the stage's code tile and writes 64 bytes of the fp16 row in
        // the 128-byte swizzled layout (16-byte piece k at piece k ^ (r % 8) of the row; 8-row
        // atoms of 1024 bytes), which is what a TMA load of the decoded operand would have
        // written.  The stage's full barrier also means the MMA has released its A tile.
        const int r = (warp & 3) * 32 + lane;
        const int half = (warp - 2 - kEpiWarps) >> 2;        // which 32 codes of the 64
        const uint32_t row_off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
        unsigned char *sAp = basep + (sA - base);
        const unsigned char *sCp = basep + (sC - base);
        uint32_t it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const int s = it % STAGES;
                const bool ok = mbar_wait(full_bar(s), (it / STAGES) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0)
                        give_up(ERR_WAIT_FULL);
                    stop = true;
                    break;
                }
                if (__shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0)) {
                    stop = true;
                    break;
                }
                const uint4 c = *reinterpret_cast<const uint4 *>(
                    sCp + s * kCodeStageBytes + r * (BK / 2) + half * 16);
                const uint32_t words[4] = {c.x, c.y, c.z, c.w};
                unsigned char *dst = sAp + s * A_STAGE_BYTES + row_off;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = half * 4 + j;               // 16-byte piece of the row
                    uint32_t o[4];
                    decode8(words[j], p.L0, p.L1, p.H0, p.H1, o);
                    *reinterpret_cast<uint4 *>(dst + ((k ^ (r & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_async_smem();                           // visible to the tensor core
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(afull_bar(s));
            }
        }
    }
    __syncwarp();
    if (p.test_wait_cycles > 0 && blockIdx.x == 0 && threadIdx.x == 0)
        armed_test_wait(smem_u32(&test_bar), p.test_wait_cycles);
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------------------------------------
// CTA-pair GEMM (cluster of two CTAs on neighbouring SMs, tcgen05 .cta_group::2).  A pair
// computes a 256 x 256 output tile: per k-block each CTA loads its own 128 rows of A and its
// own 128 rows of B (outputs n0 + 128 * rank ...), and the leader CTA (rank 0) issues
// M = 256, N = 256 MMAs that read both CTAs' tiles, each CTA's tensor memory receiving its 128
// rows of the tile.  Per SM a k-block then brings in 32 KB instead of 48 KB for the same MMA
// time, and the ring holds 6 stages.  Barriers: the leader's full barrier counts both CTAs'
// TMA bytes (only the leader arms it); the leader's MMA commits release both CTAs' stages and
// signal both CTAs' accumulator-full barriers (multicast commit); every epilogue warp of both
// CTAs arrives on the leader's accumulator-empty barrier.  Every TMA load fills only its own
// CTA's shared memory.
// ------------------------------------------------------------------------------------------
// Codes (4-bit codes of a symmetric codebook, for the activations (kCodesA) or the weights
// (kCodesB)): each CTA's TMA brings the packed codes of its own 128 rows of that operand
// (128 x 32 bytes per k-block) into a code stage and signals its own barrier; eight decoder
// warps per CTA expand them into the operand's fp16 stage in the 128-byte swizzled layout the
// MMA reads and arrive on the leader's operand-ready barrier (16 arrivals: both CTAs'
// decoders).  The ring then holds 5 stages.  The stage's tile is free when its codes land,
// because the producer issued the code load only after the MMAs that last read the stage had
// completed.  A row of codes is decoded once per tile it takes part in: an activation row
// once per 256-column tile, a weight row once per 256-row tile.
// CODES of k2_gemm_pair: which operand arrives as 4-bit codes decoded in the kernel
constexpr int kCodesNone = 0, kCodesA = 1, kCodesB = 2;
template <bool ACODES>
__host__ __device__ constexpr int pair_stages() { return ACODES ? 5 : 6; }
constexpr int P_BM = 256, P_BN = 256;                    // pair tile
constexpr int P_A_BYTES = 128 * BK * 2;                  // 16 KB: this CTA's 128 rows of A
constexpr int P_B_BYTES = 128 * BK * 2;                  // 16 KB: this CTA's 128 rows of B
constexpr int P_STAGE_BYTES = P_A_BYTES + P_B_BYTES;
constexpr int P_CODE_BYTES = 128 * BK / 2;               // ACODES: 128 rows x 32 bytes
// barriers: full, empty, [ACODES: code-full, A-ready] per stage; 2 accumulator-full,
// 2 accumulator-empty, drain
template <bool ACODES>
__host__ __device__ constexpr int pair_num_bars() { return (ACODES ? 4 : 2) * pair_stages<ACODES>() + 5; }
template <bool ACODES>
__host__ __device__ constexpr int pair_threads() { return 32 * (2 + kEpiWarps + (ACODES ? kDecWarps : 0)); }
constexpr uint32_t kIdescPair = idesc_f16(P_BM, P_BN);

template <bool ACODES>
__host__ __device__ constexpr size_t gemm_pair_smem() {
    return 1024 + (size_t)pair_stages<ACODES>() * (P_STAGE_BYTES + (ACODES ? P_CODE_BYTES : 0)) +
           (size_t)kEpiWarps * 2 * kStageOut + 8 * pair_num_bars<ACODES>() + 8 +
           kEpiWarps * 64 * sizeof(float) + 64;
}
static_assert(gemm_pair_smem<false>() <= 227 * 1024 && gemm_pair_smem<true>() <= 227 * 1024,
              "shared memory budget (pair)");

// Warp roles as in k2_gemm: warp 0 lane 0 loads (both CTAs), warp 1 owns tensor memory (both
// CTAs allocate the same columns) and its lane 0 issues the MMAs (leader only), warps 2..5
// are the epilogue (both CTAs, each its own 128 rows), ACODES: warps 6..13 decode (both CTAs,
// each its own 128 rows).  Pair p takes tiles p, p + #pairs, ...
template <bool BF16, int CODES>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads<CODES != 0>(), 1)
    k2_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmP,
                 const GemmParams p) {
    constexpr bool ACODES = CODES != 0;             // one operand arrives as codes
    constexpr int S = pair_stages<ACODES>();
    constexpr int kBarSets = ACODES ? 4 : 2;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;                 // same offsets in both CTAs
    unsigned char *basep = smem_raw + (base - raw);
    const uint32_t sA = base, sB = base + S * P_A_BYTES;
    const uint32_t sC = sB + S * P_B_BYTES;                       // ACODES: code stages
    const uint32_t sOut = sC + (ACODES ? S * P_CODE_BYTES : 0);   // [4 warps][2][4 KB]
    const uint32_t bars = sOut + kEpiWarps * 2 * kStageOut;
    auto full_bar = [&](int s) { return bars + 8u * s; };                   // leader's is used
    auto empty_bar = [&](int s) { return bars + 8u * (S + s); };
    auto cfull_bar = [&](int s) { return bars + 8u * (2 * S + s); };        // ACODES, local
    auto afull_bar = [&](int s) { return bars + 8u * (3 * S + s); };        // ACODES, leader's
    auto tfull_bar = [&](int a) { return bars + 8u * (kBarSets * S + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (kBarSets * S + 2 + a); };   // leader's
    const uint32_t drain_bar = bars + 8u * (kBarSets * S + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(basep + (drain_bar + 8u - base));
    float *rn_s = reinterpret_cast<float *>(basep + (drain_bar + 16u - base));   // [4][64]
    __shared__ int abort_flag;
    __shared__ __align__(8) unsigned long long test_bar;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();                      // 0: the leader
    const int pair0 = (int)cluster_id_x(), npair = (int)cluster_count_x();
    const int n_tiles = (p.N + P_BN - 1) / P_BN;
    const int num_tiles = ((p.M + P_BM - 1) / P_BM) * n_tiles;
    const int num_kb = p.K / BK;
    // work units: a tile, or with ksplit > 1 (the plain form, few tiles) one of its ksplit
    // k-ranges of kb_per blocks, whose fp32 partial goes to tmP for k2_splitk_reduce
    const int ksplit = p.ksplit;
    const int num_units = num_tiles * ksplit;
    auto unit_range = [&](int unit, int &tile, int &part, int &kb0, int &kb1) {
        tile = unit / ksplit;
        part = unit - tile * ksplit;
        kb0 = part * p.kb_per;
        kb1 = min(num_kb, kb0 + p.kb_per);
    };

    pdl_trigger();
    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
            if constexpr (ACODES) {
                mbar_init(cfull_bar(s), 1);
                mbar_init(afull_bar(s), 2 * kDecWarps);
            }
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), 2 * kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        mbar_init(smem_u32(&test_bar), 2);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(kTmemCols) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync_all();                 // both CTAs' barriers initialised, tensor memory held
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                         // operands, s, rn and y: earlier work of the stream done
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };
    auto give_up = [&](unsigned bit) {
        atomicOr(&g_k2_err, bit);
        atomicExch(&abort_flag, 1);
    };

    if (warp == 0) {
        // ---------------- TMA producer (both CTAs) ----------------
        if (lane == 0) {
            uint32_t it = 0;
            for (int unit = pair0; unit < num_units && !aborted(); unit += npair) {
                int tile, part, kb0, kb1;
                unit_range(unit, tile, part, kb0, kb1);
                const int m0 = (tile / n_tiles) * P_BM + (int)rank * 128;
                const int n0 = (tile % n_tiles) * P_BN + (int)rank * 128;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (it >= S && !mbar_wait(empty_bar(s), ((it / S) & 1) ^ 1)) {
                        give_up(ERR_WAIT_EMPTY);
                        break;
                    }
                    if (aborted())
                        break;
                    const uint32_t fb = mapa_shared(full_bar(s), 0);
                    if constexpr (CODES == kCodesA) {
                        if (rank == 0)
                            mbar_expect_tx(full_bar(s), 2 * P_B_BYTES);
                        mbar_expect_tx(cfull_bar(s), P_CODE_BYTES);
                        tma_load_2d(sC + s * P_CODE_BYTES, &tmA, kb * (BK / 2), m0, cfull_bar(s));
                        tma_load_2d_pair(sB + s * P_B_BYTES, &tmB, kb * BK, n0, fb);
                    } else if constexpr (CODES == kCodesB) {
                        if (rank == 0)
                            mbar_expect_tx(full_bar(s), 2 * P_A_BYTES);
                        mbar_expect_tx(cfull_bar(s), P_CODE_BYTES);
                        tma_load_2d_pair(sA + s * P_A_BYTES, &tmA, kb * BK, m0, fb);
                        tma_load_2d(sC + s * P_CODE_BYTES, &tmB, kb * (BK / 2), n0, cfull_bar(s));
                    } else {
                        if (rank == 0)
                            mbar_expect_tx(full_bar(s), 2 * P_STAGE_BYTES);
                        tma_load_2d_pair(sA + s * P_A_BYTES, &tmA, kb * BK, m0, fb);
                        tma_load_2d_pair(sB + s * P_B_BYTES, &tmB, kb * BK, n0, fb);
                    }
                }
            }
            if (aborted()) {
                // let the loads already issued land before the pair can exit
                const uint32_t from = it > (uint32_t)S ? it - S : 0;
                for (uint32_t j = from; j < it; ++j) {
                    if (rank == 0)
                        mbar_wait(full_bar(j % S), (j / S) & 1);
                    if (ACODES)
                        mbar_wait(cfull_bar(j % S), (j / S) & 1);
                }
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (leader) ----------------
        if (lane == 0 && rank == 0) {
            uint32_t it = 0;
            int i = 0;
            for (int unit = pair0; unit < num_units && !aborted(); unit += npair, ++i) {
                int tile, part, kb0, kb1;
                unit_range(unit, tile, part, kb0, kb1);
                const int acc = i & 1;
                if (i >= 2 && !mbar_wait(tempty_bar(acc), ((i >> 1) & 1) ^ 1)) {
                    give_up(ERR_WAIT_EMPTY);
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + (uint32_t)(acc * kAccCols);
                bool ok = true;
                for (int kb = kb0; kb < kb1; ++kb, ++it) {
                    const int s = it % S;
                    if (!mbar_wait(full_bar(s), (it / S) & 1) ||
                        (ACODES && !mbar_wait(afull_bar(s), (it / S) & 1))) {
                        give_up(ERR_WAIT_FULL);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sw128_desc(sA + s * P_A_BYTES);
                    const uint64_t db = sw128_desc(sB + s * P_B_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_ss_pair(d_tmem, da + 2 * kk, db + 2 * kk, kIdescPair,
                                    (kb != kb0) || (kk != 0));
                    mma_commit_pair_mc(empty_bar(s), 0x3);
                }
                if (!ok)
                    break;
                mma_commit_pair_mc(tfull_bar(acc), 0x3);
            }
            mma_commit_pair_mc(drain_bar, 0x1);
            if (!mbar_wait(drain_bar, 0))
                atomicOr(&g_k2_err, ERR_WAIT_ACCUM);
        }
    } else if (warp < 2 + kEpiWarps) {
        // ---------------- epilogue (both CTAs): this CTA's 128 rows of the tile ----------
        const int q = warp & 3;                               // TMEM lane quarter
        float *rn_w = rn_s + (warp - 2) * 64;
        const uint32_t out0 = sOut + (uint32_t)((warp - 2) * 2 * kStageOut);
        unsigned char *out0p = basep + (out0 - base);
        uint32_t u = 0;
        int i = 0;
        for (int unit = pair0; unit < num_units; unit += npair, ++i) {
            int tile, part, kb0, kb1;
            unit_range(unit, tile, part, kb0, kb1);
            const int acc = i & 1;
            const int m0 = (tile / n_tiles) * P_BM + (int)rank * 128;
            const int n0 = (tile % n_tiles) * P_BN;
            const int row = m0 + q * 32 + lane;
            const float srow = (row < p.M) ? p.s[row] * p.inv_d : 0.f;
            float rnv[P_BN / 32];
#pragma unroll
            for (int c = 0; c < P_BN / 32; ++c) {
                const int col = n0 + c * 32 + lane;
                rnv[c] = (col < p.N) ? p.rn[col] : 0.f;
            }
            const bool ok = mbar_wait(tfull_bar(acc), (i >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (!ok)
                    give_up(ERR_WAIT_ACCUM);
                break;
            }
            tc_fence_after();
            const uint32_t t_base =
                tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols);
            const bool rows_in = m0 + q * 32 < p.M;
            constexpr int kCW = BF16 ? 64 : 32;
#pragma unroll
            for (int c = 0; c < P_BN / kCW; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_base + (uint32_t)(c * kCW), r0);
                if constexpr (BF16)
                    tmem_ld32(t_base + (uint32_t)(c * kCW + 32), r1);
                if (!rows_in || n0 + c * kCW >= p.N)
                    continue;
                if (ksplit > 1) {
                    // the unscaled fp32 partial of this k-range: rows part * m_pad + row of
                    // tmP (x 1 x 1 in store_chunk is exact); bf16 y: two 32-column chunks
#pragma unroll
                    for (int h = 0; h < kCW / 32; ++h) {
                        const uint32_t b = u & 1;
                        if (lane == 0)
                            bulk_wait_read<1>();
                        __syncwarp();
                        rn_w[lane] = 1.0f;
                        __syncwarp();
                        store_chunk(&tmP, out0p + b * kStageOut, out0 + b * kStageOut,
                                    h == 0 ? r0 : r1, 1.0f, rn_w, lane, n0 + c * kCW + 32 * h,
                                    part * p.m_pad + m0 + q * 32);
                        ++u;
                    }
                    continue;
                }
                const uint32_t b = u & 1;
                if (lane == 0)
                    bulk_wait_read<1>();
                __syncwarp();
                if constexpr (BF16) {
                    rn_w[lane] = rnv[2 * c];
                    rn_w[32 + lane] = rnv[2 * c + 1];
                } else {
                    rn_w[lane] = rnv[c];
                }
                __syncwarp();
                if constexpr (BF16)
                    store_chunk_bf16(&tmY, out0p + b * kStageOut, out0 + b * kStageOut, r0, r1,
                                     srow, rn_w, lane, n0 + c * kCW, m0 + q * 32);
                else
                    store_chunk(&tmY, out0p + b * kStageOut, out0 + b * kStageOut, r0, srow,
                                rn_w, lane, n0 + c * kCW, m0 + q * 32);
                ++u;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(mapa_shared(tempty_bar(acc), 0));
        }
        if (lane == 0)
            bulk_wait_all();
    } else if constexpr (ACODES) {
        // ---------------- decoders (both CTAs): 4-bit codes -> this CTA's fp16 stages of the
        // coded operand (A rows or B rows) ----
        // Thread = row r of this CTA's 128 rows and one half of its 64 codes per k-block: 16
        // bytes of codes in, 64 bytes of the fp16 row out in the 128-byte swizzled layout
        // (16-byte piece k of row r at piece k ^ (r % 8), 8-row atoms of 1024 bytes).
        const int r = (warp & 3) * 32 + lane;
        const int half = (warp - 2 - kEpiWarps) >> 2;
        const uint32_t row_off = (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
        unsigned char *sAp = basep + ((CODES == kCodesA ? sA : sB) - base);
        const unsigned char *sCp = basep + (sC - base);
        const uint32_t ready = rank == 0 ? 0u : 1u;
        uint32_t it = 0;
        bool stop = false;
        for (int unit = pair0; unit < num_units && !stop; unit += npair) {
            int tile, part, kb0, kb1;
            unit_range(unit, tile, part, kb0, kb1);
            for (int kb = kb0; kb < kb1; ++kb, ++it) {
                const int s = it % S;
                const bool ok = mbar_wait(cfull_bar(s), (it / S) & 1);
                if (!__all_sync(0xffffffffu, ok)) {
                    if (lane == 0)
                        give_up(ERR_WAIT_FULL);
                    stop = true;
                    break;
                }
                if (__shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0)) {
                    stop = true;
                    break;
                }
                const uint4 c = *reinterpret_cast<const uint4 *>(
                    sCp + s * P_CODE_BYTES + r * (BK / 2) + half * 16);
                const uint32_t words[4] = {c.x, c.y, c.z, c.w};
                unsigned char *dst = sAp + s * P_A_BYTES + row_off;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int k = half * 4 + j;               // 16-byte piece of the row
                    uint32_t o[4];
                    decode8(words[j], p.L0, p.L1, p.H0, p.H1, o);
                    *reinterpret_cast<uint4 *>(dst + ((k ^ (r & 7)) << 4)) =
                        make_uint4(o[0], o[1], o[2], o[3]);
                }
                fence_async_smem();                           // visible to the tensor core
                __syncwarp();
                if (lane == 0) {
                    if (ready == 0)
                        mbar_arrive(afull_bar(s));
                    else
                        mbar_arrive_remote(mapa_shared(afull_bar(s), 0));
                }
            }
        }
    }
    __syncwarp();
    if (p.test_wait_cycles > 0 && blockIdx.x == 0 && threadIdx.x == 0)
        armed_test_wait(smem_u32(&test_bar), p.test_wait_cycles);
    tc_fence_before();
    cluster_sync_all();                 // no MMA, load or arrive of the pair is still pending
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// The epilogue of a K-split pair GEMM: y = (the ksplit fp32 partials summed in order) *
// (s[row] / d) * rn[col], the same expression as the one-pass epilogue, fp32 or bf16 (round to
// nearest even).  One thread per 4 consecutive columns of a row; partial k of row r at
// part + (k * m_pad + r) * N.
template <bool BF16>
__global__ void __launch_bounds__(256) k2_splitk_reduce(const float *part, int ksplit,
                                                        const GemmParams p) {
    pdl_trigger();
    pdl_wait();
    const int n4 = p.N / 4;
    const long long total = (long long)p.M * n4;
    const size_t part_stride = (size_t)p.m_pad * p.N;
    for (long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (long long)gridDim.x * blockDim.x) {
        const int row = (int)(idx / n4), c4 = (int)(idx - (long long)row * n4);
        const float *src = part + (size_t)row * p.N + 4 * (size_t)c4;
        float4 a = *reinterpret_cast<const float4 *>(src);
        for (int k = 1; k < ksplit; ++k) {
            const float4 b = *reinterpret_cast<const float4 *>(src + k * part_stride);
            a.x += b.x;
            a.y += b.y;
            a.z += b.z;
            a.w += b.w;
        }
        const float srow = p.s[row] * p.inv_d;
        const float *rn = p.rn + 4 * (size_t)c4;
        const float o0 = a.x * srow * rn[0], o1 = a.y * srow * rn[1];
        const float o2 = a.z * srow * rn[2], o3 = a.w * srow * rn[3];
        const size_t off = (size_t)row * p.N + 4 * (size_t)c4;
        if constexpr (BF16) {
            const __nv_bfloat162 h0 = __floats2bfloat162_rn(o0, o1);
            const __nv_bfloat162 h1 = __floats2bfloat162_rn(o2, o3);
            *reinterpret_cast<uint2 *>(static_cast<__nv_bfloat16 *>(p.y) + off) =
                make_uint2(*reinterpret_cast<const uint32_t *>(&h0),
                           *reinterpret_cast<const uint32_t *>(&h1));
        } else {
            *reinterpret_cast<float4 *>(static_cast<float *>(p.y) + off) =
                make_float4(o0, o1, o2, o3);
        }
    }
}

// ------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------
// Encoded tensor maps, kept per host thread: a map is a pure function of its arguments, so a
// call with the same buffer and shape (the usual case for a layer called again and again)
// reuses the encoding instead of paying for cuTensorMapEncodeTiled on every call.
struct MapKey {
    const void *ptr;
    long long rows;
    int cols, box, kind;
    bool operator==(const MapKey &o) const {
        return ptr == o.ptr && rows == o.rows && cols == o.cols && box == o.box && kind == o.kind;
    }
};
constexpr int kMapCacheSize = 16;
thread_local MapKey g_map_keys[kMapCacheSize];
thread_local CUtensorMap g_maps[kMapCacheSize];
thread_local int g_map_used = 0, g_map_next = 0;

template <class Encode>
bool cached_map(CUtensorMap *map, const MapKey &key, Encode &&encode) {
    for (int i = 0; i < g_map_used; ++i)
        if (g_map_keys[i] == key) {
            *map = g_maps[i];
            return true;
        }
    if (!encode(map))
        return false;
    const int slot = g_map_used < kMapCacheSize ? g_map_used++ : g_map_next;
    g_map_next = (slot + 1) % kMapCacheSize;
    g_map_keys[slot] = key;
    g_maps[slot] = *map;
    return true;
}

// fp16 [rows, K] row-major -> tiles of box_rows x 64 with 128-byte swizzle.
bool make_map_uncached(CUtensorMap *map, const void *ptr, long long rows, int K, int box_rows) {
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(ptr), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_map(CUtensorMap *map, const void *ptr, long long rows, int K, int box_rows) {
    return cached_map(map, MapKey{ptr, rows, K, box_rows, 0},
                      [&](CUtensorMap *m) { return make_map_uncached(m, ptr, rows, K, box_rows); });
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

bool make_out_map_uncached(CUtensorMap *map, void *y, int T, int N, bool bf16) {
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    const int esize = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)T};
    cuuint64_t strides[1] = {(cuuint64_t)N * esize};
    cuuint32_t box[2] = {(cuuint32_t)(128 / esize), 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                    2, y, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_out_map(CUtensorMap *map, void *y, int T, int N, bool bf16) {
    return cached_map(map, MapKey{y, T, N, 0, bf16 ? 2 : 1},
                      [&](CUtensorMap *m) { return make_out_map_uncached(m, y, T, N, bf16); });
}

size_t linear_workspace_bytes(int T, int d, int N) {
    return align_up((size_t)T * d * 2, 1024) + align_up((size_t)N * d * 2, 1024);
}

size_t linear_workspace_b_offset(int T, int d) { return align_up((size_t)T * d * 2, 1024); }

namespace {

// 4-bit codes, uint8 [rows, K/2] row-major -> 128-row x 32-byte boxes (one k-block), no
// swizzle.
bool make_code_map_uncached(CUtensorMap *map, const uint8_t *codes, long long rows, int K) {
    auto fn = tensor_map_encoder();
    if (!fn)
        return false;
    cuuint64_t dims[2] = {(cuuint64_t)K / 2, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K / 2};
    cuuint32_t box[2] = {(cuuint32_t)(BK / 2), (cuuint32_t)BM};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_code_map(CUtensorMap *map, const uint8_t *codes, long long rows, int K) {
    return cached_map(map, MapKey{codes, rows, K, 0, 3},
                      [&](CUtensorMap *m) { return make_code_map_uncached(m, codes, rows, K); });
}

template <bool BF16, bool ACODES>
cudaError_t launch_gemm_t(const CUtensorMap &ma, const CUtensorMap &mb, const CUtensorMap &my,
                          const GemmParams &gp, int grid, cudaStream_t st, std::string *why) {
    auto kern = k2_gemm<BF16, ACODES>;
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices))
        e = cudaErrorInvalidDevice;
    if (e == cudaSuccess) {
        std::lock_guard<std::mutex> lk(mu);
        if (!done[dev]) {        // once per device and instantiation
            e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     (int)gemm_smem<ACODES>());
            done[dev] = (e == cudaSuccess);
        }
    }
    if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(k2_gemm)";
        return e;
    }
    e = launch_pdl(kern, dim3(grid), dim3(gemm_threads<ACODES>()), gemm_smem<ACODES>(), st, ma, mb,
                   my, gp);
    if (e != cudaSuccess)
        *why = "k2_gemm launch";
    return e;
}

// Pairs of the CTA-pair GEMM that fit on the device at once (0: the form is unavailable),
// once per device and instantiation.
template <bool BF16, int CODES>
int gemm_pair_slots() {
    constexpr bool ACODES = CODES != kCodesNone;
    static std::mutex mu;
    static int slots[kMaxDevices];
    static bool done[kMaxDevices] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (!done[dev]) {
        done[dev] = true;
        slots[dev] = 0;
        auto kern = k2_gemm_pair<BF16, CODES>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)gemm_pair_smem<ACODES>()) != cudaSuccess) {
            cudaGetLastError();
            return 0;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(pair_threads<ACODES>(), 1, 1);
        cfg.dynamicSmemBytes = gemm_pair_smem<ACODES>();
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        slots[dev] = n;
    }
    return slots[dev];
}

template <bool BF16, int CODES>
cudaError_t launch_gemm_pair_t(const CUtensorMap &ma, const CUtensorMap &mb,
                               const CUtensorMap &my, const CUtensorMap &mp,
                               const GemmParams &gp, int pairs, cudaStream_t st,
                               std::string *why) {
    constexpr bool ACODES = CODES != kCodesNone;
    const cudaError_t e =
        launch_pdl(k2_gemm_pair<BF16, CODES>, dim3(2 * pairs), dim3(pair_threads<ACODES>()),
                   gemm_pair_smem<ACODES>(), st, ma, mb, my, mp, gp);
    if (e != cudaSuccess)
        *why = "k2_gemm_pair launch";
    return e;
}

}  // namespace

// The CTA-pair GEMM is used when the device can hold it; OQ_GEMM_PAIR=0 selects the
// single-CTA kernel (read once per process).
bool gemm_pair_enabled() {
    static const bool on = [] {
        const char *v = std::getenv("OQ_GEMM_PAIR");
        return !(v && v[0] == '0');
    }();
    return on;
}

cudaError_t launch_gemm(const uint16_t *A16, const uint8_t *x_codes4, const uint16_t *lut_a,
                        const uint16_t *B16, const uint8_t *w_codes4, const uint16_t *lut_w,
                        const float *s, const float *rn, void *y, bool y_bf16, int T, int N,
                        int d, cudaStream_t st, int num_sms, std::string *why,
                        long long test_wait_cycles, void *split_ws, size_t split_ws_bytes) {
    const bool acodes = A16 == nullptr, wcodes = B16 == nullptr;
    GemmParams gp;
    gp.test_wait_cycles = test_wait_cycles;
    gp.s = s;
    gp.rn = rn;
    gp.L0 = gp.L1 = gp.H0 = gp.H1 = 0;
    gp.M = T;
    gp.N = N;
    gp.K = d;
    gp.inv_d = 1.0f / (float)d;
    gp.ksplit = 1;
    gp.kb_per = d / BK;
    gp.m_pad = 0;
    gp.y = y;
    if (acodes && wcodes) {
        *why = "k2_gemm: at most one operand can arrive as codes";
        return cudaErrorInvalidValue;
    }
    if (acodes && (!x_codes4 || !lut_a ||
                   !decode8_sources(lut_a, &gp.L0, &gp.L1, &gp.H0, &gp.H1))) {
        *why = "k2_gemm: activation codes need a 4-bit odd-symmetric codebook";
        return cudaErrorInvalidValue;
    }
    if (wcodes && (!w_codes4 || !lut_w ||
                   !decode8_sources(lut_w, &gp.L0, &gp.L1, &gp.H0, &gp.H1))) {
        *why = "k2_gemm: weight codes need a 4-bit odd-symmetric codebook";
        return cudaErrorInvalidValue;
    }
    CUtensorMap ma, mb, my;
    if (gemm_pair_enabled()) {
        const int slots =
            acodes ? (y_bf16 ? gemm_pair_slots<true, kCodesA>() : gemm_pair_slots<false, kCodesA>())
            : wcodes ? (y_bf16 ? gemm_pair_slots<true, kCodesB>()
                               : gemm_pair_slots<false, kCodesB>())
                     : (y_bf16 ? gemm_pair_slots<true, kCodesNone>()
                               : gemm_pair_slots<false, kCodesNone>());
        if (slots > 0) {
            const bool a_ok = acodes ? make_code_map(&ma, x_codes4, T, d)
                                     : make_map(&ma, A16, T, d, 128);
            const bool b_ok = wcodes ? make_code_map(&mb, w_codes4, N, d)
                                     : make_map(&mb, B16, N, d, 128);
            if (!a_ok || !b_ok || !make_out_map(&my, y, T, N, y_bf16)) {
                *why = "cuTensorMapEncodeTiled failed";
                return cudaErrorInvalidValue;
            }
            const int m_tiles = (T + P_BM - 1) / P_BM;
            const int tiles = ((N + P_BN - 1) / P_BN) * m_tiles;
            // Few tiles (small T): split each tile's K loop over ksplit work units, so that
            // more CTA pairs work; their fp32 partials are summed by k2_splitk_reduce.
            // (decided on the plain kernel's pair count, so that every operand form splits the
            // same way and gives the same bits)
            const int num_kb = d / BK;
            const int plain = y_bf16 ? gemm_pair_slots<true, kCodesNone>()
                                     : gemm_pair_slots<false, kCodesNone>();
            int ksplit = 1;
            if (plain > 0 && tiles * 2 <= plain && num_kb >= 8) {
                ksplit = std::min(std::min(plain / tiles, num_kb / 4), 8);
                if (ksplit >= 2) {
                    gp.kb_per = (num_kb + ksplit - 1) / ksplit;
                    ksplit = (num_kb + gp.kb_per - 1) / gp.kb_per;
                }
            }
            auto go = [&](const CUtensorMap &mp, int pairs) -> cudaError_t {
                if (acodes)
                    return y_bf16 ? launch_gemm_pair_t<true, kCodesA>(ma, mb, my, mp, gp, pairs,
                                                                      st, why)
                                  : launch_gemm_pair_t<false, kCodesA>(ma, mb, my, mp, gp,
                                                                       pairs, st, why);
                if (wcodes)
                    return y_bf16 ? launch_gemm_pair_t<true, kCodesB>(ma, mb, my, mp, gp, pairs,
                                                                      st, why)
                                  : launch_gemm_pair_t<false, kCodesB>(ma, mb, my, mp, gp,
                                                                       pairs, st, why);
                return y_bf16 ? launch_gemm_pair_t<true, kCodesNone>(ma, mb, my, mp, gp, pairs,
                                                                     st, why)
                              : launch_gemm_pair_t<false, kCodesNone>(ma, mb, my, mp, gp, pairs,
                                                                      st, why);
            };
            if (ksplit < 2) {
                gp.kb_per = num_kb;
                return go(my, tiles < slots ? tiles : slots);
            }
            gp.ksplit = ksplit;
            gp.m_pad = m_tiles * P_BM;
            const size_t part_bytes = (size_t)ksplit * gp.m_pad * N * 4;
            void *part = split_ws;
            cudaError_t e = cudaSuccess;
            if (split_ws) {
                if (part_bytes > split_ws_bytes) {
                    *why = "k2_gemm: split-K partials exceed the given workspace";
                    return cudaErrorInvalidValue;
                }
            } else {
                e = cudaMallocAsync(&part, part_bytes, st);
                if (e != cudaSuccess) {
                    *why = "k2_gemm: split-K partial buffer";
                    return e;
                }
            }
            CUtensorMap mp;
            if (!make_out_map(&mp, part, ksplit * gp.m_pad, N, false)) {
                if (!split_ws)
                    cudaFreeAsync(part, st);
                *why = "cuTensorMapEncodeTiled failed";
                return cudaErrorInvalidValue;
            }
            const int units = tiles * ksplit;
            e = go(mp, units < slots ? units : slots);
            if (e == cudaSuccess) {
                const long long work = (long long)T * (N / 4);
                long long blocks = (work + 255) / 256;
                if (blocks > (long long)num_sms * 8)
                    blocks = (long long)num_sms * 8;
                e = y_bf16 ? launch_pdl(k2_splitk_reduce<true>, dim3((unsigned)blocks), dim3(256),
                                        0, st, static_cast<const float *>(part), ksplit, gp)
                           : launch_pdl(k2_splitk_reduce<false>, dim3((unsigned)blocks),
                                        dim3(256), 0, st, static_cast<const float *>(part),
                                        ksplit, gp);
                if (e != cudaSuccess)
                    *why = "k2_splitk_reduce launch";
            }
            const cudaError_t e2 = split_ws ? cudaSuccess : cudaFreeAsync(part, st);
            return e != cudaSuccess ? e : e2;
        }
    }
    if (wcodes) {
        *why = "k2_gemm: weight codes are decoded by the CTA-pair GEMM only";
        return cudaErrorInvalidValue;
    }
    const bool a_ok = acodes ? make_code_map(&ma, x_codes4, T, d) : make_map(&ma, A16, T, d, BM);
    if (!a_ok || !make_map(&mb, B16, N, d, BN) || !make_out_map(&my, y, T, N, y_bf16)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const int tiles = ((N + BN - 1) / BN) * ((T + BM - 1) / BM);
    const int grid = tiles < num_sms ? tiles : num_sms;
    if (acodes)
        return y_bf16 ? launch_gemm_t<true, true>(ma, mb, my, gp, grid, st, why)
                      : launch_gemm_t<false, true>(ma, mb, my, gp, grid, st, why);
    return y_bf16 ? launch_gemm_t<true, false>(ma, mb, my, gp, grid, st, why)
                  : launch_gemm_t<false, false>(ma, mb, my, gp, grid, st, why);
}

bool gemm_splits_k(int T, int N, int d, bool y_bf16) {
    if (!gemm_pair_enabled())
        return false;
    const int plain = y_bf16 ? gemm_pair_slots<true, kCodesNone>()
                             : gemm_pair_slots<false, kCodesNone>();
    const int tiles = ((N + P_BN - 1) / P_BN) * ((T + P_BM - 1) / P_BM);
    const int num_kb = d / BK;
    return plain > 0 && tiles * 2 <= plain && num_kb >= 8 &&
           std::min(std::min(plain / tiles, num_kb / 4), 8) >= 2;
}

bool make_operand_map(CUtensorMap *map, const void *ptr, long long rows, int K) {
    return make_map(map, ptr, rows, K, 128);
}

size_t noalloc_workspace_bytes() { return kNoAllocWorkspaceBytes; }
size_t noalloc_split_bytes() { return kNoAllocSplitBytes; }

cudaError_t noalloc_workspace(void **out) {
    static std::mutex mu;
    static void *addr[kMaxDevices] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_workspace);   // the current device's copy
        if (e != cudaSuccess)
            return e;
        addr[dev] = p;
    }
    *out = addr[dev];
    return cudaSuccess;
}

cudaError_t read_and_clear_k2_error(unsigned *out, cudaStream_t st) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_k2_err, sizeof(unsigned), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_k2_err, &zero, sizeof(unsigned), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace oq
