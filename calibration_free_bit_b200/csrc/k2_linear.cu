// k2_linear.cu -- codebook linear layer on sm_100a: y = (s_t rn_o / d) * sum_k Ca[xc] Cw[wc].
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video":
// rotation-cancellation paragraph (W R^T R x = W x, so codes of R x and of R w meet directly)
// and the pseudocode's x_hat = s * codebook[xc], W_hat = diag(row_norms) * codebook[wc]; its
// speed-caveat paragraph notes that non-uniform centroids cannot feed integer tensor cores,
// which is why the codes are decoded to fp16 unit centroids before the MMA.
//
// Path: (1) decode prepass: packed codes -> fp16 unit-variance centroids (LUT), for the
// activation codes and the weight codes, into stream-ordered workspace; (2) a hand-written
// persistent tcgen05 GEMM: TMA (128B swizzle) brings fp16 K-major tiles into a 4-stage
// shared-memory ring, one elected thread issues tcgen05.mma kind::f16 (M=128, N=256, K=16)
// into one of two TMEM fp32 accumulators (2 x 256 columns), and 4 epilogue warps read the
// other accumulator back with tcgen05.ld and apply the s_t * rn_o / d scale.  sigma^2 = 1/d is folded into the epilogue so the
// fp16 values are unit-variance (best fp16 precision).  Every mbarrier wait is bounded by
// wall time (%globaltimer); a wait that gives up sets a bit in the device error word.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "oq_internal.h"

namespace oq {
namespace {

__device__ unsigned int g_k2_err;

// Fixed workspace for oq_linear_noalloc: the fp16 operand buffers live here instead of in
// memory the library allocates.  Every GPU that loads the library holds this array until the
// process exits.  Host code must not use the symbol as an address (it is a host-side stand-in);
// noalloc_workspace() looks the device address up once per device.
constexpr size_t kNoAllocWorkspaceBytes = 64ull << 20;
static __device__ __align__(256) unsigned char g_noalloc_workspace[kNoAllocWorkspaceBytes];

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE_BYTES = BM * BK * 2;               // 16 KB
constexpr int B_STAGE_BYTES = BN * BK * 2;               // 32 KB
constexpr int STAGE_BYTES = A_STAGE_BYTES + B_STAGE_BYTES;
constexpr int TMEM_COLS = BN;                            // fp32 accumulator, one column per n
constexpr unsigned long long kWaitLimitNs = 2000000000ull;   // 2 s per wait

enum : unsigned {
    ERR_WAIT_FULL = 1u << 0,
    ERR_WAIT_EMPTY = 1u << 1,
    ERR_WAIT_ACCUM = 1u << 2,
};

// ------------------------------------------------------------------------------------------
// Decode prepass: 8 codes per thread-iteration -> 8 fp16 unit centroids (16 bytes).
// ------------------------------------------------------------------------------------------
struct DecodeParams {
    const uint8_t *codes;
    uint16_t *out;
    long long rows;
    int d;
    uint16_t lut[256];
};

template <int BITS>
__global__ void __launch_bounds__(256) k2_decode(const __grid_constant__ DecodeParams p) {
    __shared__ uint16_t lut[256];
    for (int i = threadIdx.x; i < (1 << BITS); i += blockDim.x)
        lut[i] = p.lut[i];
    __syncthreads();
    const long long per_row = p.d / 8;
    const long long total = p.rows * per_row;
    const size_t row_bytes = (size_t)p.d * BITS / 8;
    for (long long c = (long long)blockIdx.x * blockDim.x + threadIdx.x; c < total;
         c += (long long)gridDim.x * blockDim.x) {
        const long long row = c / per_row, col8 = c - row * per_row;
        const uint8_t *src = p.codes + row * row_bytes + col8 * BITS;   // 8 codes = BITS bytes
        uint64_t bits;
        if constexpr (BITS == 2)
            bits = *reinterpret_cast<const uint16_t *>(src);
        else if constexpr (BITS == 4)
            bits = *reinterpret_cast<const uint32_t *>(src);
        else if constexpr (BITS == 8)
            bits = *reinterpret_cast<const uint64_t *>(src);
        else
            bits = (uint64_t)src[0] | ((uint64_t)src[1] << 8) | ((uint64_t)src[2] << 16);
        uint32_t h[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
            h[i] = lut[(bits >> (i * BITS)) & ((1u << BITS) - 1)];
        uint4 o = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16),
                             h[6] | (h[7] << 16));
        *reinterpret_cast<uint4 *>(p.out + row * p.d + col8 * 8) = o;
    }
}

// ------------------------------------------------------------------------------------------
// tcgen05 GEMM helpers (inline PTX).
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ unsigned long long globaltimer() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

// Wait for the phase with the given parity to complete; false after kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    const unsigned long long t0 = globaltimer();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(done) : "r"(bar), "r"(parity) : "memory");
        if (done)
            return true;
        if (globaltimer() - t0 > kWaitLimitNs)
            return false;
    }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// K-major operand in the canonical 128-byte-swizzled layout (8-row atoms of 1024 bytes).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    return (uint64_t)((saddr >> 4) & 0x3FFFu)     // start address
           | ((uint64_t)1 << 16)                  // leading byte offset (unused for SW128 K)
           | ((uint64_t)(1024 >> 4) << 32)        // stride byte offset: next 8-row atom
           | ((uint64_t)1 << 46)                  // descriptor version (sm_100)
           | ((uint64_t)2 << 61);                 // swizzle mode: 128B
}

// Instruction descriptor: kind::f16, A = B = fp16 (K-major), D = fp32, M = BM, N = BN.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_f16(uint32_t tmem_d, uint64_t da, uint64_t db,
                                        uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(tmem_d), "l"(da), "l"(db), "r"(kIdesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, "
        "[%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

struct GemmParams {
    const float *s;
    const float *rn;
    float *y;
    int M, N, K;
    float inv_d;
};

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

constexpr int kThreads = 192;        // 6 warps
constexpr int kEpiWarps = 4;         // warps 2..5
constexpr int kAccCols = BN;         // one fp32 accumulator: 256 TMEM columns
constexpr int kTmemCols = 2 * kAccCols;

// Persistent, warp-specialised tcgen05 GEMM.  Warp 0 lane 0: TMA producer over a 4-stage
// shared-memory ring.  Warp 1: TMEM owner; its lane 0 issues the MMAs.  Warps 2..5: epilogue
// (TMEM lane quarter = warp % 4).  Two 256-column accumulators alternate between tiles, so the
// epilogue of one tile overlaps the mainloop of the next.  Tiles are walked n-fastest so
// consecutive CTAs share the same 128-row A block in L2.
__global__ void __launch_bounds__(kThreads, 1)
    k2_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const GemmParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;                 // 1 KB aligned tiles
    unsigned char *basep = smem_raw + (base - raw);
    const uint32_t sA = base, sB = base + STAGES * A_STAGE_BYTES;
    const uint32_t bars = sB + STAGES * B_STAGE_BYTES;
    auto full_bar = [&](int s) { return bars + 8u * s; };
    auto empty_bar = [&](int s) { return bars + 8u * (STAGES + s); };
    auto tfull_bar = [&](int a) { return bars + 8u * (2 * STAGES + a); };
    auto tempty_bar = [&](int a) { return bars + 8u * (2 * STAGES + 2 + a); };
    const uint32_t drain_bar = bars + 8u * (2 * STAGES + 4);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(basep + (drain_bar + 8u - base));
    float *rn_s = reinterpret_cast<float *>(basep + (drain_bar + 16u - base));   // [4][BN]
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + BN - 1) / BN;
    const int num_tiles = ((p.M + BM - 1) / BM) * n_tiles;
    const int num_kb = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(tfull_bar(a), 1);
            mbar_init(tempty_bar(a), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
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
                    mbar_expect_tx(full_bar(s), STAGE_BYTES);
                    tma_load_2d(sA + s * A_STAGE_BYTES, &tmA, kb * BK, m0, full_bar(s));
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
                    if (!mbar_wait(full_bar(s), (it / STAGES) & 1)) {
                        give_up(ERR_WAIT_FULL);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t da = sw128_desc(sA + s * A_STAGE_BYTES);
                    const uint64_t db = sw128_desc(sB + s * B_STAGE_BYTES);
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)   // 16 fp16 = 32 bytes = 2 desc units
                        mma_f16(d_tmem, da + 2 * kk, db + 2 * kk, (kb | kk) != 0);
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
    } else {
        // ---------------- epilogue: TMEM -> registers -> scale -> global ----------------
        // Each epilogue warp keeps its own copy of the tile's row norms (no cross-warp barrier,
        // so one warp giving up a wait cannot strand the others).
        const int q = warp & 3;                               // TMEM lane quarter
        float *rn_t = rn_s + (warp - 2) * BN;
        int i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int acc = i & 1;
            const int m0 = (tile / n_tiles) * BM, n0 = (tile % n_tiles) * BN;
            __syncwarp();                                     // previous tile's reads are done
            for (int j = lane; j < BN; j += 32)
                rn_t[j] = (n0 + j < p.N) ? p.rn[n0 + j] : 0.f;
            __syncwarp();
            const bool ok = mbar_wait(tfull_bar(acc), (i >> 1) & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (!ok)
                    give_up(ERR_WAIT_ACCUM);
                break;
            }
            tc_fence_after();
            const int row = m0 + q * 32 + lane;
            const float srow = (row < p.M) ? p.s[row] * p.inv_d : 0.f;
            float *yrow = p.y + (size_t)row * p.N + n0;
            const uint32_t t_base =
                tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * kAccCols);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t_base + (uint32_t)(c * 32), r);
                if (row < p.M) {
#pragma unroll
                    for (int j = 0; j < 32; j += 4) {
                        const int col = c * 32 + j;
                        if (n0 + col < p.N) {
                            const float4 rn4 = *reinterpret_cast<const float4 *>(rn_t + col);
                            float4 o;
                            o.x = __uint_as_float(r[j + 0]) * srow * rn4.x;
                            o.y = __uint_as_float(r[j + 1]) * srow * rn4.y;
                            o.z = __uint_as_float(r[j + 2]) * srow * rn4.z;
                            o.w = __uint_as_float(r[j + 3]) * srow * rn4.w;
                            *reinterpret_cast<float4 *>(yrow + col) = o;
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(tempty_bar(acc));
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(kTmemCols) : "memory");
    }
}

// ------------------------------------------------------------------------------------------
// Host side.
// ------------------------------------------------------------------------------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

// fp16 [rows, K] row-major -> tiles of box_rows x 64 with 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *ptr, long long rows, int K, int box_rows) {
    auto fn = encode_fn();
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

template <int BITS>
cudaError_t decode(const uint8_t *codes, uint16_t *out, long long rows, int d,
                   const uint16_t *lut, cudaStream_t st, int num_sms) {
    DecodeParams dp;
    dp.codes = codes;
    dp.out = out;
    dp.rows = rows;
    dp.d = d;
    for (int i = 0; i < 256; ++i)
        dp.lut[i] = lut[i];
    const long long total = rows * (d / 8);
    long long blocks = (total + 255) / 256;
    const long long cap = (long long)num_sms * 8;
    if (blocks > cap)
        blocks = cap;
    if (blocks < 1)
        blocks = 1;
    k2_decode<BITS><<<(unsigned)blocks, 256, 0, st>>>(dp);
    return cudaGetLastError();
}

cudaError_t decode_any(int bits, const uint8_t *codes, uint16_t *out, long long rows, int d,
                       const uint16_t *lut, cudaStream_t st, int num_sms) {
    switch (bits) {
        case 2: return decode<2>(codes, out, rows, d, lut, st, num_sms);
        case 3: return decode<3>(codes, out, rows, d, lut, st, num_sms);
        case 4: return decode<4>(codes, out, rows, d, lut, st, num_sms);
        case 8: return decode<8>(codes, out, rows, d, lut, st, num_sms);
        default: return cudaErrorInvalidValue;
    }
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

}  // namespace

size_t linear_workspace_bytes(int T, int d, int N) {
    return align_up((size_t)T * d * 2, 1024) + align_up((size_t)N * d * 2, 1024);
}

size_t linear_workspace_b_offset(int T, int d) { return align_up((size_t)T * d * 2, 1024); }

cudaError_t launch_decode(int bits, const uint8_t *codes, uint16_t *out, long long rows, int d,
                          const uint16_t *lut, cudaStream_t st, int num_sms, std::string *why) {
    cudaError_t e = decode_any(bits, codes, out, rows, d, lut, st, num_sms);
    if (e != cudaSuccess)
        *why = "decode launch";
    return e;
}

cudaError_t launch_gemm(const uint16_t *A16, const uint16_t *B16, const float *s,
                        const float *rn, float *y, int T, int N, int d, cudaStream_t st,
                        int num_sms, std::string *why) {
    CUtensorMap ma, mb;
    if (!make_map(&ma, A16, T, d, BM) || !make_map(&mb, B16, N, d, BN)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const size_t smem = 1024 + (size_t)STAGES * STAGE_BYTES + 8 * (2 * STAGES + 5) + 8 +
                        kEpiWarps * BN * sizeof(float) + 64;
    cudaError_t e =
        cudaFuncSetAttribute(k2_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) {
        *why = "cudaFuncSetAttribute(k2_gemm)";
        return e;
    }
    GemmParams gp;
    gp.s = s;
    gp.rn = rn;
    gp.y = y;
    gp.M = T;
    gp.N = N;
    gp.K = d;
    gp.inv_d = 1.0f / (float)d;
    const int tiles = ((N + BN - 1) / BN) * ((T + BM - 1) / BM);
    k2_gemm<<<tiles < num_sms ? tiles : num_sms, kThreads, smem, st>>>(ma, mb, gp);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        *why = "k2_gemm launch";
    return e;
}

size_t noalloc_workspace_bytes() { return kNoAllocWorkspaceBytes; }

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
