// k2_fused.cu -- codebook GEMM with the 4-bit activation codes decoded inside the kernel.
//
// Method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and Video",
// rotation-cancellation paragraph and pseudocode (x_hat = s * codebook[xc],
// W_hat = diag(row_norms) * codebook[wc]); its speed-caveat paragraph names the fused
// non-uniform-codebook GEMM as the missing piece for real speed.
//
// y[t, o] = (s_t * rn_o / d) * sum_k Ca[xc[t,k]] * Cw[wc[o,k]]
//
// Activation codes never leave their packed form in memory: eight decoder warps read each
// 128-row x 64-code block of x_codes (32 bytes per row; two warps per row quarter, 16 bytes
// each), turn the codes into fp16 unit centroids in registers and store them straight into
// tensor memory (tcgen05.st), where the MMA reads its A operand (tcgen05.mma ... [a_tmem],
// b_desc).  Each decoded block feeds two 128 x 192 MMAs, so a tile is 128 x 384 and decoding
// costs half as much per MMA cycle.  The weight operand is fp16 unit centroids (decoded by the
// prepass) streamed by TMA through a 4-stage ring of 48 KB stages.  TMEM holds the two
// 192-column fp32 accumulators and four 32-column A stages: 512 columns.  The epilogue drains
// the accumulators and releases them before storing the last chunk.
//
// Decoding: decode8() of decode4.cuh (byte permutes on the symmetric codebook, no shared
// memory).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "decode4.cuh"
#include "oq_internal.h"
#include "sm100_common.cuh"

namespace oq {
namespace {

using namespace sm100;

__device__ unsigned int g_k2f_err;

constexpr int FBM = 128, FBN = 192, FBK = 64;
constexpr int FHALVES = 2;                          // a tile is 2 x 192 = 384 columns wide
constexpr int FTN = FHALVES * FBN;
constexpr int FB_STAGES = 4;                        // TMA ring of fp16 weight tiles
constexpr int FA_STAGES = 4;                        // TMEM ring of decoded activation tiles
constexpr int FB_HALF_BYTES = FBN * FBK * 2;        // 24 KB: one 192 x 64 box
constexpr int FB_STAGE_BYTES = FHALVES * FB_HALF_BYTES;
constexpr int FACC_COLS = FBN;                      // one fp32 accumulator (per half)
constexpr int FA_COLS = FBK / 2;                    // 64 fp16 per row = 32 columns
constexpr int FA_COL0 = FHALVES * FACC_COLS;        // 384
constexpr int FTMEM_COLS = 512;
static_assert(FA_COL0 + FA_STAGES * FA_COLS <= FTMEM_COLS, "TMEM budget");
constexpr int kFEpiWarps = 4;                       // warps 2..5
constexpr int kFDecWarps = 8;                       // warps 6..13: 2 per TMEM lane quarter
constexpr int kFThreads = 32 * (2 + kFEpiWarps + kFDecWarps);
constexpr uint32_t kFIdesc = idesc_f16(FBM, FBN);
constexpr int kFStageOut = 32 * 32 * 4;             // one 32 x 32 fp32 output chunk
constexpr size_t kFusedSmem = 1024 + (size_t)FB_STAGES * FB_STAGE_BYTES +
                              (size_t)kFEpiWarps * 2 * kFStageOut +
                              8 * (2 * FB_STAGES + 2 * FA_STAGES + 3) + 8 +
                              kFEpiWarps * 64 * sizeof(float) + 64;
static_assert(kFusedSmem <= 227 * 1024, "shared memory budget");

enum : unsigned {
    F_ERR_WAIT_B = 1u << 0,
    F_ERR_WAIT_A = 1u << 1,
    F_ERR_WAIT_SLOT = 1u << 2,
    F_ERR_WAIT_ACC = 1u << 3,
};

struct FusedParams {
    const uint8_t *xc;          // [M, K/2] 4-bit activation codes
    const float *s;             // [M]
    const float *rn;            // [N]
    int M, N, K;
    float inv_d;
    uint32_t magL0, magL1;      // low bytes of the fp16 centroids 8..11 / 12..15
    uint32_t magH0, magH1;      // high bytes of the same
};

__device__ __forceinline__ uint4 ldg_nc16(const uint8_t *p) {
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
    return v;
}

// Persistent, warp-specialised.  Warp 0 lane 0: TMA producer of weight tiles.  Warp 1: TMEM
// owner; lane 0 issues the MMAs.  Warps 2..5: epilogue (TMEM lane quarter = warp % 4).
// Warps 6..13: activation decoders (row quarter = warp % 4, one row per thread, one half of
// each 64-code block per warp).  When a tile's second 192-column half lies wholly past N,
// neither its weight box nor its MMAs are issued; its accumulator columns are never stored.
template <bool BF16>
__global__ void __launch_bounds__(kFThreads, 1)
    k2_gemm_fused(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmY,
                  const FusedParams p) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t base = (raw + 1023u) & ~1023u;
    unsigned char *basep = smem_raw + (base - raw);
    const uint32_t sB = base;
    const uint32_t sOut = sB + FB_STAGES * FB_STAGE_BYTES;      // [4 warps][2][4 KB]
    const uint32_t bars = sOut + kFEpiWarps * 2 * kFStageOut;
    auto fullB = [&](int s) { return bars + 8u * s; };
    auto emptyB = [&](int s) { return bars + 8u * (FB_STAGES + s); };
    auto fullA = [&](int s) { return bars + 8u * (2 * FB_STAGES + s); };
    auto emptyA = [&](int s) { return bars + 8u * (2 * FB_STAGES + FA_STAGES + s); };
    const uint32_t tfull = bars + 8u * (2 * FB_STAGES + 2 * FA_STAGES);
    const uint32_t tempty = tfull + 8u;
    const uint32_t drain = tfull + 16u;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(basep + (drain + 8u - base));
    float *rn_s = reinterpret_cast<float *>(basep + (drain + 16u - base));   // [4][64]
    __shared__ int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n_tiles = (p.N + FTN - 1) / FTN;
    const int num_tiles = ((p.M + FBM - 1) / FBM) * n_tiles;
    const int num_kb = p.K / FBK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < FB_STAGES; ++s) {
            mbar_init(fullB(s), 1);
            mbar_init(emptyB(s), 1);
        }
        for (int s = 0; s < FA_STAGES; ++s) {
            mbar_init(fullA(s), kFDecWarps);
            mbar_init(emptyA(s), 1);
        }
        mbar_init(tfull, 1);
        mbar_init(tempty, kFEpiWarps);
        mbar_init(drain, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        abort_flag = 0;
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                     ::"r"(smem_u32(tmem_slot)), "r"(FTMEM_COLS) : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    auto aborted = [&]() { return *(volatile int *)&abort_flag != 0; };
    auto give_up = [&](unsigned bit) {
        atomicOr(&g_k2f_err, bit);
        atomicExch(&abort_flag, 1);
    };

    if (warp == 0) {
        // ---------------- TMA producer: weight tiles ----------------
        if (lane == 0) {
            uint32_t it = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !aborted(); tile += gridDim.x) {
                const int n0 = (tile % n_tiles) * FTN;
                const int halves = (n0 + FBN < p.N) ? FHALVES : 1;   // skip an empty half
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = it % FB_STAGES;
                    if (it >= FB_STAGES &&
                        !mbar_wait(emptyB(s), ((it / FB_STAGES) & 1) ^ 1)) {
                        give_up(F_ERR_WAIT_SLOT);
                        break;
                    }
                    if (aborted())
                        break;
                    mbar_expect_tx(fullB(s), (uint32_t)(halves * FB_HALF_BYTES));
                    for (int hh = 0; hh < halves; ++hh)
                        tma_load_2d(sB + s * FB_STAGE_BYTES + hh * FB_HALF_BYTES, &tmB, kb * FBK,
                                    n0 + hh * FBN, fullB(s));
                }
            }
            if (aborted()) {
                const uint32_t from = it > (uint32_t)FB_STAGES ? it - FB_STAGES : 0;
                for (uint32_t j = from; j < it; ++j)
                    mbar_wait(fullB(j % FB_STAGES), (j / FB_STAGES) & 1);
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t it = 0;
            int i = 0;
            for (int tile = blockIdx.x; tile < num_tiles && !aborted();
                 tile += gridDim.x, ++i) {
                if (i >= 1 && !mbar_wait(tempty, (i & 1) ^ 1)) {
                    give_up(F_ERR_WAIT_SLOT);
                    break;
                }
                tc_fence_after();
                const int halves = ((tile % n_tiles) * FTN + FBN < p.N) ? FHALVES : 1;
                bool ok = true;
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int sb = it % FB_STAGES, sa = it % FA_STAGES;
                    if (!mbar_wait(fullB(sb), (it / FB_STAGES) & 1)) {
                        give_up(F_ERR_WAIT_B);
                        ok = false;
                        break;
                    }
                    if (!mbar_wait(fullA(sa), (it / FA_STAGES) & 1)) {
                        give_up(F_ERR_WAIT_A);
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_tmem = tmem + (uint32_t)(FA_COL0 + sa * FA_COLS);
                    for (int hh = 0; hh < halves; ++hh) {
                        const uint64_t db =
                            sw128_desc(sB + sb * FB_STAGE_BYTES + hh * FB_HALF_BYTES);
                        const uint32_t d_tmem = tmem + (uint32_t)(hh * FACC_COLS);
#pragma unroll
                        for (int kk = 0; kk < FBK / 16; ++kk)   // K = 16: 8 A cols, 32 B of B
                            mma_ts(d_tmem, a_tmem + 8 * kk, db + 2 * kk, kFIdesc,
                                   (kb | kk) != 0);
                    }
                    mma_commit(emptyB(sb));
                    mma_commit(emptyA(sa));
                }
                if (!ok)
                    break;
                mma_commit(tfull);
            }
            mma_commit(drain);
            if (!mbar_wait(drain, 0))
                atomicOr(&g_k2f_err, F_ERR_WAIT_ACC);
        }
    } else if (warp < 2 + kFEpiWarps) {
        // ---------------- epilogue: TMEM -> registers -> scale -> smem -> TMA store -------
        const int q = warp & 3;
        float *rn_w = rn_s + (warp - 2) * 64;
        const uint32_t out0 = sOut + (uint32_t)((warp - 2) * 2 * kFStageOut);
        unsigned char *out0p = basep + (out0 - base);
        constexpr int kCW = BF16 ? 64 : 32;                 // columns per stored chunk
        constexpr int kChunks = FTN / kCW;
        uint32_t u = 0;                                     // chunks stored so far
        int i = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++i) {
            const int m0 = (tile / n_tiles) * FBM, n0 = (tile % n_tiles) * FTN;
            const int row = m0 + q * 32 + lane;
            const float srow = (row < p.M) ? p.s[row] * p.inv_d : 0.f;
            float rnv[FTN / 32];                            // rn of column c*32 + lane
#pragma unroll
            for (int c = 0; c < FTN / 32; ++c) {
                const int col = n0 + c * 32 + lane;
                rnv[c] = (col < p.N) ? p.rn[col] : 0.f;
            }
            const bool ok = mbar_wait(tfull, i & 1);
            if (!__all_sync(0xffffffffu, ok && !aborted())) {
                if (!ok)
                    give_up(F_ERR_WAIT_ACC);
                break;
            }
            tc_fence_after();
            const uint32_t t_base = tmem + ((uint32_t)(q * 32) << 16);
            const bool rows_in = m0 + q * 32 < p.M;
#pragma unroll
            for (int c = 0; c < kChunks; ++c) {
                uint32_t r0[32], r1[32];
                tmem_ld32(t_base + (uint32_t)(c * kCW), r0);   // halves are adjacent in TMEM
                if constexpr (BF16)
                    tmem_ld32(t_base + (uint32_t)(c * kCW + 32), r1);
                if (c == kChunks - 1) {
                    // every column has been read: hand the accumulators back to the MMA
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(tempty);
                }
                if (!rows_in || n0 + c * kCW >= p.N)
                    continue;                               // box wholly outside y
                const uint32_t b = u & 1;
                if (lane == 0)
                    bulk_wait_read<1>();                    // the store that used buffer b
                __syncwarp();
                if constexpr (BF16) {
                    rn_w[lane] = rnv[2 * c];
                    rn_w[32 + lane] = rnv[2 * c + 1];
                } else {
                    rn_w[lane] = rnv[c];
                }
                __syncwarp();
                if constexpr (BF16)
                    store_chunk_bf16(&tmY, out0p + b * kFStageOut, out0 + b * kFStageOut, r0, r1,
                                     srow, rn_w, lane, n0 + c * kCW, m0 + q * 32);
                else
                    store_chunk(&tmY, out0p + b * kFStageOut, out0 + b * kFStageOut, r0, srow,
                                rn_w, lane, n0 + c * kCW, m0 + q * 32);
                ++u;
            }
        }
        if (lane == 0)
            bulk_wait_all();
    } else {
        // ---------------- activation decoders: codes -> fp16 -> TMEM ----------------
        // warp w: row quarter w % 4, code half (w - 6) / 4 of each 64-code block
        const int q = warp & 3;
        const int half = (warp - 2 - kFEpiWarps) >> 2;
        const int r = q * 32 + lane;                        // row within the tile
        const uint32_t col_base =
            tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(FA_COL0 + half * (FA_COLS / 2));
        const size_t row_bytes = (size_t)p.K / 2;
        uint32_t it = 0;
        bool stop = false;
        for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
            const int m0 = (tile / n_tiles) * FBM;
            const int row = min(m0 + r, p.M - 1);           // rows past M: any valid row
            const uint8_t *src = p.xc + (size_t)row * row_bytes + half * 16;
            uint4 c0 = ldg_nc16(src);
            for (int kb = 0; kb < num_kb; ++kb, ++it) {
                const uint4 n0 = (kb + 1 < num_kb) ? ldg_nc16(src + (kb + 1) * 32) : c0;
                const int s = it % FA_STAGES;
                if (it >= FA_STAGES) {
                    const bool ok = mbar_wait(emptyA(s), ((it / FA_STAGES) & 1) ^ 1);
                    if (!__all_sync(0xffffffffu, ok)) {
                        if (lane == 0)
                            give_up(F_ERR_WAIT_SLOT);
                        stop = true;
                        break;
                    }
                }
                if (__shfl_sync(0xffffffffu, aborted() ? 1 : 0, 0)) {
                    stop = true;
                    break;
                }
                uint32_t v[16];
                const uint32_t words[4] = {c0.x, c0.y, c0.z, c0.w};
#pragma unroll
                for (int wi = 0; wi < 4; ++wi) {
                    uint32_t o[4];
                    decode8(words[wi], p.magL0, p.magL1, p.magH0, p.magH1, o);
                    v[4 * wi + 0] = o[0];
                    v[4 * wi + 1] = o[1];
                    v[4 * wi + 2] = o[2];
                    v[4 * wi + 3] = o[3];
                }
                tmem_st16(col_base + (uint32_t)(s * FA_COLS), v);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(fullA(s));
                c0 = n0;
            }
        }
    }
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                     ::"r"(tmem), "r"(FTMEM_COLS) : "memory");
    }
}

}  // namespace

cudaError_t launch_gemm_fused_a4(const uint8_t *xc, const uint16_t *lut_a, const uint16_t *B16,
                                 const float *s, const float *rn, void *y, bool y_bf16, int T,
                                 int N, int d, cudaStream_t st, int num_sms, std::string *why) {
    auto fn = tensor_map_encoder();
    if (!fn) {
        *why = "cuTensorMapEncodeTiled unavailable";
        return cudaErrorInvalidValue;
    }
    CUtensorMap mb, my;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)N};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {(cuuint32_t)FBK, (cuuint32_t)FBN};
    cuuint32_t estr[2] = {1, 1};
    if (fn(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t *>(B16), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS ||
        !make_out_map(&my, y, T, N, y_bf16)) {
        *why = "cuTensorMapEncodeTiled failed";
        return cudaErrorInvalidValue;
    }
    const size_t smem = kFusedSmem;
    cudaError_t e = cudaSuccess;
    {
        static std::mutex mu;
        static bool done[kMaxDevices][2] = {};
        int dev = 0;
        e = cudaGetDevice(&dev);
        if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices))
            e = cudaErrorInvalidDevice;
        if (e == cudaSuccess) {
            std::lock_guard<std::mutex> lk(mu);
            if (!done[dev][y_bf16]) {
                e = cudaFuncSetAttribute(y_bf16 ? k2_gemm_fused<true> : k2_gemm_fused<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
                done[dev][y_bf16] = (e == cudaSuccess);
            }
        }
        if (e != cudaSuccess) {
            *why = "cudaFuncSetAttribute(k2_gemm_fused)";
            return e;
        }
    }
    FusedParams fp;
    fp.xc = xc;
    fp.s = s;
    fp.rn = rn;
    fp.M = T;
    fp.N = N;
    fp.K = d;
    fp.inv_d = 1.0f / (float)d;
    if (!decode8_sources(lut_a, &fp.magL0, &fp.magL1, &fp.magH0, &fp.magH1)) {
        *why = "k2_gemm_fused: activation codebook is not odd-symmetric";
        return cudaErrorInvalidValue;
    }
    const int tiles = ((N + FTN - 1) / FTN) * ((T + FBM - 1) / FBM);
    const int grid = tiles < num_sms ? tiles : num_sms;
    if (y_bf16)
        k2_gemm_fused<true><<<grid, kFThreads, smem, st>>>(mb, my, fp);
    else
        k2_gemm_fused<false><<<grid, kFThreads, smem, st>>>(mb, my, fp);
    e = cudaGetLastError();
    if (e != cudaSuccess)
        *why = "k2_gemm_fused launch";
    return e;
}

cudaError_t read_and_clear_k2f_error(unsigned *out, cudaStream_t st) {
    unsigned zero = 0;
    cudaError_t e = cudaMemcpyFromSymbolAsync(out, g_k2f_err, sizeof(unsigned), 0,
                                              cudaMemcpyDeviceToHost, st);
    if (e == cudaSuccess)
        e = cudaMemcpyToSymbolAsync(g_k2f_err, &zero, sizeof(unsigned), 0,
                                    cudaMemcpyHostToDevice, st);
    if (e == cudaSuccess)
        e = cudaStreamSynchronize(st);
    return e;
}

}  // namespace oq
