// oq_internal.h -- internal types shared by liboq's host code and its CUDA kernels.
// Not part of the public ABI (include/oq.h is).
#pragma once

#include <cstdint>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>

#include "oq.h"

namespace oq {

constexpr int kMaxDevices = 32;

// Programmatic dependent launch.  liboq launches every kernel of the hot path so that it may
// start while the previous kernel of its stream is finishing: the kernel signals at once that
// its own successor may start (pdl_trigger), does its set-up from data no earlier work writes
// (barriers, tensor memory, its host-built tables), and waits for all earlier work of the
// stream before it reads or writes anything else (pdl_wait; a no-op for a launch without a
// programmatic dependency).
#if defined(__CUDACC__)
__device__ __forceinline__ void pdl_trigger() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}
#endif

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t st, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

// Shared-memory images of K1, built on the host (oq_host.cpp) and bulk-copied per CTA.
//   Gather entries: d/32 rows of kK1EntStride words; row g holds, for positions g*32+e,
//   (byte offset of x[perm[pos]] in the staged row data) | (sign[pos] < 0) << 31.  For fp32
//   input the offset is 4*perm[pos].  For bf16 input the staged pair lives in 16-byte slots
//   of four 32-bit words (x_t0[j], x_t1[j]): element j is word j & 3 of the slot of half-chunk
//   (c = j >> 3, lh = (j >> 2) & 1), slot(g, k, lh) = (2k + lh)*GT + (g & ~7) + colour with
//   GT = d/32, c = g + k*GT, and the colours of each octet of threads a permutation of 0..7
//   chosen on the host (oq_host.cpp, pair_slot_colours); the offset is 16*slot + 4*(j & 3).
//   Words 32..35 of row g (bf16 image) hold the slots of that thread's interleave stores as
//   16-bit values, half-word 2k + lh.
//   Quantizer table: G+1 words, each repeated 32 times (one copy per lane, k*32 + lane) when
//   bits <= 4, else stored once; padded to a multiple of 4 words.
constexpr int kK1EntStride = 36;

// Parameters of the fused rotate + norm + quantize kernel (K1).
struct K1Params {
    const void *x;          // [T, d] rows, fp32 or bf16
    uint8_t *codes;         // [T, d*bits/8]
    float *norms;           // [T]
    const uint32_t *ent_img;   // gather-entry image (see above)
    const uint32_t *tbl_img;   // quantizer-table image (see above)
    int ent_words, tbl_words;  // image sizes in 32-bit words (multiples of 4)
    int T, d;
    int h;                  // Hadamard block size (read by the kernel only when h < 32)
    float eps;              // added to the norm before division (0 for weights)
    float K;                // sqrt(d/h) / (G * delta): z_unnormalised * K / (s+eps) = u/(G delta)
    int G, F;               // grid cells (power of two), F = 23 - log2(G)
    int groups;             // token pairs processed at once per CTA (set by launch_k1)
    int stages;             // raw row buffers per group, fp32 input only (set by launch_k1)
    int gelu;               // 1: quantize R GELU(x) (erf form; bf16 input only)
    uint16_t *a16;          // non-null: write fp16 unit centroids [T, d] here, not codes
    const uint32_t *dec_img;   // byte -> centroid table for a16 (bits 2, 8)
    int dec_words;             // its size in words (multiple of 4; 0 without a16)
    uint32_t dec_src[4];       // a16 with 4-bit codes: byte-permute decode sources
    // Fused weight decode (a16, groups of whole warps): once a group has no token pair left it
    // decodes weight codes into fp16 unit centroids, each CTA an equal share of the
    // wdec_groups 32-bit code words.  4-bit codes of an odd-symmetric codebook: byte-permute
    // decode, one word -> 8 centroids (16 bytes).  2-bit codes: the codebook's byte table
    // (wdec_img, bulk-copied beside the other images), one word -> 16 centroids (32 bytes).
    const uint32_t *wdec_codes;   // [wdec_groups] code words (W_codes [N, d*bits/8] as words)
    uint4 *wdec_out;              // B16 [N, d]: 1 (4-bit) or 2 (2-bit) uint4 per word
    long long wdec_groups;        // 0: no fused decode
    int wdec_bits;                // 4 or 2
    uint32_t wdec_src[4];         // 4-bit: byte-permute decode sources of the weight codebook
    const uint32_t *wdec_img;     // 2-bit: byte -> four fp16 centroids (256 x 8 bytes)
    int wdec_words;               // its size in words (0 for 4-bit)
    long long test_wait_cycles;   // > 0: the armed test wait (oq_debug_arm_wait_timeout)
    const uint32_t *gelu_img;     // gelu: the GELU table of the bf16 values (k1_ops.cuh)
    int gelu_words;               // its size in words (0 without gelu)
};
// GELU(x) for every bf16 x with 2^-16 <= |x| < 16 (layout in k1_ops.cuh, gelu_lookup), in fp64
// rounded to fp32: the host image K1 copies into shared memory for its fused GELU.
std::vector<uint32_t> gelu_table_image();
// True when K1 can write fp16 centroids itself (launch_k1 with p.a16 set).
inline bool k1_a16_supported(int bits, int h, bool bf16_in) {
    return bf16_in && h >= 32 && h <= 256 && (bits == 2 || bits == 4 || bits == 8);
}
// Threads of a named-barrier K1 group: the d/32 position-owning threads of a token pair,
// padded to whole warps.
inline int k1_group_threads(int d) { return (d / 32 + 31) & ~31; }
// True when K1 runs as one CTA per SM with named-barrier groups: bf16 rows, and the padding
// to whole warps leaves at most one lane in eight idle (d/32 a multiple of 32, or large
// enough: d = 9728 and 13824 qualify, 2560 does not); the fused weight decode needs it.
inline bool k1_named(int d, bool bf16_in) {
    const int gt = d / 32, gtp = k1_group_threads(d);
    return bf16_in && 8 * (gtp - gt) <= gtp;
}
// (4-bit additionally needs an odd-symmetric codebook, which every Lloyd-Max codebook here is;
// the host checks it when it builds dec_src.)

// Tensor-core K1 (k1_tc.cu): bf16 rows; the block transform as tcgen05.mma.
struct K1TcParams {
    const uint8_t *x;          // [T, d] bf16 rows
    uint8_t *codes;            // [T, d*bits/8]
    float *norms;              // [T]
    const uint16_t *ent;       // [d] perm[i] | (sign[i] < 0) << 15
    const uint32_t *tbl_img;   // quantizer-table image (as K1)
    int tbl_words;
    int T, d, h;
    float eps, K;              // as K1
    int G, F;
};
bool k1_tc_supported(int d, int h, int bits, int tbl_words);
size_t k1_tc_smem(int d, int tbl_words);
cudaError_t launch_k1_tc(const K1TcParams &p, int bits, cudaStream_t st, int num_sms,
                         std::string *why);
cudaError_t read_and_clear_k1tc_error(unsigned *out, cudaStream_t st);

// Launch K1 for (bits, h, dtype); `num_sms` sizes the grid.
cudaError_t launch_k1(const K1Params &p, int bits, int h, int in_f32, cudaStream_t st,
                      int num_sms, std::string *why);

// Codebook linear layer: decode prepass (codes -> fp16 unit centroids) + tcgen05 GEMM.
// Workspace layout: A16 [T, d] fp16 at offset 0, B16 [N, d] fp16 at linear_workspace_b_offset.
size_t linear_workspace_bytes(int T, int d, int N);
size_t linear_workspace_b_offset(int T, int d);

cudaError_t launch_decode(int bits, const uint8_t *codes, uint16_t *out, long long rows, int d,
                          const uint16_t *lut, cudaStream_t st, int num_sms, std::string *why);
// Both operands' codes in one decode launch when both are 4-bit codes of odd-symmetric
// codebooks (byte-permute decode); false (nothing launched) otherwise.  *err: the launch.
bool launch_decode_pair(int bits_a, const uint8_t *codes_a, uint16_t *out_a, long long rows_a,
                        const uint16_t *lut_a, int bits_b, const uint8_t *codes_b,
                        uint16_t *out_b, long long rows_b, const uint16_t *lut_b, int d,
                        cudaStream_t st, int num_sms, cudaError_t *err, std::string *why);

// y[T, N] = (s_t rn_o / d) * A[T, d] . B[N, d]^T   (fp16 x fp16 -> fp32 in TMEM)
// A is A16 (fp16 centroids from the prepass) or, when A16 is null, x_codes4: 4-bit codes of
// the codebook whose fp16 LUT is lut_a (must be odd-symmetric), decoded inside the kernel.
// B likewise: B16, or (B16 null; CTA-pair kernel only) w_codes4 with lut_w.  At most one
// operand as codes.  y is fp32, or bf16 (round to nearest even of the fp32 epilogue value)
// when y_bf16.  test_wait_cycles > 0 arms the kernel's test of its bounded waits
// (oq_debug_arm_wait_timeout).  With few output tiles (fp16 operands, CTA-pair kernel) the
// K loop is split over more CTA pairs and a reduce kernel sums their fp32 partials, in
// split_ws (split_ws_bytes; an error if too small) or, when it is null, a stream-ordered
// temporary buffer.
cudaError_t launch_gemm(const uint16_t *A16, const uint8_t *x_codes4, const uint16_t *lut_a,
                        const uint16_t *B16, const uint8_t *w_codes4, const uint16_t *lut_w,
                        const float *s, const float *rn, void *y, bool y_bf16, int T, int N,
                        int d, cudaStream_t st, int num_sms, std::string *why,
                        long long test_wait_cycles = 0, void *split_ws = nullptr,
                        size_t split_ws_bytes = 0);

// The online step in one persistent kernel (k3_fused.cu): the quantize stage and the CTA-pair
// GEMM side by side on every SM, rows handed over through per-block counters.
struct FusedStepParams {
    // quantize stage (as K1 with fp16 output)
    const unsigned char *x;             // bf16 [T, d]
    uint16_t *a16;                      // fp16 [T, d]: the GEMM's A operand
    float *s;                           // [T]
    const uint32_t *ent_img, *tbl_img, *dec_img;   // K1's bf16 entry image and tables
    int ent_words, tbl_words, dec_words;
    uint32_t dec_src[4];
    float eps, K;
    int G, F;
    // GEMM
    const float *rn;
    int T, N, d;
    float inv_d;
    // weight decode inside the kernel (2- or 4-bit weight codes; wdec_words = 0: B16 was
    // decoded before the launch): W_codes as 32-bit words -> fp16 B16 [N, d]
    const uint32_t *wcodes;
    uint4 *b16;
    long long wdec_words;
    int wdec_bits;
    uint32_t wdec_src[4];               // 4-bit: byte-permute sources of the weight codebook
    const uint2 *wdec_tab;              // 2-bit: byte -> four fp16 centroids
    // progress counters, zeroed before the launch: [0] next token pair, [1] next tile,
    // [2] unused, [3] weight-decoding warps done, [4 + b] rows of 256-row block b of x done
    // (fused_step_counter_words(T, N) words)
    unsigned *ctr;
    long long test_wait_cycles;
    int ramp_rounds;                    // token pairs a ramp group quantizes (0: no ramp groups)
};
bool fused_step_supported(int d, int h, int bits, bool bf16_in);
size_t fused_step_counter_words(int T, int N);
// Zero n counter words on the stream (a programmatic-launch kernel, see k3_fused.cu).
cudaError_t launch_zero_counters(unsigned *ctr, int n, cudaStream_t st);
cudaError_t launch_fused_step(const FusedStepParams &p, int bits, int h, bool y_bf16,
                              const uint16_t *B16, void *y, cudaStream_t st, std::string *why);
cudaError_t read_and_clear_k3_error(unsigned *out, cudaStream_t st);
// fp16 [rows, K] row-major operand -> TMA map of 128-row x 64 boxes, 128-byte swizzle
bool make_operand_map(CUtensorMap *map, const void *ptr, long long rows, int K);

// False when OQ_GEMM_PAIR=0 asks for the single-CTA GEMM (read once per process).
bool gemm_pair_enabled();
// True when launch_gemm splits the K loop of a [T, d] x [N, d] product (few output tiles).
bool gemm_splits_k(int T, int N, int d, bool y_bf16);

// Fixed device workspace of oq_linear_noalloc (a static __device__ array in k2_linear.cu):
// its size, and its address on the current device (looked up once per device).
size_t noalloc_workspace_bytes();
// its region past the operands for split-K partials (noalloc_workspace + the size above)
size_t noalloc_split_bytes();
cudaError_t noalloc_workspace(void **out);

// Device error words written by the kernels (bounded waits that gave up etc.):
// read-and-clear on the current device.
cudaError_t read_and_clear_k1_error(unsigned *out, cudaStream_t st);
cudaError_t read_and_clear_k2_error(unsigned *out, cudaStream_t st);

}  // namespace oq
