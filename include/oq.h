/*
 * oq.h -- C ABI of liboq, the B200 (sm_100a) OrbitQuant online quantized-linear path.
 *
 * The method is the one summarised on rcap.io, "OrbitQuant: Data-Agnostic Quantization for
 * Image and Video" [RCAP]: rotate every activation row x (dimension d) with a Randomized
 * Permuted Block-Hadamard (RPBH) rotation R, take its norm s, encode each rotated coordinate
 * as a b-bit nearest-centroid code of one Lloyd-Max codebook built offline for the fixed
 * N(0, 1/d) marginal, and multiply against weights stored the same way (row norms times codes
 * of W R^T).  Since R is orthogonal, W R^T R x = W x and the rotation cancels inside the
 * layer.
 *
 * Conventions shared by every call
 *   - Return value: OQ_OK (0) or a negative OQ_E* status.  On failure nothing was launched,
 *     and oq_last_error() returns a thread-local message.
 *   - Data buffers are owned by the caller.  Pointers named "device" must be CUDA device
 *     pointers on the current device, 16-byte aligned.  Host pointers are plain memory.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).  Launches
 *     are asynchronous on it; a fault inside a kernel is reported by oq_check() or by the
 *     next synchronising CUDA call.
 *   - Handles (oq_rpbh, oq_codebook) are immutable once built, may be shared by several
 *     streams and threads, and are freed with oq_free_*.  Their first use on a device copies
 *     small tables to that device synchronously; make that first use outside any CUDA graph
 *     capture.
 *   - The library keeps per-device state (uploaded tables, its memory pool, side stream and
 *     events, the device address of its fixed workspace).  cudaDeviceReset() on a device the
 *     library has used invalidates that state: do not call the library on that device (or
 *     free handles used there) after resetting it.
 *   - Sizes: d is a multiple of 128 and of h, 128 <= d <= 16384; h is a power of two,
 *     2 <= h <= 1024; bits in {2, 3, 4, 6, 8}; 0 <= T < 2^31 rows (T = 0 is a no-op returning
 *     OQ_OK); the linear layer also needs 1 <= out_features < 2^31 with rows of y a
 *     multiple of 16 bytes (out_features a multiple of 4 for fp32 y, of 8 for bf16 y).
 *     Why these limits: a row of 3-bit codes is d*3/8 bytes, a multiple of 16 (the alignment
 *     of the 128-bit stores and TMA copies of code rows) only when d is a multiple of 128;
 *     the quantizer stages a token pair in shared memory (8*d bytes for bf16 rows, 128 KB at
 *     d = 16384); y is written by TMA tensor stores, whose row stride must be a multiple of
 *     16 bytes.
 *   - Packed codes: row-major, one row per token (or weight row), row stride d*bits/8 bytes,
 *     element k of a row in bits [k*bits, k*bits + bits) of the row's byte stream, bit i of
 *     the stream being bit (i mod 8) of byte i/8 (LSB first).  Code 0 is the most negative
 *     centroid.
 */
#ifndef OQ_H
#define OQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define OQ_OK 0
#define OQ_EINVAL (-1)        /* bad argument: size, alignment, null pointer, bit width   */
#define OQ_EUNSUPPORTED (-2)  /* current device is not sm_100 (B200-class)                 */
#define OQ_ECUDA (-3)         /* a CUDA runtime/driver call failed                         */
#define OQ_EDEVICE (-4)       /* a kernel reported an internal error (see oq_check)        */
#define OQ_ENOMEM (-5)        /* host allocation failed                                    */

#define OQ_F32 0              /* element types for `dtype` / `out_dtype`                  */
#define OQ_BF16 1

typedef struct oq_rpbh oq_rpbh;
typedef struct oq_codebook oq_codebook;

/* Build the RPBH rotation of dimension d with Hadamard blocks of size h from `seed`.
 * [RCAP] RPBH paragraph (uniform random permutation, random sign flips, block-diagonal
 * Walsh-Hadamard blocks) and pseudocode build_rpbh(d).  Definition used here: SplitMix64
 * seeded with `seed` draws a Fisher-Yates (Durstenfeld) permutation perm[d] (j = r mod (i+1)
 * for i = d-1..1, rejecting r >= 2^64 - (2^64 mod (i+1))), then sign[k] for k = 0..d-1 from
 * the top bit of each next draw (set = -1).  R x = blockdiag(H_h/sqrt(h)) diag(sign) y with
 * y[i] = x[perm[i]] and Sylvester H_h[i][j] = (-1)^popcount(i & j).
 * Host-only; no GPU needed.  *out receives a new handle (free with oq_free_rpbh).
 * Errors: OQ_EINVAL for d, h outside the limits above or out == NULL. */
int oq_build_rpbh(int d, int h, uint64_t seed, oq_rpbh **out);

/* Block-RHT: the ablation in [RCAP]'s results list that removes the leading uniform
 * permutation.  The handle is that of oq_build_rpbh(d, h, seed) with the permutation replaced
 * by the identity (same sign flips, same blocks), so it runs through the same calls
 * (oq_quantize_act / oq_quantize_weight) and only P differs.  Same arguments and errors. */
int oq_build_block_rht(int d, int h, uint64_t seed, oq_rpbh **out);

/* Copy the handle's tables to host memory: perm_out[d] (int32), sign_out[d] (+1/-1).
 * Either pointer may be NULL.  Host-only. */
int oq_rpbh_tables(const oq_rpbh *r, int32_t *perm_out, int8_t *sign_out);

/* Build the Lloyd-Max codebook with 2^bits levels for the N(0, 1/d) marginal.
 * [RCAP] change-of-basis paragraph ("the standard Lloyd-Max quantizer construction" against
 * the fixed marginal, close to N(0, 1/d) for d > 64) and pseudocode lloyd_max(f_d, b).
 * The unit (N(0,1)) quantizer is solved in fp64 and scaled by sigma = 1/sqrt(d).
 * Host-only; no GPU needed.  Errors: OQ_EINVAL for bits not in {2,3,4,6,8}, d < 1. */
int oq_lloyd_max(int d, int bits, oq_codebook **out);

#define OQ_MARGINAL_GAUSSIAN 0   /* N(0, 1/d), the reading oq_lloyd_max uses                */
#define OQ_MARGINAL_EXACT 1      /* f_d, the exact law of one coordinate of a unit vector   */

/* oq_lloyd_max against a chosen marginal.  OQ_MARGINAL_EXACT: f_d(x) = (1 - x^2)^((d-3)/2) /
 * B(1/2, (d-1)/2) on [-1, 1], the law of one coordinate of a uniformly random unit vector in
 * R^d ([RCAP] change-of-basis paragraph: the fixed marginal that depends only on d, which
 * N(0, 1/d) approximates above d = 64).  The codebook is stored as sqrt(d) times the f_d
 * quantizer, so it plugs into the same kernels as the Gaussian one (oq_codebook_values
 * returns the f_d quantizer itself).  Host-only.  Errors: OQ_EINVAL for an unknown
 * marginal, bits not in {2,3,4,6,8}, d < 1 (d < 3 for the exact marginal). */
int oq_lloyd_max_marginal(int d, int bits, int marginal, oq_codebook **out);

/* Copy the codebook to host memory in fp64, sigma-scaled: centroids[2^bits] ascending,
 * bounds[2^bits - 1] ascending (bounds[j] is the midpoint of centroids j and j+1).
 * Either pointer may be NULL.  Host-only. */
int oq_codebook_values(const oq_codebook *cb, double *centroids, double *bounds);

/* Introspection of the fast quantizer table the activation/weight kernel uses (for tests):
 * grid_cells (G, a power of two), cell width in unit-codebook units (delta), and the G+1
 * table words (table may be NULL to query G first).  A unit value u maps to
 * a = sat(u/(G*delta) + 1/2); with q = floor(a * 2^23), word = table[q >> (23 - log2 G)],
 * code = (word + q*G + 0x3F800000*G) >> 24 in 32-bit unsigned arithmetic.  Host-only. */
int oq_codebook_grid(const oq_codebook *cb, int *grid_cells, double *delta, uint32_t *table);

/* Offline weight step: [RCAP] pseudocode "W_rot = W @ rotation.T; row_norms = norm(W_rot);
 * W_hat = diag(row_norms) nearest_centroid(W_rot / row_norms, codebook[d, bw])".
 * W: device, [out_features, d] row-major of `dtype` (OQ_F32 or OQ_BF16).
 * W_codes: device, [out_features, d*bw/8] packed codes (bw = cw's bits).
 * row_norms: device, fp32 [out_features] = ||R w_o|| (fp32 accumulation).
 * No eps; an all-zero row gives codes 2^bw/2 and norm 0.
 * Errors: OQ_EINVAL (d mismatch with r/cw, sizes, null or misaligned pointers),
 * OQ_EUNSUPPORTED, OQ_ECUDA. */
int oq_quantize_weight(const oq_rpbh *r, const oq_codebook *cw, const void *W, int dtype,
                       int out_features, int d, uint8_t *W_codes, float *row_norms,
                       void *stream);

/* Online activation step: [RCAP] pseudocode "x_rot = x @ rotation.T; s = norm(x_rot);
 * x_hat = s * nearest_centroid(x_rot / (s + eps), codebook[d, ba])", eps = 1e-8.
 * x: device, [T, d] row-major of `dtype`.  x_codes: device, [T, d*ba/8] packed codes.
 * s: device, fp32 [T], the per-token norm ("the only input-dependent number at runtime").
 * A code is the number of sigma-scaled boundaries <= x_rot/(s+eps) (ties go up), decided in
 * fp32.  An all-zero row gives codes 2^ba/2 and s = 0.  The rotation runs as register
 * butterflies on the CUDA cores; with the environment variable OQ_K1_PATH=tc (read once per
 * process) bf16 rows with 32 <= h <= 256 and d up to about 3.9K use a kernel that runs the block
 * transform as tcgen05 MMAs instead (same results under the same parity rules).
 * Errors: as oq_quantize_weight. */
int oq_quantize_act(const oq_rpbh *r, const oq_codebook *ca, const void *x, int dtype, int T,
                    int d, uint8_t *x_codes, float *s, void *stream);

/* oq_quantize_act applied to GELU(x) = x Phi(x) = x (1 + erf(x/sqrt 2)) / 2, computed inside
 * the kernel: the quantized input of an MLP's down projection straight from the up
 * projection's pre-activation, with no GELU pass over memory.  GELU of each bf16 element is
 * its fp64 value rounded to fp32 (a table over 2^-16 <= |x| < 16; x/2 below, x or 0 beyond
 * +-16); s = ||R GELU(x)||.  x must be OQ_BF16.  Same layouts and
 * errors as oq_quantize_act, plus OQ_EINVAL for fp32 input.  The pages' models (FLUX, Wan)
 * feed their MLP down projections through GELU; this is the fused form of that step. */
int oq_quantize_act_gelu(const oq_rpbh *r, const oq_codebook *ca, const void *x, int dtype,
                         int T, int d, uint8_t *x_codes, float *s, void *stream);

/* Codebook linear layer: y[t][o] = s[t] * row_norms[o] * sum_k ca[x_codes[t][k]] *
 * cw[W_codes[o][k]] with sigma-scaled centroids, i.e. x_hat . w_hat in the rotated basis,
 * which equals the quantized W x because W R^T R x = W x ([RCAP] rotation-cancellation
 * paragraph; the fused low-bit GEMM is the speed caveat paragraph's missing piece).
 * x_codes: device [T, d*ba/8]; s: device fp32 [T]; W_codes: device [out_features, d*bw/8];
 * row_norms: device fp32 [out_features]; y: device [T, out_features] of out_dtype: OQ_F32,
 * or OQ_BF16 (the fp32 epilogue value s*rn/d*acc rounded to nearest even; adds up to 2^-9
 * relative error per element on top of the fp32 result).
 * Centroids enter the tensor cores as fp16 unit-variance values; accumulation is fp32.
 * Both code operands are decoded into fp16 buffers first.  With 4-bit activation codes and
 * the environment variable OQ_LINEAR_PATH=fused (read once per process), the activation codes
 * are instead brought into the GEMM kernel by TMA as packed codes and decoded there, through
 * the codebook's fp16 LUT held in registers, into its shared-memory operand tiles; only the
 * weight codes get an fp16 buffer (less device memory and traffic, more decode work per call;
 * the same y bit for bit, since both forms feed the MMA the same fp16 values).  With 4-bit
 * weight codes and OQ_LINEAR_PATH=wcodes, the weight codes are the ones decoded inside the
 * (CTA-pair) GEMM, each weight row once per 256-row tile of y, and only the activation codes
 * get an fp16 buffer (again the same y; with OQ_GEMM_PAIR=0 the variable has no effect).
 * Without OQ_LINEAR_PATH, 4-bit weight codes of an odd-symmetric codebook take that form
 * when T <= 256 (one row of tiles: each weight row is decoded once either way).  When the
 * product has few 256 x 256 output tiles (small T), the GEMM splits its K loop over more CTA
 * pairs and a second kernel sums their fp32 partials in a fixed order (a stream-ordered
 * temporary buffer of at most ~19 MB): y then differs from the unsplit product by fp32
 * summation order only, and every form of the call splits the same way.
 * Either way the temporary device memory is stream-ordered, from a library-owned
 * pool.  The fp16 operands meet in a tcgen05 GEMM on pairs of CTAs (256 x 256 output tiles);
 * the environment variable OQ_GEMM_PAIR=0 (read once per process) selects the single-CTA
 * GEMM (128 x 256 tiles) instead; both give the same y.
 * Errors: as above, plus OQ_ECUDA if the pool allocation fails. */
int oq_linear(const oq_codebook *ca, const oq_codebook *cw, const uint8_t *x_codes,
              const float *s, const uint8_t *W_codes, const float *row_norms, int T, int d,
              int out_features, void *y, int out_dtype, void *stream);

#define OQ_FORWARD_GELU 1u   /* oq_quantized_linear flag: the input is a GELU pre-activation */

/* The whole online path in one call: y = W_hat x_hat with x_hat the activation step of x
 * ([RCAP] pseudocode, online part, and rotation-cancellation paragraph), i.e. the result of
 * oq_quantize_act followed by oq_linear, without materialising x_codes: the rotate+quantize
 * kernel writes each code's fp16 unit centroid straight into the GEMM's A operand (bf16 x,
 * ba in {2, 4, 8}, 32 <= h <= 256; otherwise codes and the decode prepass are used inside the
 * call).  With OQ_LINEAR_PATH=fused (read once per process), bf16 x and 4-bit activation
 * codes, the rotate+quantize kernel writes the packed codes instead and the GEMM decodes them
 * in shared memory (as oq_linear does under that variable); with OQ_LINEAR_PATH=wcodes, or
 * by default when T <= 256, 4-bit weight codes of an odd-symmetric codebook are decoded by the
 * GEMM itself (no weight decode launch and no [out_features, d] fp16 buffer); with few output
 * tiles the GEMM splits its K loop as oq_linear does.  Otherwise, with 2- or 4-bit weight codes, d up to 5120
 * whose d/32 threads a token pair fill whole warps (or nearly: d a multiple of 1024, or
 * 896, 3968, ...), bf16 x and out_features <= T, the rotate+quantize kernel
 * also decodes the weight codes into the GEMM's B operand once it runs out of tokens;
 * otherwise the weight codes are decoded on a library-owned side stream of the device while x
 * is quantized.  With OQ_FUSED_STEP=1 (read once per process), bf16 x without GELU, 2/4/8-bit
 * activation codes, h in {64, 128, 256} and d in {1024, 2048, 3072, 4096}, one persistent
 * kernel decodes 2- or 4-bit weight codes (others: a decode launch before it), then runs the
 * rotate+quantize stage and the GEMM side by side on every SM, the GEMM taking each 256-row
 * block as soon as its rows are quantized (opt-in: measured within 2 % of the default form
 * on a 4608 x 3072 x 3072 W4A4 projection).  OQ_FUSED_RAMP=n (0..8, read once per process;
 * default 0) lets the GEMM's own warps quantize n token pairs a group before their GEMM roles.  y and s are bit-identical to oq_quantize_act + oq_linear in every form.
 * x: device [T, d] of dtype; W_codes [out_features, d*bw/8]; row_norms fp32 [out_features];
 * y: device [T, out_features] of out_dtype (OQ_F32 or OQ_BF16); s: optional device fp32 [T]
 * receiving the norms (NULL: kept internal).  flags: OQ_FORWARD_GELU quantizes GELU(x)
 * (as oq_quantize_act_gelu; bf16 x).  Temporary device memory comes from the library's
 * stream-ordered pool.  The side stream and its fork/join events are per device and shared
 * by all callers (enqueues are serialised); while a graph capture is open on one host
 * thread, no other thread may call this function on the same device.
 * Errors: as oq_quantize_act and oq_linear. */
int oq_quantized_linear(const oq_rpbh *r, const oq_codebook *ca, const oq_codebook *cw,
                        const void *x, int dtype, const uint8_t *W_codes, const float *row_norms,
                        int T, int d, int out_features, void *y, int out_dtype, float *s,
                        int flags, void *stream);

/* oq_linear for callers that cannot allocate device memory.  The paper has no counterpart;
 * this is a deployment variant of the same computation, with the same arguments and errors as
 * oq_linear.  It always runs the decode prepass into fp16 operands followed by the GEMM,
 * bit-identical to oq_linear's default forms (which feed the GEMM the same fp16 values, and
 * split its K loop the same way at small T); it ignores OQ_LINEAR_PATH, so in a process
 * that set OQ_LINEAR_PATH=fused the two calls may differ in the last bits (both are within the
 * linear layer's parity bound).  oq_timing_* records its kernels like oq_linear's.
 * Who needs it: code that runs inside a host framework which owns all device memory and gives
 * plug-ins no allocator (a side cudaMalloc would bypass its accounting or fail under its
 * memory cap), and latency-critical serving loops that forbid allocation on the request path
 * because cudaMalloc/cudaFree can synchronise the device and stall other streams.
 * How: the two fp16 operand buffers live in a fixed array compiled into the library
 * (OQ_NOALLOC_WORKSPACE_BYTES = 64 MiB, plus 20 MiB for the split-K partials of small-T
 * calls), which every GPU that loads the library holds until the process exits.  The call
 * allocates and frees nothing.
 * Limit: 2*(T*d + out_features*d) bytes, each part rounded up to 1 KiB, must fit in
 * OQ_NOALLOC_WORKSPACE_BYTES (e.g. T = 4608, d = out_features = 3072 needs 47 MB); larger
 * calls return OQ_EINVAL with the sizes in oq_last_error(), before touching the device.
 * Set-up: the first call on each device looks up the array's device address once (it may
 * load the library's kernels on that device); make that first call before any stream capture.
 * Sharing: every call uses the same array and it keeps the last call's contents; nothing in it
 * needs to start at zero because each call overwrites the parts it reads.  Calls that can run
 * at the same time on the GPU (different streams, or threads without ordering between them)
 * race on the array: order them on one stream or with events. */
#define OQ_NOALLOC_WORKSPACE_BYTES (64u << 20)
int oq_linear_noalloc(const oq_codebook *ca, const oq_codebook *cw, const uint8_t *x_codes,
                      const float *s, const uint8_t *W_codes, const float *row_norms, int T,
                      int d, int out_features, void *y, int out_dtype, void *stream);

/* Test of failure detection (the pages have no counterpart; this checks the library's own
 * error path).  Every wait inside liboq's kernels is bounded: a wait that runs out records a
 * bit in a device error word and the kernel returns instead of hanging.  This call arms, for
 * the calling thread, a one-shot test of that path: the next launch of `kernel` made by this
 * thread (OQ_KERNEL_QUANTIZE: the CUDA-core rotate+quantize kernel; OQ_KERNEL_GEMM: either
 * GEMM form) does all of its normal work, then one of its threads waits on a shared-memory
 * barrier that nothing completes, gives up after `limit_cycles` SM clock cycles and records
 * the timeout (quantize bit 2, linear bit 8) before returning normally.  oq_check() then
 * returns OQ_EDEVICE and names the bit; the outputs are those of an unarmed call and the
 * context stays usable.  No fault, trap or unbounded wait is involved.
 * kernel = 0 disarms.  Errors: OQ_EINVAL for another kernel id or limit_cycles outside
 * [1e3, 1e9]. */
int oq_debug_arm_wait_timeout(int kernel, long long limit_cycles);

/* Synchronise `stream`, then read and clear the library's device error word.
 * Returns OQ_OK, OQ_EDEVICE (a kernel gave up a bounded wait or saw an internal
 * inconsistency; oq_last_error() says which), or OQ_ECUDA. */
int oq_check(void *stream);

void oq_free_rpbh(oq_rpbh *r);
void oq_free_codebook(oq_codebook *cb);

/* Per-kernel timing, for profilers and benchmarks (the pages have no counterpart; it only
 * observes the path).  While enabled on the calling thread, every kernel that oq_quantize_*
 * and oq_linear launch is bracketed by two CUDA events recorded on the caller's stream.
 * oq_timing_collect() waits for those events, writes up to `capacity` records in launch
 * order (kernel id, milliseconds) and forgets all pending records; *count receives the number
 * written.  Records belong to the device that was current at launch. */
#define OQ_KERNEL_QUANTIZE 1   /* fused rotate + norm + quantize */
#define OQ_KERNEL_DECODE 2     /* codes -> fp16 centroid prepass of oq_linear */
#define OQ_KERNEL_GEMM 3       /* tcgen05 codebook GEMM of oq_linear */
#define OQ_KERNEL_FUSED 4      /* quantize stage and GEMM in one kernel (OQ_FUSED_STEP=1) */
#define OQ_KERNEL_AUX 5        /* auxiliary launch: the fused step's counter reset */
typedef struct {
    int kernel;
    float ms;
} oq_timing_record;
int oq_timing_enable(int on);
int oq_timing_collect(oq_timing_record *out, int capacity, int *count);

/* Thread-local text of the last non-OK status returned on this thread. */
const char *oq_last_error(void);

/* Library version string. */
const char *oq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* OQ_H */
