/*
 * oracle.h -- plain fp64 CPU reference for the OrbitQuant online quantized-linear path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path may include, link or call this
 * code: only the tests, the smoke check and the CPU-baseline leg of the benchmark use it.
 * It shares no code, header, table or constant generator with the CUDA library.
 *
 * Source of the method: rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and
 * Video" (summary of the preprint), cited below as [RCAP]:
 *   - change-of-basis paragraph: a normalised vector, randomly rotated, has coordinates with
 *     one fixed marginal f_d, close to N(0, 1/d) for d > 64; one Lloyd-Max quantizer is
 *     built offline against it;
 *   - rotation-cancellation paragraph: the weight rows are rotated offline, and
 *     W R^T R x = W x because R is orthogonal;
 *   - RPBH paragraph: uniform random permutation, then random sign flips and block-diagonal
 *     Walsh-Hadamard blocks, O(d log h) per token;
 *   - pseudocode block: build_rpbh(d), lloyd_max(f_d, b) once per dimension; W_rot, its row
 *     norms and nearest-centroid codes per weight matrix; x_rot, s = norm(x_rot) and
 *     nearest-centroid codes of x_rot/(s+eps) per token.
 *
 * Readings where the page is silent:
 *   RNG = SplitMix64; permutation = Fisher-Yates (Durstenfeld) with rejection-sampled
 *   bounded integers; sign[k] = top bit of the next draw, drawn after the permutation;
 *   gather semantics y[i] = x[perm[i]]; signs applied after the permutation and before the
 *   Hadamard blocks; Sylvester (natural-order) Hadamard H[i][j] = (-1)^popcount(i&j),
 *   normalised by 1/sqrt(h); f_d read as N(0, 1/d); eps = 1e-8 for activations and 0 for
 *   weights; ties at a boundary go to the upper cell; a zero row gives code 2^b/2 and
 *   norm 0; codes are packed LSB-first, row stride d*b/8 bytes, code 0 = most negative
 *   centroid; the linear output is y[t,o] = s_t * rn_o * sum_k ca[xc] * cw[wc] with
 *   sigma-scaled centroids, no bias.
 */
#ifndef OQ_ORACLE_H
#define OQ_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* SplitMix64: advances *state and returns the next 64-bit output. */
uint64_t orc_splitmix64_next(uint64_t *state);

/* Uniform integer in [0, n), n >= 1, by rejection of the top partial range. */
uint64_t orc_uniform_below(uint64_t *state, uint64_t n);

/* RPBH tables: perm[d] (a bijection on 0..d-1) and sign[d] (+1/-1). Returns 0 on success. */
int orc_build_rpbh(int d, uint64_t seed, int32_t *perm, int8_t *sign);

/* Block-RHT tables, the ablation of [RCAP]'s results list ("removing the leading uniform
 * permutation"): the RPBH tables of the same seed with perm replaced by the identity, so the
 * sign flips and blocks are those of RPBH and only P differs (a reading). */
int orc_build_block_rht(int d, uint64_t seed, int32_t *perm, int8_t *sign);

/* Sylvester Hadamard matrix entry (-1)^popcount(i & j) as an integer. */
int orc_hadamard_entry(int i, int j);

/* z = B D P x for one row: P gather, D signs, B = blockdiag(H_h / sqrt(h)).
 * The block product is done as an explicit h x h matrix-vector product. */
int orc_rotate_row(int d, int h, const int32_t *perm, const int8_t *sign,
                   const double *x, double *z);

/* Lloyd-Max quantizer for N(0,1) with L = 2^bits levels.
 * centroids[L] ascending, bounds[L-1] ascending (bounds[j-1] = t_j, the midpoint of
 * centroids j-1 and j).  Iterates the two Lloyd conditions until the largest centroid
 * move is <= tol or max_iter is reached.  *iters and *residual report what happened.
 * Returns 0 on convergence, 1 if the cap was hit. */
int orc_lloyd_max_gauss(int bits, double tol, int max_iter,
                        double *centroids, double *bounds, int *iters, double *residual);

/* Mean squared error of a quantizer (centroids, bounds) under N(0,1), in closed form. */
double orc_gauss_mse(int levels, const double *centroids, const double *bounds);

/* Regularized incomplete beta function I_x(a, b) for a, b > 0, 0 <= x <= 1, by its
 * continued fraction (evaluated where it converges fast, else through
 * I_x(a, b) = 1 - I_{1-x}(b, a)). */
double orc_betainc(double a, double b, double x);

/* The exact marginal of one coordinate of a uniformly random unit vector in R^d ([RCAP]
 * change-of-basis paragraph: "one fixed marginal that depends only on the dimension d"):
 * f_d(x) = (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on [-1, 1], d >= 3.
 * orc_sphere_cdf(d, x) = P(X <= x); orc_sphere_density(d, x) = f_d(x). */
double orc_sphere_cdf(int d, double x);
double orc_sphere_density(int d, double x);

/* Lloyd-Max quantizer with 2^bits levels for f_d (same two conditions and stopping rule as
 * orc_lloyd_max_gauss; tol is in units of the standard deviation 1/sqrt(d)).  Centroids and
 * bounds are in the coordinate's own units (inside [-1, 1]); multiplied by sqrt(d) they are
 * the unit codebook the quantizer compares against.  d >= 3. */
int orc_lloyd_max_sphere(int d, int bits, double tol, int max_iter,
                         double *centroids, double *bounds, int *iters, double *residual);

/* Nearest-centroid code of v against sigma-scaled unit boundaries:
 * code = #{ j : sigma * t_j <= v }. */
int orc_code_of(double v, int levels, const double *unit_bounds, double sigma);

/* Pack / unpack `n` codes of `bits` bits, LSB-first, into ceil(n*bits/8) bytes. */
void orc_pack(int n, int bits, const uint8_t *codes, uint8_t *out);
void orc_unpack(int n, int bits, const uint8_t *packed, uint8_t *codes);

/* Per-row quantizer (the pseudocode's online activation step, and with eps = 0 the
 * offline weight step): for each of `rows` rows of x[rows][d]:
 *   z = R x;  s = ||z||_2;  v = z / (s + eps)  (v = 0 when s + eps == 0);
 *   codes of v against sigma * unit_bounds, sigma = 1/sqrt(d); packed into
 *   packed[rows][d*bits/8].  norms[rows] receives s.
 * unit_bounds has 2^bits - 1 entries. */
int orc_quantize_rows(int rows, int d, int h, const int32_t *perm, const int8_t *sign,
                      int bits, const double *unit_bounds, double eps,
                      const double *x, uint8_t *packed, double *norms);

/* Same, but also returns the rotated rows z[rows][d] and unit values
 * u = v * sqrt(d) (so the boundaries are the unit ones) for boundary-distance checks. */
int orc_quantize_rows_detail(int rows, int d, int h, const int32_t *perm,
                             const int8_t *sign, int bits, const double *unit_bounds,
                             double eps, const double *x, uint8_t *packed, double *norms,
                             double *z, double *u);

/* Codebook linear layer, naive triple loop in fp64:
 *   y[t][o] = s[t] * rn[o] * sum_k (sigma*ca[xc[t][k]]) * (sigma*cw[wc[o][k]]),
 * sigma = 1/sqrt(d); ca, cw are unit centroids; codes are unpacked from the packed rows. */
int orc_linear(int T, int d, int out, int bits_a, const double *ca, int bits_w,
               const double *cw, const uint8_t *x_packed, const double *s,
               const uint8_t *w_packed, const double *rn, double *y);

#ifdef __cplusplus
}
#endif

#endif
