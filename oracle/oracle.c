/*
 * oracle.c -- plain fp64 CPU reference for the OrbitQuant online quantized-linear path.
 *
 * TEST INFRASTRUCTURE ONLY (see oracle.h): slow, single-threaded and written to be checked
 * by eye against the rcap.io summary "OrbitQuant: Data-Agnostic Quantization for Image and
 * Video" [RCAP].  No blocking, no fused loops, no fast transform: every step is the
 * textbook definition the summary names.
 *
 * Parity pins (tests/test_oracle_*.py): SplitMix64 published outputs, Fisher-Yates
 * uniformity, H H^T = h I, R R^T = I against an explicit dense matrix, W R^T R x = W x,
 * the classical Gaussian Lloyd-Max optima (Max 1960) and closed forms at 1 bit, fixed-point
 * conditions checked by numerical quadrature, exhaustive nearest-centroid argmin, hand
 * packed bytes, and the linear layer against a dense matrix product of decoded codes.
 */
#include "oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------------------------------
 * Random tables.  [RCAP] RPBH paragraph: "a uniform random permutation followed by ...
 * random sign flips".  The generator and draw order are a reading (oracle.h).
 * ------------------------------------------------------------------------------------- */

/* SplitMix64 as published by Steele, Lea and Flood (2014), public-domain constants. */
uint64_t orc_splitmix64_next(uint64_t *state)
{
    uint64_t z;
    *state += 0x9E3779B97F4A7C15ULL;
    z = *state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Uniform integer in [0, n): draw r, reject r >= 2^64 - (2^64 mod n), return r mod n. */
uint64_t orc_uniform_below(uint64_t *state, uint64_t n)
{
    uint64_t rem = (0 - n) % n;          /* 2^64 mod n */
    uint64_t limit = 0 - rem;            /* 2^64 - rem, as a wrapped uint64 (0 means 2^64) */
    for (;;) {
        uint64_t r = orc_splitmix64_next(state);
        if (rem == 0 || r < limit)
            return r % n;
    }
}

int orc_build_rpbh(int d, uint64_t seed, int32_t *perm, int8_t *sign)
{
    uint64_t state = seed;
    int i, k;
    if (d < 1 || !perm || !sign)
        return -1;
    for (i = 0; i < d; ++i)
        perm[i] = i;
    /* Fisher-Yates (Durstenfeld): for i = d-1 down to 1, swap i with uniform j in [0, i]. */
    for (i = d - 1; i >= 1; --i) {
        int j = (int)orc_uniform_below(&state, (uint64_t)i + 1);
        int32_t t = perm[i];
        perm[i] = perm[j];
        perm[j] = t;
    }
    /* One sign per position, drawn after the permutation: top bit set means -1. */
    for (k = 0; k < d; ++k)
        sign[k] = (orc_splitmix64_next(&state) >> 63) ? -1 : 1;
    return 0;
}

int orc_build_block_rht(int d, uint64_t seed, int32_t *perm, int8_t *sign)
{
    int i, rc = orc_build_rpbh(d, seed, perm, sign);
    if (rc != 0)
        return rc;
    for (i = 0; i < d; ++i)
        perm[i] = i;
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * Rotation.  [RCAP] RPBH paragraph and pseudocode "x_rot = x @ rotation[d].T".
 * R = B D P with P the gather y[i] = x[perm[i]], D = diag(sign), B = blockdiag(H_h/sqrt h).
 * ------------------------------------------------------------------------------------- */

int orc_hadamard_entry(int i, int j)
{
    unsigned v = (unsigned)(i & j);
    int parity = 0;
    while (v) {
        parity ^= (int)(v & 1u);
        v >>= 1;
    }
    return parity ? -1 : 1;
}

static int is_pow2(int h)
{
    return h > 0 && (h & (h - 1)) == 0;
}

int orc_rotate_row(int d, int h, const int32_t *perm, const int8_t *sign,
                   const double *x, double *z)
{
    double *y;
    double inv_sqrt_h;
    int i, j, b;
    if (d < 1 || !is_pow2(h) || d % h != 0)
        return -1;
    y = (double *)malloc(sizeof(double) * (size_t)d);
    if (!y)
        return -2;
    /* P then D */
    for (i = 0; i < d; ++i)
        y[i] = (double)sign[i] * x[perm[i]];
    /* B: each h-block multiplied by the explicit Sylvester matrix, then 1/sqrt(h) */
    inv_sqrt_h = 1.0 / sqrt((double)h);
    for (b = 0; b < d / h; ++b) {
        const double *yb = y + (size_t)b * h;
        double *zb = z + (size_t)b * h;
        for (i = 0; i < h; ++i) {
            double acc = 0.0;
            for (j = 0; j < h; ++j)
                acc += (double)orc_hadamard_entry(i, j) * yb[j];
            zb[i] = acc * inv_sqrt_h;
        }
    }
    free(y);
    return 0;
}

/* ---------------------------------------------------------------------------------------
 * Lloyd-Max codebook.  [RCAP] change-of-basis paragraph: "the standard Lloyd-Max quantizer
 * construction" against the fixed marginal, read as N(0, 1/d).  Built for N(0,1) (unit
 * codebook) and scaled by sigma = 1/sqrt(d) where it is used.
 * ------------------------------------------------------------------------------------- */

static double phi(double x)          /* standard normal density; 0 at +-infinity */
{
    if (isinf(x))
        return 0.0;
    return exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
}

static double upper_tail(double x)   /* Q(x) = P(X >= x) */
{
    if (isinf(x))
        return x > 0 ? 0.0 : 1.0;
    return 0.5 * erfc(x / sqrt(2.0));
}

/* P(a <= X < b) for a < b, through the tail that avoids cancellation. */
static double cell_prob(double a, double b)
{
    if (a >= 0.0)
        return upper_tail(a) - upper_tail(b);
    if (b <= 0.0)
        return upper_tail(-b) - upper_tail(-a);
    return 1.0 - upper_tail(-a) - upper_tail(b);
}

/* Inverse standard normal CDF by bisection on the tail function (init only). */
static double normal_quantile(double p)
{
    double lo = -40.0, hi = 40.0;
    int it;
    for (it = 0; it < 200; ++it) {
        double mid = 0.5 * (lo + hi);
        if (1.0 - upper_tail(mid) < p)
            lo = mid;
        else
            hi = mid;
    }
    return 0.5 * (lo + hi);
}

int orc_lloyd_max_gauss(int bits, double tol, int max_iter,
                        double *centroids, double *bounds, int *iters, double *residual)
{
    int L, i, it;
    double *t;           /* t[0] = -inf, t[1..L-1] interior boundaries, t[L] = +inf */
    double *dens, *tail, *ltail;
    double move = INFINITY;
    if (bits < 1 || bits > 12 || !centroids || !bounds)
        return -1;
    L = 1 << bits;
    t = (double *)malloc(sizeof(double) * (size_t)(4 * (L + 1)));
    if (!t)
        return -2;
    dens = t + (L + 1);
    tail = dens + (L + 1);
    ltail = tail + (L + 1);
    /* Start: centroids at the cell medians of the companding point density phi^(1/3),
     * i.e. quantiles of N(0, 3).  The optimum is unique for a log-concave density, so
     * the start only affects the number of iterations. */
    for (i = 0; i < L; ++i)
        centroids[i] = sqrt(3.0) * normal_quantile((i + 0.5) / L);
    t[0] = -INFINITY;
    t[L] = INFINITY;
    for (it = 0; it < max_iter; ++it) {
        /* condition 1: each boundary is the midpoint of its two neighbouring centroids */
        for (i = 1; i < L; ++i)
            t[i] = 0.5 * (centroids[i - 1] + centroids[i]);
        /* density and tail at every boundary, shared by the two cells that meet there */
        for (i = 0; i <= L; ++i) {
            dens[i] = phi(t[i]);
            tail[i] = upper_tail(t[i]);
            ltail[i] = upper_tail(-t[i]);
        }
        /* condition 2: each centroid is the conditional mean of its cell,
         * E[X | a <= X < b] = (phi(a) - phi(b)) / P(a <= X < b), P from the tail that
         * avoids cancellation */
        move = 0.0;
        for (i = 0; i < L; ++i) {
            double P;
            if (t[i] >= 0.0)
                P = tail[i] - tail[i + 1];
            else if (t[i + 1] <= 0.0)
                P = ltail[i + 1] - ltail[i];
            else
                P = 1.0 - ltail[i] - tail[i + 1];
            double c = (dens[i] - dens[i + 1]) / P;
            double dm = fabs(c - centroids[i]);
            if (dm > move)
                move = dm;
            centroids[i] = c;
        }
        /* keep the exact symmetry of the N(0,1) problem against rounding drift */
        for (i = 0; i < L / 2; ++i) {
            double m = 0.5 * (centroids[L - 1 - i] - centroids[i]);
            centroids[i] = -m;
            centroids[L - 1 - i] = m;
        }
        if (move <= tol) {
            ++it;
            break;
        }
    }
    for (i = 1; i < L; ++i)
        bounds[i - 1] = 0.5 * (centroids[i - 1] + centroids[i]);
    if (iters)
        *iters = it;
    if (residual)
        *residual = move;
    free(t);
    return move <= tol ? 0 : 1;
}

double orc_gauss_mse(int levels, const double *centroids, const double *bounds)
{
    /* Sum over cells of E[(X - c)^2 ; a <= X < b] using, for the standard normal,
     *   int_a^b phi = P,  int_a^b x phi = phi(a) - phi(b),
     *   int_a^b x^2 phi = P + a phi(a) - b phi(b)   (terms at infinity are 0). */
    double mse = 0.0;
    int i;
    for (i = 0; i < levels; ++i) {
        double a = (i == 0) ? -INFINITY : bounds[i - 1];
        double b = (i == levels - 1) ? INFINITY : bounds[i];
        double P = cell_prob(a, b);
        double m1 = phi(a) - phi(b);
        double aphi = isinf(a) ? 0.0 : a * phi(a);
        double bphi = isinf(b) ? 0.0 : b * phi(b);
        double m2 = P + aphi - bphi;
        double c = centroids[i];
        mse += m2 - 2.0 * c * m1 + c * c * P;
    }
    return mse;
}

/* ---------------------------------------------------------------------------------------
 * Exact marginal f_d.  A coordinate X of a uniform unit vector in R^d has
 * P(|X| <= r) = I_{r^2}(1/2, (d-1)/2) (X^2 ~ Beta(1/2, (d-1)/2)), density
 * (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2), and first moment over a cell in closed form:
 * int_a^b x f_d(x) dx = ((1 - a^2)^((d-1)/2) - (1 - b^2)^((d-1)/2)) / ((d-1) B(1/2, (d-1)/2)).
 * [RCAP] change-of-basis paragraph; the f3 variant of the codebook.
 * ------------------------------------------------------------------------------------- */

/* Continued fraction of I_x(a, b): I_x(a, b) = x^a (1-x)^b / (a B(a, b) F) with
 * F = 1 + d1 / (1 + d2 / (1 + ...)), d_{2m+1} = -(a+m)(a+b+m)x / ((a+2m)(a+2m+1)),
 * d_{2m} = m(b-m)x / ((a+2m-1)(a+2m)).  Returns F; converges quickly for
 * x < (a+1)/(a+b+2). */
static double betacf(double a, double b, double x)
{
    /* modified Lentz evaluation of F */
    const double tiny = 1e-300;
    double f = 1.0, C = 1.0, D = 0.0;
    int n;
    for (n = 1; n <= 100000; ++n) {
        int m = n / 2;
        double dn;
        if (n % 2 == 1)
            dn = -(a + m) * (a + b + m) * x / ((a + 2.0 * m) * (a + 2.0 * m + 1.0));
        else
            dn = m * (b - m) * x / ((a + 2.0 * m - 1.0) * (a + 2.0 * m));
        D = 1.0 + dn * D;
        if (fabs(D) < tiny)
            D = tiny;
        D = 1.0 / D;
        C = 1.0 + dn / C;
        if (fabs(C) < tiny)
            C = tiny;
        f *= C * D;
        if (fabs(C * D - 1.0) < 1e-16)
            break;
    }
    return f;
}

double orc_betainc(double a, double b, double x)
{
    double lfront;
    if (x <= 0.0)
        return 0.0;
    if (x >= 1.0)
        return 1.0;
    lfront = lgamma(a + b) - lgamma(a) - lgamma(b) + a * log(x) + b * log1p(-x);
    if (x < (a + 1.0) / (a + b + 2.0))
        return exp(lfront) / (a * betacf(a, b, x));
    return 1.0 - exp(lfront) / (b * betacf(b, a, 1.0 - x));
}

static double log_beta_half(int d)   /* log B(1/2, (d-1)/2) */
{
    double b = 0.5 * (d - 1);
    return lgamma(0.5) + lgamma(b) - lgamma(0.5 + b);
}

double orc_sphere_density(int d, double x)
{
    if (x <= -1.0 || x >= 1.0)
        return (d == 3 && fabs(x) == 1.0) ? 0.5 : 0.0;
    return exp(0.5 * (d - 3) * log1p(-x * x) - log_beta_half(d));
}

double orc_sphere_cdf(int d, double x)
{
    double half;
    if (x <= -1.0)
        return 0.0;
    if (x >= 1.0)
        return 1.0;
    half = 0.5 * orc_betainc(0.5, 0.5 * (d - 1), x * x);   /* P(0 <= X <= |x|) */
    return x >= 0.0 ? 0.5 + half : 0.5 - half;
}

/* P(|X| >= r) for r >= 0, without the cancellation of 1 - cdf. */
static double sphere_upper(int d, double r)
{
    if (r >= 1.0)
        return 0.0;
    return 0.5 * orc_betainc(0.5 * (d - 1), 0.5, 1.0 - r * r);   /* I_{1-r^2}(b, 1/2) / 2 */
}



int orc_lloyd_max_sphere(int d, int bits, double tol, int max_iter,
                         double *centroids, double *bounds, int *iters, double *residual)
{
    int L, i, it;
    double *t, *up, *g;
    double sd, k1, norm, move = INFINITY;
    if (d < 3 || bits < 1 || bits > 12 || !centroids || !bounds)
        return -1;
    L = 1 << bits;
    sd = 1.0 / sqrt((double)d);
    k1 = 0.5 * (d - 1);
    norm = (d - 1) * exp(log_beta_half(d));
    t = (double *)malloc(sizeof(double) * (size_t)(3 * (L + 1)));
    if (!t)
        return -2;
    up = t + (L + 1);     /* P(|X| >= |t_i|) at every boundary */
    g = up + (L + 1);     /* (1 - t_i^2)^((d-1)/2) at every boundary */
    /* Start: the Gaussian companding start scaled to the standard deviation 1/sqrt(d) and
     * squashed into (-1, 1).  f_d is log-concave for d >= 3, so the optimum is unique. */
    for (i = 0; i < L; ++i)
        centroids[i] = tanh(sqrt(3.0) * normal_quantile((i + 0.5) / L) * sd);
    t[0] = -1.0;
    t[L] = 1.0;
    for (it = 0; it < max_iter; ++it) {
        /* condition 1: boundaries at the midpoints of neighbouring centroids */
        for (i = 1; i < L; ++i)
            t[i] = 0.5 * (centroids[i - 1] + centroids[i]);
        /* tail and first-moment term at every boundary, shared by the two cells there */
        for (i = 0; i <= L; ++i) {
            up[i] = sphere_upper(d, fabs(t[i]));
            g[i] = fabs(t[i]) >= 1.0 ? 0.0 : exp(k1 * log1p(-t[i] * t[i]));
        }
        /* condition 2: centroid = E[X | cell] = first moment / probability */
        move = 0.0;
        for (i = 0; i < L; ++i) {
            double a = t[i], b = t[i + 1], P;
            if (a >= 0.0)
                P = up[i] - up[i + 1];
            else if (b <= 0.0)
                P = up[i + 1] - up[i];
            else
                P = 1.0 - up[i] - up[i + 1];
            double c = (g[i] - g[i + 1]) / norm / P;
            double dm = fabs(c - centroids[i]);
            if (dm > move)
                move = dm;
            centroids[i] = c;
        }
        for (i = 0; i < L / 2; ++i) {
            double m = 0.5 * (centroids[L - 1 - i] - centroids[i]);
            centroids[i] = -m;
            centroids[L - 1 - i] = m;
        }
        move /= sd;
        if (move <= tol) {
            ++it;
            break;
        }
    }
    for (i = 1; i < L; ++i)
        bounds[i - 1] = 0.5 * (centroids[i - 1] + centroids[i]);
    if (iters)
        *iters = it;
    if (residual)
        *residual = move;
    free(t);
    return move <= tol ? 0 : 1;
}

/* ---------------------------------------------------------------------------------------
 * Nearest centroid and packing.  [RCAP] pseudocode "nearest_centroid(...)".  The boundary
 * count with "<=" sends an exact tie to the upper cell (a reading).
 * ------------------------------------------------------------------------------------- */

int orc_code_of(double v, int levels, const double *unit_bounds, double sigma)
{
    int code = 0, j;
    for (j = 0; j < levels - 1; ++j)
        if (sigma * unit_bounds[j] <= v)
            ++code;
    return code;
}

void orc_pack(int n, int bits, const uint8_t *codes, uint8_t *out)
{
    int nbytes = (n * bits + 7) / 8;
    int k, b;
    memset(out, 0, (size_t)nbytes);
    for (k = 0; k < n; ++k)
        for (b = 0; b < bits; ++b) {
            int bit = k * bits + b;                 /* position in the row's bit stream */
            if ((codes[k] >> b) & 1)
                out[bit / 8] |= (uint8_t)(1u << (bit % 8));
        }
}

void orc_unpack(int n, int bits, const uint8_t *packed, uint8_t *codes)
{
    int k, b;
    for (k = 0; k < n; ++k) {
        unsigned c = 0;
        for (b = 0; b < bits; ++b) {
            int bit = k * bits + b;
            c |= (unsigned)((packed[bit / 8] >> (bit % 8)) & 1) << b;
        }
        codes[k] = (uint8_t)c;
    }
}

/* ---------------------------------------------------------------------------------------
 * Per-row quantizer: [RCAP] pseudocode, online per-token part (x_rot, s = norm(x_rot),
 * nearest_centroid(x_rot / (s + eps))) and, with eps = 0, the offline weight part
 * (W_rot rows, row_norms, nearest_centroid(W_rot / row_norms)).
 * ------------------------------------------------------------------------------------- */

int orc_quantize_rows_detail(int rows, int d, int h, const int32_t *perm,
                             const int8_t *sign, int bits, const double *unit_bounds,
                             double eps, const double *x, uint8_t *packed, double *norms,
                             double *z_out, double *u_out)
{
    int L = 1 << bits;
    int row_bytes = (d * bits) / 8;
    double sigma = 1.0 / sqrt((double)d);
    double *z = (double *)malloc(sizeof(double) * (size_t)d);
    uint8_t *codes = (uint8_t *)malloc((size_t)d);
    int r, k;
    if (!z || !codes) {
        free(z);
        free(codes);
        return -2;
    }
    if ((d * bits) % 8 != 0) {
        free(z);
        free(codes);
        return -1;
    }
    for (r = 0; r < rows; ++r) {
        const double *xr = x + (size_t)r * d;
        double ss = 0.0, s, denom;
        if (orc_rotate_row(d, h, perm, sign, xr, z) != 0) {
            free(z);
            free(codes);
            return -1;
        }
        for (k = 0; k < d; ++k)
            ss += z[k] * z[k];
        s = sqrt(ss);
        denom = s + eps;
        for (k = 0; k < d; ++k) {
            double v = (denom > 0.0) ? z[k] / denom : 0.0;
            codes[k] = (uint8_t)orc_code_of(v, L, unit_bounds, sigma);
            if (u_out)
                u_out[(size_t)r * d + k] = v / sigma;
        }
        if (z_out)
            memcpy(z_out + (size_t)r * d, z, sizeof(double) * (size_t)d);
        orc_pack(d, bits, codes, packed + (size_t)r * row_bytes);
        norms[r] = s;
    }
    free(z);
    free(codes);
    return 0;
}

int orc_quantize_rows(int rows, int d, int h, const int32_t *perm, const int8_t *sign,
                      int bits, const double *unit_bounds, double eps,
                      const double *x, uint8_t *packed, double *norms)
{
    return orc_quantize_rows_detail(rows, d, h, perm, sign, bits, unit_bounds, eps, x,
                                    packed, norms, NULL, NULL);
}

/* ---------------------------------------------------------------------------------------
 * Linear layer on codes.  [RCAP] rotation-cancellation paragraph (W R^T R x = W x) and the
 * pseudocode's W_hat = diag(row_norms) nearest_centroid(.) and x_hat = s nearest_centroid(.):
 * y = x_hat^T W_hat^T in the rotated basis.  Naive triple loop.
 * ------------------------------------------------------------------------------------- */

int orc_linear(int T, int d, int out, int bits_a, const double *ca, int bits_w,
               const double *cw, const uint8_t *x_packed, const double *s,
               const uint8_t *w_packed, const double *rn, double *y)
{
    double sigma = 1.0 / sqrt((double)d);
    int xa_bytes = (d * bits_a) / 8, w_bytes = (d * bits_w) / 8;
    uint8_t *xc = (uint8_t *)malloc((size_t)d);
    uint8_t *wc = (uint8_t *)malloc((size_t)out * d);
    int t, o, k;
    if (!xc || !wc) {
        free(xc);
        free(wc);
        return -2;
    }
    for (o = 0; o < out; ++o)
        orc_unpack(d, bits_w, w_packed + (size_t)o * w_bytes, wc + (size_t)o * d);
    for (t = 0; t < T; ++t) {
        orc_unpack(d, bits_a, x_packed + (size_t)t * xa_bytes, xc);
        for (o = 0; o < out; ++o) {
            const uint8_t *wr = wc + (size_t)o * d;
            double acc = 0.0;
            for (k = 0; k < d; ++k)
                acc += (sigma * ca[xc[k]]) * (sigma * cw[wr[k]]);
            y[(size_t)t * out + o] = s[t] * rn[o] * acc;
        }
    }
    free(xc);
    free(wc);
    return 0;
}
