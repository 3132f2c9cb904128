// oq_host.cpp -- host side of liboq: handles, table builders, validation and launches.
//
// Table builders follow rcap.io, "OrbitQuant: Data-Agnostic Quantization for Image and
// Video": pseudocode build_rpbh(d) (RPBH paragraph: uniform random permutation, random sign
// flips, block Walsh-Hadamard) and lloyd_max(f_d, b) (change-of-basis paragraph: the standard
// Lloyd-Max quantizer for the fixed marginal, read as N(0, 1/d)).  The generator and draw
// order are the ones documented in include/oq.h.
#include <algorithm>
#include <array>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <new>

#include "decode4.cuh"
#include "oq_internal.h"

namespace {

thread_local std::string g_last_error = "no error";

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int fail_cuda(cudaError_t e, const char *what) {
    return fail(OQ_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// Optional per-kernel timing (oq_timing_enable / oq_timing_collect): events recorded on the
// caller's stream around every kernel this thread launches through the C ABI.
struct TimedLaunch {
    int kernel;
    cudaEvent_t start, stop;
};
thread_local bool g_timing = false;
thread_local std::vector<TimedLaunch> g_timed;
thread_local std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess)
        return nullptr;
    return e;
}

// Run `launch` (returning cudaError_t), bracketed by events when timing is on.  While the
// stream is being captured into a CUDA graph the events are recorded as external event nodes,
// so each replay of the graph re-records them and they stay readable afterwards.
template <class F>
cudaError_t timed(int kernel, cudaStream_t st, F &&launch) {
    if (!g_timing)
        return launch();
    TimedLaunch t{kernel, take_event(), take_event()};
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(st, &cs);
    const unsigned flags =
        cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : cudaEventRecordDefault;
    if (t.start)
        cudaEventRecordWithFlags(t.start, st, flags);
    cudaError_t e = launch();
    if (t.stop)
        cudaEventRecordWithFlags(t.stop, st, flags);
    if (t.start && t.stop)
        g_timed.push_back(t);
    return e;
}

// Armed test of the kernels' bounded waits (oq_debug_arm_wait_timeout): one-shot, per thread.
thread_local int g_armed_kernel = 0;
thread_local long long g_armed_cycles = 0;

// The armed wait's limit for a launch of `kernel` (0 if not armed for it); disarms.
long long take_armed(int kernel) {
    if (g_armed_kernel != kernel)
        return 0;
    g_armed_kernel = 0;
    return g_armed_cycles;
}

// ---------------------------------------------------------------------------------------
// RPBH tables.  SplitMix64 (Steele, Lea & Flood 2014), Fisher-Yates (Durstenfeld) with
// rejection-sampled bounded integers, then one sign per position from the draw's top bit.
// ---------------------------------------------------------------------------------------
struct SplitMix64 {
    uint64_t x;
    uint64_t next() {
        uint64_t z = (x += 0x9E3779B97F4A7C15ULL);
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
        return z ^ (z >> 31);
    }
    // uniform in [0, n): reject the top 2^64 mod n values
    uint64_t below(uint64_t n) {
        const uint64_t cut = (uint64_t)(-n) % n;     // 2^64 mod n
        for (;;) {
            const uint64_t r = next();
            if (cut == 0 || r < (uint64_t)0 - cut)
                return r % n;
        }
    }
};

// ---------------------------------------------------------------------------------------
// Lloyd-Max: Lloyd warm-up, then Newton on the centroid conditions
// c_i = E[U | t_i <= U < t_{i+1}], t_i = (c_{i-1} + c_i)/2, with the tridiagonal Jacobian
// d mu_i / d t_i = f(t_i)(mu_i - t_i)/P_i,  d mu_i / d t_{i+1} = f(t_{i+1})(t_{i+1} - mu_i)/P_i,
// for a symmetric log-concave density f of the unit-scale coordinate U = sqrt(d) * x_rot / s.
// ---------------------------------------------------------------------------------------
double npdf(double x) { return std::isinf(x) ? 0.0 : std::exp(-0.5 * x * x) * 0.3989422804014327; }
double ntail(double x) {   // P(X > x)
    if (std::isinf(x))
        return x > 0 ? 0.0 : 1.0;
    return 0.5 * std::erfc(x * 0.7071067811865476);
}
double nprob(double a, double b) {   // P(a <= X < b), a < b
    if (a >= 0)
        return ntail(a) - ntail(b);
    if (b <= 0)
        return ntail(-b) - ntail(-a);
    return 1.0 - ntail(-a) - ntail(b);
}

// N(0,1): the marginal read as N(0, 1/d), in unit scale ([RCAP] change-of-basis paragraph).
struct GaussMarginal {
    double lo = -std::numeric_limits<double>::infinity();
    double hi = std::numeric_limits<double>::infinity();
    double pdf(double u) const { return npdf(u); }
    double prob(double a, double b) const { return nprob(a, b); }
    double moment(double a, double b) const { return npdf(a) - npdf(b); }
};

// Gauss-Legendre rule on [-1, 1]: nodes are the roots of P_n found by Newton's method from
// the usual cosine estimates, weights 2 / ((1 - x^2) P_n'(x)^2).
struct GaussLegendre {
    static constexpr int n = 12;
    double x[n], w[n];
    GaussLegendre() {
        const double pi = 3.14159265358979323846;
        for (int i = 0; i < n; ++i) {
            double z = std::cos(pi * (i + 0.75) / (n + 0.5)), dp = 1.0;
            for (int it = 0; it < 100; ++it) {
                double p0 = 1.0, p1 = z;                 // P_0, P_1
                for (int k = 2; k <= n; ++k) {           // (k) P_k = (2k-1) z P_{k-1} - (k-1) P_{k-2}
                    const double p2 = ((2.0 * k - 1.0) * z * p1 - (k - 1.0) * p0) / k;
                    p0 = p1;
                    p1 = p2;
                }
                dp = n * (z * p1 - p0) / (z * z - 1.0);  // P_n'(z)
                const double dz = p1 / dp;
                z -= dz;
                if (std::fabs(dz) < 1e-16)
                    break;
            }
            x[i] = z;
            w[i] = 2.0 / ((1.0 - z * z) * dp * dp);
        }
    }
};

// The exact marginal f_d of one coordinate of a uniform unit vector in R^d, in unit scale
// u = sqrt(d) x: f(u) = (1 - u^2/d)^((d-3)/2) / (sqrt(d) B(1/2, (d-1)/2)) on [-sqrt(d), sqrt(d)].
// Cell probabilities by composite 12-point Gauss-Legendre quadrature (panels of width <= 1/2,
// outside |u| > 45 the density is below 1e-400 and is dropped); first moments in closed form,
// int_a^b u f(u) du = sqrt(d) ((1 - a^2/d)^((d-1)/2) - (1 - b^2/d)^((d-1)/2)) / ((d-1) B).
struct SphereMarginal {
    double d, lo, hi, log_norm_pdf, mom_scale, cut;
    const GaussLegendre *gl;
    SphereMarginal(int dim, const GaussLegendre *rule) : d(dim), gl(rule) {
        hi = std::sqrt(d);
        lo = -hi;
        const double log_b = std::lgamma(0.5) + std::lgamma(0.5 * (d - 1)) - std::lgamma(0.5 * d);
        log_norm_pdf = -0.5 * std::log(d) - log_b;
        mom_scale = std::sqrt(d) / ((d - 1) * std::exp(log_b));
        cut = std::min(hi, 45.0);
    }
    double pdf(double u) const {
        if (u <= lo || u >= hi)
            return 0.0;
        return std::exp(0.5 * (d - 3) * std::log1p(-u * u / d) + log_norm_pdf);
    }
    double prob(double a, double b) const {
        a = std::max(a, -cut);
        b = std::min(b, cut);
        if (!(b > a))
            return 0.0;
        const int panels = (int)std::ceil((b - a) / 0.5);
        const double h = (b - a) / panels;
        double sum = 0.0;
        for (int k = 0; k < panels; ++k) {
            const double m = a + (k + 0.5) * h;
            for (int i = 0; i < GaussLegendre::n; ++i)
                sum += gl->w[i] * pdf(m + 0.5 * h * gl->x[i]);
        }
        return 0.5 * h * sum;
    }
    double moment(double a, double b) const {
        auto g = [&](double u) {
            return (u <= lo || u >= hi) ? 0.0 : std::exp(0.5 * (d - 1) * std::log1p(-u * u / d));
        };
        return mom_scale * (g(a) - g(b));
    }
};

template <class Marginal>
bool solve_lloyd_max(const Marginal &f, int L, std::vector<double> &c) {
    c.assign(L, 0.0);
    const double span = std::min(1.5 + 0.4 * std::log2((double)L), 0.9 * f.hi);
    for (int i = 0; i < L; ++i)
        c[i] = span * (2.0 * (i + 0.5) / L - 1.0);
    std::vector<double> t(L + 1), mu(L), da(L), db(L);
    auto cells = [&]() {
        t[0] = f.lo;
        t[L] = f.hi;
        for (int i = 1; i < L; ++i)
            t[i] = 0.5 * (c[i - 1] + c[i]);
        for (int i = 0; i < L; ++i) {
            const double a = t[i], b = t[i + 1];
            const double P = f.prob(a, b);
            mu[i] = f.moment(a, b) / P;
            da[i] = i == 0 ? 0.0 : f.pdf(a) * (mu[i] - a) / P;          // support edges
            db[i] = i == L - 1 ? 0.0 : f.pdf(b) * (b - mu[i]) / P;      // are not free
        }
    };
    // Lloyd iterations bring every cell near the optimum
    for (int it = 0; it < 400 + 4 * L; ++it) {
        cells();
        for (int i = 0; i < L; ++i)
            c[i] = mu[i];
    }
    // Newton with step halving that keeps the centroids ordered
    std::vector<double> lo(L), di(L), up(L), r(L), step(L), cp(L), dp(L);
    for (int it = 0; it < 60; ++it) {
        cells();
        double rmax = 0.0;
        for (int i = 0; i < L; ++i) {
            r[i] = c[i] - mu[i];
            rmax = std::max(rmax, std::fabs(r[i]));
            lo[i] = -0.5 * da[i];
            up[i] = -0.5 * db[i];
            di[i] = 1.0 - 0.5 * (da[i] + db[i]);
        }
        if (rmax < 1e-15)
            break;
        // Thomas algorithm (diagonally dominant: da + db < 1 for a log-concave density)
        cp[0] = up[0] / di[0];
        dp[0] = r[0] / di[0];
        for (int i = 1; i < L; ++i) {
            const double m = di[i] - lo[i] * cp[i - 1];
            cp[i] = up[i] / m;
            dp[i] = (r[i] - lo[i] * dp[i - 1]) / m;
        }
        step[L - 1] = dp[L - 1];
        for (int i = L - 2; i >= 0; --i)
            step[i] = dp[i] - cp[i] * step[i + 1];
        double lam = 1.0;
        for (int tries = 0; tries < 30; ++tries, lam *= 0.5) {
            bool ordered = true;
            for (int i = 1; i < L && ordered; ++i)
                ordered = (c[i] - lam * step[i]) > (c[i - 1] - lam * step[i - 1]);
            if (ordered)
                break;
        }
        for (int i = 0; i < L; ++i)
            c[i] -= lam * step[i];
    }
    // exact symmetry of the (symmetric) problem
    for (int i = 0; i < L / 2; ++i) {
        const double m = 0.5 * (c[L - 1 - i] - c[i]);
        c[i] = -m;
        c[L - 1 - i] = m;
    }
    cells();
    double rmax = 0.0;
    for (int i = 0; i < L; ++i)
        rmax = std::max(rmax, std::fabs(c[i] - mu[i]));
    return rmax < 1e-12;
}

// IEEE binary16, round to nearest even (normal range and zero; centroids are in [1e-3, 5]).
uint16_t to_half_bits(double x) {
    uint16_t sgn = std::signbit(x) ? 0x8000 : 0;
    x = std::fabs(x);
    if (x == 0.0)
        return sgn;
    int e;
    const double m = std::frexp(x, &e);          // x = m 2^e, m in [0.5, 1)
    int E = e - 1 + 15;                           // x = (2m) 2^(e-1)
    if (E <= 0)
        return sgn;                               // not reached for codebook values
    double frac = (2.0 * m - 1.0) * 1024.0;
    double fl = std::floor(frac);
    uint32_t f = (uint32_t)fl;
    const double rem = frac - fl;
    if (rem > 0.5 || (rem == 0.5 && (f & 1u)))
        ++f;
    if (f == 1024) {
        f = 0;
        ++E;
    }
    if (E >= 31)
        return (uint16_t)(sgn | 0x7C00);
    return (uint16_t)(sgn | (E << 10) | f);
}

}  // namespace

// ---------------------------------------------------------------------------------------
// Handles.
// ---------------------------------------------------------------------------------------
struct oq_rpbh {
    int d = 0, h = 0;
    uint64_t seed = 0;
    std::vector<int32_t> perm;
    std::vector<int8_t> sign;
    std::vector<uint32_t> ent_img[2];             // K1 gather-entry images: [0] bf16, [1] fp32
    std::vector<uint16_t> ent16;                  // tensor-core K1: perm[i] | sign bit << 15
    std::mutex mu;
    uint32_t *dev_ent[2][oq::kMaxDevices] = {};
    uint32_t *dev_ent16[oq::kMaxDevices] = {};
};

struct oq_codebook {
    int d = 0, bits = 0, marginal = OQ_MARGINAL_GAUSSIAN;
    std::vector<double> c, t;                     // unit centroids / boundaries
    uint16_t lut[256] = {};                       // unit centroids, fp16 bits
    int G = 0, F = 0;
    double delta = 0.0;
    std::vector<uint32_t> grid;                   // G + 1 words
    std::vector<uint32_t> tbl_img;                // K1 shared-memory image of the table
    std::vector<uint32_t> dec_img;                // K1 fp16 output: byte -> centroids (b 2,4,8)
    std::mutex mu;
    uint32_t *dev_tbl[oq::kMaxDevices] = {};
    uint32_t *dev_dec[oq::kMaxDevices] = {};
};

namespace {

// Uniform grid over the unit axis with at most one boundary per cell; see include/oq.h.
bool build_grid(oq_codebook *cb) {
    const int L = 1 << cb->bits;
    double gap = std::numeric_limits<double>::infinity(), tmax = 0.0;
    for (int j = 0; j + 1 < L - 1; ++j)
        gap = std::min(gap, cb->t[j + 1] - cb->t[j]);
    for (double v : cb->t)
        tmax = std::max(tmax, std::fabs(v));
    if (L - 1 == 1)
        gap = 2.0 * tmax > 0 ? 2.0 * tmax : 1.0;
    for (double shrink = 0.999; shrink > 0.1; shrink *= 0.5) {
        const double delta = gap * shrink;
        int G = 8;
        while (G * delta < 2.0 * tmax * 1.001 + 2.0 * delta)
            G *= 2;
        if (G > (1 << 20))
            return false;
        int lg = 0;
        while ((1 << lg) < G)
            ++lg;
        const int F = 23 - lg;
        const double two23 = 8388608.0;
        std::vector<long long> qthr(L - 1), cell(L - 1);
        bool ok = true;
        for (int j = 0; j < L - 1; ++j) {
            const double A = cb->t[j] / (G * delta) + 0.5;
            qthr[j] = (long long)std::ceil(A * two23);
            cell[j] = qthr[j] >> F;
            if (qthr[j] <= 0 || qthr[j] >= (1LL << 23))
                ok = false;
            if (j > 0 && cell[j] == cell[j - 1])
                ok = false;                       // two boundaries in one cell
        }
        if (!ok)
            continue;
        cb->G = G;
        cb->F = F;
        cb->delta = delta;
        cb->grid.assign(G + 1, 0);
        for (int k = 0; k <= G; ++k) {
            long long base = 0, thr = ((long long)k + 1) << F;   // unreachable by default
            for (int j = 0; j < L - 1; ++j) {
                if (cell[j] < k)
                    ++base;
                else if (cell[j] == k)
                    thr = qthr[j];
            }
            const uint32_t word = (uint32_t)((uint64_t)(base + 1) << 24) -
                                  (uint32_t)((uint64_t)(thr + 0x3F800000LL) * (uint64_t)G);
            cb->grid[k] = word;
        }
        return true;
    }
    return false;
}

struct DeviceInfo {
    int checked = 0;       // 0 unknown, 1 ok, -1 unsupported
    int sms = 0;
    cudaMemPool_t pool = nullptr;
    cudaStream_t side = nullptr;      // oq_quantized_linear: weight decode beside K1
    cudaEvent_t fork = nullptr, join = nullptr;
    uint32_t *gelu_tab = nullptr;     // the fused GELU's table (oq::gelu_table_image)
};
DeviceInfo g_dev[oq::kMaxDevices];
std::mutex g_dev_mu;

int current_device(int *dev_out, DeviceInfo **info_out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return fail_cuda(e, "cudaGetDevice");
    if (dev < 0 || dev >= oq::kMaxDevices)
        return fail(OQ_EUNSUPPORTED, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &di = g_dev[dev];
    if (di.checked == 0) {
        int major = 0, minor = 0, sms = 0;
        cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess)
            return fail_cuda(e, "cudaDeviceGetAttribute");
        di.checked = (major == 10 && minor == 0) ? 1 : -1;
        di.sms = sms;
    }
    if (di.checked < 0)
        return fail(OQ_EUNSUPPORTED, "device %d is not sm_100 (B200 class); liboq is built for "
                                     "sm_100a only", dev);
    *dev_out = dev;
    *info_out = &di;
    return OQ_OK;
}

template <class T>
int upload(std::mutex &mu, uint32_t **slot, const std::vector<T> &host, const char *what) {
    std::lock_guard<std::mutex> lk(mu);
    if (*slot)
        return OQ_OK;
    void *p = nullptr;
    cudaError_t e = cudaMalloc(&p, host.size() * sizeof(T));
    if (e != cudaSuccess)
        return fail_cuda(e, what);
    e = cudaMemcpy(p, host.data(), host.size() * sizeof(T), cudaMemcpyHostToDevice);
    if (e != cudaSuccess) {
        cudaFree(p);
        return fail_cuda(e, what);
    }
    *slot = static_cast<uint32_t *>(p);
    return OQ_OK;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// y rows are written by TMA tensor stores, whose global row stride must be a multiple of 16
// bytes: out_features a multiple of 4 for fp32 y, of 8 for bf16 y.
bool out_rows_aligned(int out_features, int out_dtype) {
    return ((long long)out_features * (out_dtype == OQ_BF16 ? 2 : 4)) % 16 == 0;
}

int check_dims(int d, const char *who) {
    if (d < 128 || d > 16384 || d % 128 != 0)
        return fail(OQ_EINVAL, "%s: d = %d must be a multiple of 128 in [128, 16384]", who, d);
    return OQ_OK;
}

// OQ_K1_PATH=tc sends bf16 rows (h <= 256, d up to ~3.9K) to the tensor-core rotate+quantize
// kernel instead of the CUDA-core one (read once per process).
bool tc_k1_requested() {
    static const bool v = [] {
        const char *e = std::getenv("OQ_K1_PATH");
        return e != nullptr && std::strcmp(e, "tc") == 0;
    }();
    return v;
}

// K1 for `rows` rows of x: packed codes into `codes`, or (a16 non-null, bits 2/4/8, bf16, h <=
// 256) the codes' fp16 unit centroids into a16 [rows, d]; norms into `norms`.
// A weight decode that K1 takes on (fp16 output, whole-warp groups, 4-bit weights of an
// odd-symmetric codebook): the codes of `rows` weight rows into fp16 unit centroids.
struct FusedDecode {
    const oq_codebook *cb = nullptr;
    const uint8_t *codes = nullptr;
    uint16_t *out = nullptr;
    long long rows = 0;
};

int quantize_rows(const oq_rpbh *r, const oq_codebook *cb, const void *x, int dtype, int rows,
                  int d, uint8_t *codes, float *norms, void *stream, float eps,
                  const char *who, bool gelu = false, uint16_t *a16 = nullptr,
                  const FusedDecode *fd = nullptr) {
    if (!r || !cb)
        return fail(OQ_EINVAL, "%s: null handle", who);
    if (check_dims(d, who) != OQ_OK)
        return OQ_EINVAL;
    if (r->d != d || cb->d != d)
        return fail(OQ_EINVAL, "%s: d = %d but rotation has d = %d and codebook d = %d", who, d,
                    r->d, cb->d);
    if (dtype != OQ_F32 && dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: dtype must be OQ_F32 or OQ_BF16", who);
    if (gelu && dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: the fused GELU takes bf16 input", who);
    if (rows < 0)
        return fail(OQ_EINVAL, "%s: negative row count %d", who, rows);
    if (rows == 0)
        return OQ_OK;
    uint8_t *out = a16 ? reinterpret_cast<uint8_t *>(a16) : codes;
    if (!x || !out || !norms)
        return fail(OQ_EINVAL, "%s: null data pointer", who);
    if (!aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(norms) & 3u))
        return fail(OQ_EINVAL, "%s: x and codes must be 16-byte aligned, norms 4-byte", who);
    int dev;
    DeviceInfo *di;
    int rc = current_device(&dev, &di);
    if (rc != OQ_OK)
        return rc;
    oq_rpbh *rw = const_cast<oq_rpbh *>(r);
    oq_codebook *cw = const_cast<oq_codebook *>(cb);
    if ((rc = upload(cw->mu, &cw->dev_tbl[dev], cw->tbl_img, "upload quantizer table")) != OQ_OK)
        return rc;
    const float Kq = (float)(std::sqrt((double)d / r->h) / (cb->G * cb->delta));
    std::string why;
    cudaStream_t st = (cudaStream_t)stream;
    if (dtype == OQ_BF16 && !gelu && !a16 && tc_k1_requested() &&
        oq::k1_tc_supported(d, r->h, cb->bits, (int)cw->tbl_img.size())) {
        // block transform on the tensor cores
        if ((rc = upload(rw->mu, &rw->dev_ent16[dev], rw->ent16, "upload rotation entries")) !=
            OQ_OK)
            return rc;
        oq::K1TcParams p{};
        p.x = static_cast<const uint8_t *>(x);
        p.codes = codes;
        p.norms = norms;
        p.ent = reinterpret_cast<const uint16_t *>(rw->dev_ent16[dev]);
        p.tbl_img = cw->dev_tbl[dev];
        p.tbl_words = (int)cw->tbl_img.size();
        p.T = rows;
        p.d = d;
        p.h = r->h;
        p.eps = eps;
        p.K = Kq;
        p.G = cb->G;
        p.F = cb->F;
        cudaError_t e = timed(OQ_KERNEL_QUANTIZE, st, [&] {
            return oq::launch_k1_tc(p, cb->bits, st, di->sms, &why);
        });
        if (e != cudaSuccess)
            return fail_cuda(e, why.c_str());
        return OQ_OK;
    }
    const int f = dtype == OQ_F32 ? 1 : 0;
    if ((rc = upload(rw->mu, &rw->dev_ent[f][dev], rw->ent_img[f], "upload rotation table")) !=
        OQ_OK)
        return rc;
    oq::K1Params p{};
    p.x = x;
    p.codes = codes;
    p.norms = norms;
    p.ent_img = rw->dev_ent[f][dev];
    p.tbl_img = cw->dev_tbl[dev];
    p.ent_words = (int)rw->ent_img[f].size();
    p.tbl_words = (int)cw->tbl_img.size();
    p.T = rows;
    p.d = d;
    p.h = r->h;
    p.eps = eps;
    p.K = Kq;
    p.G = cb->G;
    p.F = cb->F;
    p.gelu = gelu ? 1 : 0;
    if (gelu) {
        static std::mutex gelu_mu;
        static const std::vector<uint32_t> gelu_img = oq::gelu_table_image();
        if ((rc = upload(gelu_mu, &di->gelu_tab, gelu_img, "upload GELU table")) != OQ_OK)
            return rc;
        p.gelu_img = di->gelu_tab;
        p.gelu_words = (int)gelu_img.size();
    }
    p.test_wait_cycles = take_armed(OQ_KERNEL_QUANTIZE);
    if (a16) {
        if (!oq::k1_a16_supported(cb->bits, r->h, dtype == OQ_BF16))
            return fail(OQ_EINVAL, "%s: no fp16 centroid output for bits %d, h %d", who,
                        cb->bits, r->h);
        if ((rc = upload(cw->mu, &cw->dev_dec[dev], cw->dec_img, "upload decode table")) != OQ_OK)
            return rc;
        p.a16 = a16;
        if (cb->bits == 4) {
            if (!oq::decode8_sources(cb->lut, &p.dec_src[0], &p.dec_src[1], &p.dec_src[2],
                                     &p.dec_src[3]))
                return fail(OQ_EINVAL, "%s: 4-bit codebook is not odd-symmetric", who);
        } else {
            p.dec_img = cw->dev_dec[dev];
            p.dec_words = (int)cw->dec_img.size();
        }
    }
    {
        if (fd && fd->rows > 0) {
            oq_codebook *fw = const_cast<oq_codebook *>(fd->cb);
            if (fw->bits == 4) {
                if (!oq::decode8_sources(fw->lut, &p.wdec_src[0], &p.wdec_src[1],
                                         &p.wdec_src[2], &p.wdec_src[3]))
                    return fail(OQ_EINVAL, "%s: 4-bit weight codebook is not odd-symmetric",
                                who);
            } else if (fw->bits == 2) {
                if ((rc = upload(fw->mu, &fw->dev_dec[dev], fw->dec_img,
                                 "upload weight decode table")) != OQ_OK)
                    return rc;
                p.wdec_img = fw->dev_dec[dev];
                p.wdec_words = (int)fw->dec_img.size();
            } else {
                return fail(OQ_EINVAL, "%s: fused weight decode takes 2- or 4-bit codes", who);
            }
            p.wdec_bits = fw->bits;
            p.wdec_codes = reinterpret_cast<const uint32_t *>(fd->codes);
            p.wdec_out = reinterpret_cast<uint4 *>(fd->out);
            p.wdec_groups = fd->rows * (long long)d * fw->bits / 32;
        }
    }
    cudaError_t e = timed(OQ_KERNEL_QUANTIZE, st, [&] {
        return oq::launch_k1(p, cb->bits, r->h, dtype == OQ_F32, st, di->sms, &why);
    });
    if (e != cudaSuccess)
        return fail_cuda(e, why.c_str());
    return OQ_OK;
}

cudaMemPool_t device_pool(int dev, DeviceInfo *di, int *rc) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (di->pool)
        return di->pool;
    cudaMemPoolProps props{};
    props.allocType = cudaMemAllocationTypePinned;
    props.location.type = cudaMemLocationTypeDevice;
    props.location.id = dev;
    cudaMemPool_t pool;
    cudaError_t e = cudaMemPoolCreate(&pool, &props);
    if (e != cudaSuccess) {
        *rc = fail_cuda(e, "cudaMemPoolCreate");
        return nullptr;
    }
    uint64_t keep = std::numeric_limits<uint64_t>::max();
    cudaMemPoolSetAttribute(pool, cudaMemPoolAttrReleaseThreshold, &keep);
    di->pool = pool;
    return pool;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// The library's side stream of a device and the two events oq_quantized_linear forks and joins
// it with (created once; nullptr and *rc set on failure).
std::mutex g_side_mu;          // serialises the fork/join enqueues of concurrent callers
cudaStream_t device_side(DeviceInfo *di, int *rc) {
    std::lock_guard<std::mutex> lk(g_dev_mu);
    if (di->side)
        return di->side;
    cudaStream_t st = nullptr;
    cudaEvent_t a = nullptr, b = nullptr;
    cudaError_t e = cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking);
    if (e == cudaSuccess)
        e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
    if (e == cudaSuccess)
        e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
    if (e != cudaSuccess) {
        *rc = fail_cuda(e, "side stream / events");
        return nullptr;
    }
    di->fork = a;
    di->join = b;
    di->side = st;
    return st;
}

// OQ_LINEAR_PATH (read once per process): "fused" decodes 4-bit activation codes inside the
// GEMM kernel instead of in the prepass (no [T, d] fp16 workspace, but each 128-row tile of
// codes is decoded once per 256-column tile of the output); "wcodes" decodes 4-bit weight
// codes inside the CTA-pair GEMM (no [N, d] fp16 workspace and no weight decode launch, but
// each weight row is decoded once per 256-row tile of the output).
int linear_path() {
    static const int v = [] {
        const char *e = std::getenv("OQ_LINEAR_PATH");
        if (e != nullptr && std::strcmp(e, "fused") == 0)
            return 1;
        if (e != nullptr && std::strcmp(e, "wcodes") == 0)
            return 2;
        return 0;
    }();
    return v;
}
bool fused_requested() { return linear_path() == 1; }

// The weight operand of this codebook decoded inside the GEMM: 4-bit codes of an
// odd-symmetric codebook and the CTA-pair GEMM, with OQ_LINEAR_PATH=wcodes, or by default when
// T <= 256 (one 256-row tile: each weight row is decoded once either way, and the call saves
// the decode launch and the [N, d] fp16 buffer; measured 19.8-22.8 against 24.6-28.0 us per
// one-call step at d = N = 3072).
bool wcodes_applies(const oq_codebook *cw, int T) {
    uint32_t src[4];
    const int path = linear_path();
    return (path == 2 || (path == 0 && T <= 256)) && cw->bits == 4 &&
           oq::gemm_pair_enabled() &&
           oq::decode8_sources(cw->lut, &src[0], &src[1], &src[2], &src[3]);
}

// OQ_FUSED_STEP=1 runs oq_quantized_linear as one persistent kernel (k3_fused.cu) where it
// applies (read once per process).
bool fused_step_requested() {
    static const bool v = [] {
        const char *e = std::getenv("OQ_FUSED_STEP");
        return e != nullptr && std::strcmp(e, "1") == 0;
    }();
    return v;
}

// Token pairs each ramp group of the fused step quantizes before its GEMM roles
// (OQ_FUSED_RAMP = 0..8, read once per process; 0, no ramp groups, unless set).
int fused_ramp_rounds() {
    static const int v = [] {
        const char *e = std::getenv("OQ_FUSED_RAMP");
        if (e == nullptr || e[0] < '0' || e[0] > '8' || e[1] != '\0')
            return 0;
        return e[0] - '0';
    }();
    return v;
}

// oq_quantized_linear as one persistent kernel: the decode prepass of the weights, then the
// quantize stage and the CTA-pair GEMM side by side (k3_fused.cu).  Arguments validated by
// the caller.
int fused_step(const oq_rpbh *r, const oq_codebook *ca, const oq_codebook *cw, const void *x,
               const uint8_t *W_codes, const float *row_norms, int T, int d, int out_features,
               void *y, int out_dtype, float *s, cudaStream_t st, int dev, DeviceInfo *di,
               cudaMemPool_t pool, const char *who) {
    oq_rpbh *rw = const_cast<oq_rpbh *>(r);
    oq_codebook *caw = const_cast<oq_codebook *>(ca);
    int rc;
    if ((rc = upload(caw->mu, &caw->dev_tbl[dev], caw->tbl_img, "upload quantizer table")) !=
        OQ_OK)
        return rc;
    if ((rc = upload(rw->mu, &rw->dev_ent[0][dev], rw->ent_img[0], "upload rotation table")) !=
        OQ_OK)
        return rc;
    oq::FusedStepParams p{};
    if (ca->bits == 4) {
        if (!oq::decode8_sources(ca->lut, &p.dec_src[0], &p.dec_src[1], &p.dec_src[2],
                                 &p.dec_src[3]))
            return fail(OQ_EINVAL, "%s: 4-bit codebook is not odd-symmetric", who);
    } else {
        if ((rc = upload(caw->mu, &caw->dev_dec[dev], caw->dec_img, "upload decode table")) !=
            OQ_OK)
            return rc;
        p.dec_img = caw->dev_dec[dev];
        p.dec_words = (int)caw->dec_img.size();
    }
    // workspace: A16 [T, d] | B16 [N, d] | s [T] (if not given) | progress counters
    const size_t a_bytes = align_up((size_t)T * d * 2, 1024);
    const size_t b_bytes = align_up((size_t)out_features * d * 2, 1024);
    const size_t s_bytes = s ? 0 : align_up((size_t)T * 4, 1024);
    const size_t c_bytes = align_up(4 * oq::fused_step_counter_words(T, out_features), 256);
    void *ws = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(&ws, a_bytes + b_bytes + s_bytes + c_bytes, pool, st);
    if (e != cudaSuccess)
        return fail_cuda(e, "oq_quantized_linear: workspace allocation");
    unsigned char *w8 = static_cast<unsigned char *>(ws);
    uint16_t *A16 = reinterpret_cast<uint16_t *>(w8);
    uint16_t *B16 = reinterpret_cast<uint16_t *>(w8 + a_bytes);
    float *sv = s ? s : reinterpret_cast<float *>(w8 + a_bytes + b_bytes);
    unsigned *ctr = reinterpret_cast<unsigned *>(w8 + a_bytes + b_bytes + s_bytes);
    std::string why;
    // 2-bit weights, or 4-bit weights of an odd-symmetric codebook: decoded inside the kernel
    oq_codebook *cww = const_cast<oq_codebook *>(cw);
    bool wdec_in = false;
    if (cw->bits == 4 && oq::decode8_sources(cw->lut, &p.wdec_src[0], &p.wdec_src[1],
                                             &p.wdec_src[2], &p.wdec_src[3])) {
        wdec_in = true;
    } else if (cw->bits == 2) {
        if ((rc = upload(cww->mu, &cww->dev_dec[dev], cww->dec_img,
                         "upload weight decode table")) != OQ_OK) {
            cudaFreeAsync(ws, st);
            return rc;
        }
        p.wdec_tab = reinterpret_cast<const uint2 *>(cww->dev_dec[dev]);
        wdec_in = true;
    }
    if (wdec_in) {
        p.wcodes = reinterpret_cast<const uint32_t *>(W_codes);
        p.b16 = reinterpret_cast<uint4 *>(B16);
        p.wdec_words = (long long)out_features * d * cw->bits / 32;
        p.wdec_bits = cw->bits;
    }
    e = timed(OQ_KERNEL_AUX, st, [&] {
        return oq::launch_zero_counters(ctr, (int)oq::fused_step_counter_words(T, out_features),
                                        st);
    });
    if (e == cudaSuccess && !wdec_in)
        e = timed(OQ_KERNEL_DECODE, st, [&] {
            return oq::launch_decode(cw->bits, W_codes, B16, out_features, d, cw->lut, st,
                                     di->sms, &why);
        });
    if (e == cudaSuccess) {
        p.x = static_cast<const unsigned char *>(x);
        p.a16 = A16;
        p.s = sv;
        p.ent_img = rw->dev_ent[0][dev];
        p.tbl_img = caw->dev_tbl[dev];
        p.ent_words = (int)rw->ent_img[0].size();
        p.tbl_words = (int)caw->tbl_img.size();
        p.eps = 1e-8f;
        p.K = (float)(std::sqrt((double)d / r->h) / (ca->G * ca->delta));
        p.G = ca->G;
        p.F = ca->F;
        p.rn = row_norms;
        p.T = T;
        p.N = out_features;
        p.d = d;
        p.inv_d = 1.0f / (float)d;
        p.ctr = ctr;
        p.test_wait_cycles = take_armed(OQ_KERNEL_GEMM);
        p.ramp_rounds = fused_ramp_rounds();
        e = timed(OQ_KERNEL_FUSED, st, [&] {
            return oq::launch_fused_step(p, ca->bits, r->h, out_dtype == OQ_BF16, B16, y, st,
                                         &why);
        });
    }
    cudaError_t e2 = cudaFreeAsync(ws, st);
    if (e != cudaSuccess)
        return fail_cuda(e, why.empty() ? "oq_quantized_linear: fused step" : why.c_str());
    if (e2 != cudaSuccess)
        return fail_cuda(e2, "oq_quantized_linear: workspace release");
    return OQ_OK;
}

}  // namespace

namespace oq {

// GELU(x) = x Phi(x) = x erfc(-x / sqrt 2) / 2 in fp64, rounded to fp32, for every bf16 x with
// 2^-16 <= |x| < 16: entry sign * 2560 + (e + 16) * 128 + m holds |x| = (1 + m/128) 2^e.
std::vector<uint32_t> gelu_table_image() {
    std::vector<uint32_t> img(5120);
    for (int sgn = 0; sgn < 2; ++sgn)
        for (int e = -16; e <= 3; ++e)
            for (int m = 0; m < 128; ++m) {
                const double x = (sgn ? -1.0 : 1.0) * std::ldexp(1.0 + m / 128.0, e);
                const float g = (float)(0.5 * x * std::erfc(-x / std::sqrt(2.0)));
                uint32_t u;
                std::memcpy(&u, &g, 4);
                img[(size_t)sgn * 2560 + (size_t)(e + 16) * 128 + m] = u;
            }
    return img;
}

}  // namespace oq

// ---------------------------------------------------------------------------------------
// C ABI.
// ---------------------------------------------------------------------------------------
extern "C" {

namespace {

// RPBH tables (permute = true) or Block-RHT tables (the same draws, identity permutation).
// Pair-buffer slot colours for the bf16 K1 (layout in oq_internal.h).  The staged token pair
// lives in 16-byte slots of 4 positions; thread g's interleave writes the two halves of chunks
// c = g + k*GT (k = 0..3, GT = d/32) to slot (2k + lh)*GT + (g & ~7) + colour, where the colours
// of each octet of threads are a permutation of 0..7 (so every quarter-warp store covers all
// banks).  The gather of rotated position i reads slot word (j & 3) of j = perm[i] with the
// 32 lanes of a warp at the same step e reading positions perm[32g + e]; its bank is
// 4 * colour + (j & 3).  A local search over colour swaps inside each octet lowers the sum
// over (warp, step) of the largest number of lanes on one bank (for a random permutation
// from about 3.6 to about 2.1 per load; for the identity, from 16 to 4).  The search runs
// for the named-barrier K1, whose groups start at a warp (padded to whole warps); groups
// that share warps (the lockstep K1) keep colour = g & 7.
std::vector<uint8_t> pair_slot_colours(const std::vector<int32_t> &perm, int d) {
    const int GT = d / 32, NH = d / 4;
    std::vector<uint8_t> col(NH);
    for (int h = 0; h < NH; ++h) {
        const int c = h >> 1, g = c % GT;
        col[h] = (uint8_t)(((g & ~7) + 8 <= GT) ? ((g + (c / GT) * 3) & 7) : (g & 7));
    }
    if (!oq::k1_named(d, true))
        return col;
    // reads of each half-chunk: (event = warp * 32 + step, j & 3)
    std::vector<std::array<std::pair<int, int>, 4>> reads(NH);
    std::vector<int> nread(NH, 0);
    for (int i = 0; i < d; ++i) {
        const int j = perm[i], g = i >> 5, e = i & 31;
        reads[j >> 2][nread[j >> 2]++] = {(g >> 5) * 32 + e, j & 3};
    }
    const int NE = ((GT + 31) / 32) * 32;
    std::vector<int> cnt((size_t)NE * 32, 0);
    for (int h = 0; h < NH; ++h)
        for (int t = 0; t < 4; ++t)
            ++cnt[(size_t)reads[h][t].first * 32 + 4 * col[h] + reads[h][t].second];
    auto evmax = [&](int ev) {
        int m = 0;
        for (int b = 0; b < 32; ++b)
            m = std::max(m, cnt[(size_t)ev * 32 + b]);
        return m;
    };
    auto move = [&](int h, int from, int to) {
        for (int t = 0; t < 4; ++t) {
            const size_t base = (size_t)reads[h][t].first * 32 + reads[h][t].second;
            --cnt[base + 4 * from];
            ++cnt[base + 4 * to];
        }
    };
    SplitMix64 rng{0x5eedULL + (uint64_t)d};
    const long long iters = std::min(60LL * NH, 200000LL);
    int evs[8];
    for (long long it = 0; it < iters; ++it) {
        // a random octet (g0, k, lh) and two of its members
        const int oct = (int)rng.below((uint64_t)(GT / 8) * 8);
        const int g0 = (oct >> 3) * 8, k = (oct >> 1) & 3, lh = oct & 1;
        const int a = (int)rng.below(8), b = (int)rng.below(7);
        const int ha = 2 * (g0 + a + k * GT) + lh;
        const int hb = 2 * (g0 + (b >= a ? b + 1 : b) + k * GT) + lh;
        int ne = 0;
        for (int t = 0; t < 4; ++t) {
            evs[ne++] = reads[ha][t].first;
            evs[ne++] = reads[hb][t].first;
        }
        std::sort(evs, evs + ne);
        ne = (int)(std::unique(evs, evs + ne) - evs);
        int before = 0, after = 0;
        for (int q = 0; q < ne; ++q)
            before += evmax(evs[q]);
        const int ca = col[ha], cb = col[hb];
        move(ha, ca, cb);
        move(hb, cb, ca);
        for (int q = 0; q < ne; ++q)
            after += evmax(evs[q]);
        if (after <= before) {
            col[ha] = (uint8_t)cb;
            col[hb] = (uint8_t)ca;
        } else {
            move(ha, cb, ca);
            move(hb, ca, cb);
        }
    }
    return col;
}

int build_rotation(int d, int h, uint64_t seed, bool permute, oq_rpbh **out, const char *who) {
    if (!out)
        return fail(OQ_EINVAL, "%s: out is NULL", who);
    *out = nullptr;
    if (check_dims(d, who) != OQ_OK)
        return OQ_EINVAL;
    if (h < 2 || h > 1024 || (h & (h - 1)) != 0 || d % h != 0)
        return fail(OQ_EINVAL, "%s: h = %d must be a power of two in [2, 1024] dividing "
                               "d = %d", who, h, d);
    oq_rpbh *r = new (std::nothrow) oq_rpbh;
    if (!r)
        return fail(OQ_ENOMEM, "%s: out of host memory", who);
    r->d = d;
    r->h = h;
    r->seed = seed;
    r->perm.resize(d);
    r->sign.resize(d);
    SplitMix64 g{seed};
    for (int i = 0; i < d; ++i)
        r->perm[i] = i;
    for (int i = d - 1; i > 0; --i) {
        const int j = (int)g.below((uint64_t)i + 1);
        std::swap(r->perm[i], r->perm[j]);
    }
    for (int k = 0; k < d; ++k)
        r->sign[k] = (g.next() >> 63) ? -1 : 1;
    if (!permute)
        for (int i = 0; i < d; ++i)
            r->perm[i] = i;
    r->ent16.resize(d);
    for (int i = 0; i < d; ++i)
        r->ent16[i] = (uint16_t)(r->perm[i] | (r->sign[i] < 0 ? 0x8000 : 0));
    // K1 gather-entry images (layout documented in oq_internal.h)
    const std::vector<uint8_t> colour = pair_slot_colours(r->perm, d);
    auto slot_of = [&](int g, int k, int lh) {               // 16-byte slot of a half-chunk
        const int GT = d / 32;
        return (2 * k + lh) * GT + (g & ~7) + colour[(size_t)2 * (g + k * GT) + lh];
    };
    for (int f = 0; f < 2; ++f) {
        r->ent_img[f].assign((size_t)(d / 32) * oq::kK1EntStride, 0u);
        for (int i = 0; i < d; ++i) {
            const uint32_t j = (uint32_t)r->perm[i];
            const int c = (int)(j >> 3), GT = d / 32;
            const uint32_t word = 4u * (uint32_t)slot_of(c % GT, c / GT, (int)(j >> 2) & 1) +
                                  (j & 3u);
            const uint32_t off = (f == 1) ? 4u * j : 4u * word;
            r->ent_img[f][(size_t)(i >> 5) * oq::kK1EntStride + (i & 31)] =
                off | (r->sign[i] < 0 ? 0x80000000u : 0u);
        }
        if (f == 0) {
            // words 32..35 of row g: the 16-byte slots its interleave stores go to, as 16-bit
            // indices (k, lh) -> halfword 2k + lh
            for (int g = 0; g < d / 32; ++g)
                for (int k = 0; k < 4; ++k)
                    for (int lh = 0; lh < 2; ++lh) {
                        const uint32_t slot = (uint32_t)slot_of(g, k, lh);
                        const int hw = 2 * k + lh;
                        r->ent_img[0][(size_t)g * oq::kK1EntStride + 32 + hw / 2] |=
                            slot << (16 * (hw & 1));
                    }
        }
    }
    *out = r;
    return OQ_OK;
}

}  // namespace

int oq_build_rpbh(int d, int h, uint64_t seed, oq_rpbh **out) {
    return build_rotation(d, h, seed, true, out, "oq_build_rpbh");
}

int oq_build_block_rht(int d, int h, uint64_t seed, oq_rpbh **out) {
    return build_rotation(d, h, seed, false, out, "oq_build_block_rht");
}

int oq_rpbh_tables(const oq_rpbh *r, int32_t *perm_out, int8_t *sign_out) {
    if (!r)
        return fail(OQ_EINVAL, "oq_rpbh_tables: null handle");
    if (perm_out)
        std::memcpy(perm_out, r->perm.data(), sizeof(int32_t) * r->d);
    if (sign_out)
        std::memcpy(sign_out, r->sign.data(), r->d);
    return OQ_OK;
}

int oq_lloyd_max_marginal(int d, int bits, int marginal, oq_codebook **out) {
    const char *who = "oq_lloyd_max";
    if (!out)
        return fail(OQ_EINVAL, "%s: out is NULL", who);
    *out = nullptr;
    if (marginal != OQ_MARGINAL_GAUSSIAN && marginal != OQ_MARGINAL_EXACT)
        return fail(OQ_EINVAL, "%s: marginal = %d (OQ_MARGINAL_GAUSSIAN or OQ_MARGINAL_EXACT)",
                    who, marginal);
    if (d < 1 || (marginal == OQ_MARGINAL_EXACT && d < 3))
        return fail(OQ_EINVAL, "%s: d = %d (the exact marginal needs d >= 3)", who, d);
    if (bits != 2 && bits != 3 && bits != 4 && bits != 6 && bits != 8)
        return fail(OQ_EINVAL, "%s: bits = %d not in {2, 3, 4, 6, 8}", who, bits);
    oq_codebook *cb = new (std::nothrow) oq_codebook;
    if (!cb)
        return fail(OQ_ENOMEM, "%s: out of host memory", who);
    cb->d = d;
    cb->bits = bits;
    cb->marginal = marginal;
    const int L = 1 << bits;
    bool ok;
    if (marginal == OQ_MARGINAL_GAUSSIAN) {
        ok = solve_lloyd_max(GaussMarginal{}, L, cb->c);
    } else {
        static const GaussLegendre rule;
        ok = solve_lloyd_max(SphereMarginal(d, &rule), L, cb->c);
    }
    if (!ok) {
        delete cb;
        return fail(OQ_EINVAL, "%s: solver did not converge for %d levels", who, L);
    }
    cb->t.resize(L - 1);
    for (int j = 0; j < L - 1; ++j)
        cb->t[j] = 0.5 * (cb->c[j] + cb->c[j + 1]);
    for (int i = 0; i < L; ++i)
        cb->lut[i] = to_half_bits(cb->c[i]);
    if (!build_grid(cb)) {
        delete cb;
        return fail(OQ_EINVAL, "%s: could not build the quantizer grid", who);
    }
    // K1 fp16-output image: entry e (a byte of packed codes) = the fp16 centroids of the
    // 8/bits codes in it, lowest code first (bits 2: four, 4: two, 8: one per entry)
    if (bits == 2 || bits == 4 || bits == 8) {
        const int per = 8 / bits;
        std::vector<uint16_t> tab((size_t)256 * per);
        for (int e = 0; e < 256; ++e)
            for (int i = 0; i < per; ++i)
                tab[(size_t)e * per + i] = cb->lut[(e >> (i * bits)) & (L - 1)];
        cb->dec_img.assign((tab.size() / 2 + 3) / 4 * 4, 0u);
        std::memcpy(cb->dec_img.data(), tab.data(), tab.size() * 2);
    }
    // K1 table image: one copy per lane when bits <= 4 (conflict-free lookups), padded to 16 B
    const int copies = bits <= 4 ? 32 : 1;
    cb->tbl_img.assign((((size_t)(cb->G + 1) * copies + 3) / 4) * 4, 0u);
    for (int k = 0; k <= cb->G; ++k)
        for (int l = 0; l < copies; ++l)
            cb->tbl_img[(size_t)k * copies + l] = cb->grid[k];
    *out = cb;
    return OQ_OK;
}

int oq_lloyd_max(int d, int bits, oq_codebook **out) {
    return oq_lloyd_max_marginal(d, bits, OQ_MARGINAL_GAUSSIAN, out);
}

int oq_codebook_values(const oq_codebook *cb, double *centroids, double *bounds) {
    if (!cb)
        return fail(OQ_EINVAL, "oq_codebook_values: null handle");
    const double sigma = 1.0 / std::sqrt((double)cb->d);
    const int L = 1 << cb->bits;
    if (centroids)
        for (int i = 0; i < L; ++i)
            centroids[i] = sigma * cb->c[i];
    if (bounds)
        for (int j = 0; j < L - 1; ++j)
            bounds[j] = sigma * cb->t[j];
    return OQ_OK;
}

int oq_codebook_grid(const oq_codebook *cb, int *grid_cells, double *delta, uint32_t *table) {
    if (!cb)
        return fail(OQ_EINVAL, "oq_codebook_grid: null handle");
    if (grid_cells)
        *grid_cells = cb->G;
    if (delta)
        *delta = cb->delta;
    if (table)
        std::memcpy(table, cb->grid.data(), sizeof(uint32_t) * cb->grid.size());
    return OQ_OK;
}

int oq_quantize_weight(const oq_rpbh *r, const oq_codebook *cw, const void *W, int dtype,
                       int out_features, int d, uint8_t *W_codes, float *row_norms,
                       void *stream) {
    return quantize_rows(r, cw, W, dtype, out_features, d, W_codes, row_norms, stream, 0.0f,
                         "oq_quantize_weight");
}

int oq_quantize_act(const oq_rpbh *r, const oq_codebook *ca, const void *x, int dtype, int T,
                    int d, uint8_t *x_codes, float *s, void *stream) {
    return quantize_rows(r, ca, x, dtype, T, d, x_codes, s, stream, 1e-8f, "oq_quantize_act");
}

int oq_quantize_act_gelu(const oq_rpbh *r, const oq_codebook *ca, const void *x, int dtype,
                         int T, int d, uint8_t *x_codes, float *s, void *stream) {
    return quantize_rows(r, ca, x, dtype, T, d, x_codes, s, stream, 1e-8f,
                         "oq_quantize_act_gelu", true);
}

int oq_linear(const oq_codebook *ca, const oq_codebook *cw, const uint8_t *x_codes,
              const float *s, const uint8_t *W_codes, const float *row_norms, int T, int d,
              int out_features, void *y, int out_dtype, void *stream) {
    const char *who = "oq_linear";
    if (!ca || !cw)
        return fail(OQ_EINVAL, "%s: null codebook", who);
    if (check_dims(d, who) != OQ_OK)
        return OQ_EINVAL;
    if (ca->d != d || cw->d != d)
        return fail(OQ_EINVAL, "%s: d = %d but codebooks have d = %d / %d", who, d, ca->d,
                    cw->d);
    if (out_dtype != OQ_F32 && out_dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: out_dtype must be OQ_F32 or OQ_BF16", who);
    if (T < 0 || out_features < 1 || !out_rows_aligned(out_features, out_dtype))
        return fail(OQ_EINVAL, "%s: T = %d must be >= 0 and out_features = %d positive with "
                               "16-byte rows of y (a multiple of 4 for fp32, 8 for bf16)", who,
                    T, out_features);
    if (T == 0)
        return OQ_OK;
    if (!x_codes || !s || !W_codes || !row_norms || !y)
        return fail(OQ_EINVAL, "%s: null data pointer", who);
    if (!aligned16(x_codes) || !aligned16(W_codes) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(s) & 3u) || (reinterpret_cast<uintptr_t>(row_norms) & 3u))
        return fail(OQ_EINVAL, "%s: codes and y must be 16-byte aligned, s/row_norms 4-byte",
                    who);
    int dev;
    DeviceInfo *di;
    int rc = current_device(&dev, &di);
    if (rc != OQ_OK)
        return rc;
    cudaMemPool_t pool = device_pool(dev, di, &rc);
    if (!pool)
        return rc;
    // Both operands decoded to fp16 by the prepass, then the TMA/tcgen05 GEMM; with
    // OQ_LINEAR_PATH=fused, 4-bit activation codes are decoded inside the GEMM kernel and only
    // the weight codes get the prepass.
    const bool fused = ca->bits == 4 && fused_requested();
    const bool wcodes = !fused && wcodes_applies(cw, T);
    const size_t ws_bytes = fused    ? (size_t)out_features * d * 2
                            : wcodes ? (size_t)T * d * 2
                                     : oq::linear_workspace_bytes(T, d, out_features);
    void *ws = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMallocFromPoolAsync(&ws, ws_bytes, pool, st);
    if (e != cudaSuccess)
        return fail_cuda(e, "oq_linear: workspace allocation");
    std::string why;
    uint16_t *A16 = nullptr, *B16 = static_cast<uint16_t *>(ws);
    if (wcodes)
        B16 = nullptr;
    // both operands' 4-bit codes of odd-symmetric codebooks: one decode launch for the two
    uint32_t src_a[4], src_w[4];
    const bool both = !fused && !wcodes && ca->bits == 4 && cw->bits == 4 &&
                      oq::decode8_sources(ca->lut, &src_a[0], &src_a[1], &src_a[2], &src_a[3]) &&
                      oq::decode8_sources(cw->lut, &src_w[0], &src_w[1], &src_w[2], &src_w[3]);
    if (!fused) {
        A16 = static_cast<uint16_t *>(ws);
        if (!wcodes)
            B16 = reinterpret_cast<uint16_t *>(static_cast<unsigned char *>(ws) +
                                               oq::linear_workspace_b_offset(T, d));
        if (both)
            e = timed(OQ_KERNEL_DECODE, st, [&] {
                cudaError_t err = cudaErrorInvalidValue;
                oq::launch_decode_pair(ca->bits, x_codes, A16, T, ca->lut, cw->bits, W_codes,
                                       B16, out_features, cw->lut, d, st, di->sms, &err, &why);
                return err;
            });
        else
            e = timed(OQ_KERNEL_DECODE, st, [&] {
                return oq::launch_decode(ca->bits, x_codes, A16, T, d, ca->lut, st, di->sms,
                                         &why);
            });
    }
    if (e == cudaSuccess && !wcodes && !both)
        e = timed(OQ_KERNEL_DECODE, st, [&] {
            return oq::launch_decode(cw->bits, W_codes, B16, out_features, d, cw->lut, st,
                                     di->sms, &why);
        });
    if (e == cudaSuccess)
        e = timed(OQ_KERNEL_GEMM, st, [&] {
            return oq::launch_gemm(A16, x_codes, ca->lut, B16, W_codes, cw->lut, s, row_norms,
                                   y, out_dtype == OQ_BF16, T, out_features, d, st, di->sms,
                                   &why, take_armed(OQ_KERNEL_GEMM));
        });
    cudaError_t e2 = cudaFreeAsync(ws, st);
    if (e != cudaSuccess)
        return fail_cuda(e, why.c_str());
    if (e2 != cudaSuccess)
        return fail_cuda(e2, "oq_linear: workspace release");
    return OQ_OK;
}

int oq_linear_noalloc(const oq_codebook *ca, const oq_codebook *cw, const uint8_t *x_codes,
                      const float *s, const uint8_t *W_codes, const float *row_norms, int T,
                      int d, int out_features, void *y, int out_dtype, void *stream) {
    const char *who = "oq_linear_noalloc";
    if (!ca || !cw)
        return fail(OQ_EINVAL, "%s: null codebook", who);
    if (check_dims(d, who) != OQ_OK)
        return OQ_EINVAL;
    if (ca->d != d || cw->d != d)
        return fail(OQ_EINVAL, "%s: d = %d but codebooks have d = %d / %d", who, d, ca->d,
                    cw->d);
    if (out_dtype != OQ_F32 && out_dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: out_dtype must be OQ_F32 or OQ_BF16", who);
    if (T < 0 || out_features < 1 || !out_rows_aligned(out_features, out_dtype))
        return fail(OQ_EINVAL, "%s: T = %d must be >= 0 and out_features = %d positive with "
                               "16-byte rows of y (a multiple of 4 for fp32, 8 for bf16)", who,
                    T, out_features);
    const size_t need = oq::linear_workspace_bytes(T, d, out_features);
    const size_t have = oq::noalloc_workspace_bytes();
    if (need > have)
        return fail(OQ_EINVAL, "%s: T = %d, d = %d, out_features = %d need %zu bytes of "
                               "workspace, more than the fixed %zu bytes "
                               "(OQ_NOALLOC_WORKSPACE_BYTES); use oq_linear or split T", who,
                    T, d, out_features, need, have);
    if (T == 0)
        return OQ_OK;
    if (!x_codes || !s || !W_codes || !row_norms || !y)
        return fail(OQ_EINVAL, "%s: null data pointer", who);
    if (!aligned16(x_codes) || !aligned16(W_codes) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(s) & 3u) || (reinterpret_cast<uintptr_t>(row_norms) & 3u))
        return fail(OQ_EINVAL, "%s: codes and y must be 16-byte aligned, s/row_norms 4-byte",
                    who);
    int dev;
    DeviceInfo *di;
    int rc = current_device(&dev, &di);
    if (rc != OQ_OK)
        return rc;
    void *ws = nullptr;
    cudaError_t e = oq::noalloc_workspace(&ws);
    if (e != cudaSuccess)
        return fail_cuda(e, "oq_linear_noalloc: workspace address lookup");
    cudaStream_t st = (cudaStream_t)stream;
    uint16_t *A16 = static_cast<uint16_t *>(ws);
    uint16_t *B16 = reinterpret_cast<uint16_t *>(static_cast<unsigned char *>(ws) +
                                                 oq::linear_workspace_b_offset(T, d));
    std::string why;
    uint32_t src_a[4], src_w[4];
    const bool both = ca->bits == 4 && cw->bits == 4 &&
                      oq::decode8_sources(ca->lut, &src_a[0], &src_a[1], &src_a[2], &src_a[3]) &&
                      oq::decode8_sources(cw->lut, &src_w[0], &src_w[1], &src_w[2], &src_w[3]);
    if (both) {
        e = timed(OQ_KERNEL_DECODE, st, [&] {
            cudaError_t err = cudaErrorInvalidValue;
            oq::launch_decode_pair(ca->bits, x_codes, A16, T, ca->lut, cw->bits, W_codes, B16,
                                   out_features, cw->lut, d, st, di->sms, &err, &why);
            return err;
        });
    } else {
        e = timed(OQ_KERNEL_DECODE, st, [&] {
            return oq::launch_decode(ca->bits, x_codes, A16, T, d, ca->lut, st, di->sms, &why);
        });
        if (e == cudaSuccess)
            e = timed(OQ_KERNEL_DECODE, st, [&] {
                return oq::launch_decode(cw->bits, W_codes, B16, out_features, d, cw->lut, st,
                                         di->sms, &why);
            });
    }
    if (e == cudaSuccess)
        e = timed(OQ_KERNEL_GEMM, st, [&] {
            return oq::launch_gemm(A16, nullptr, nullptr, B16, nullptr, nullptr, s, row_norms,
                                   y, out_dtype == OQ_BF16, T, out_features, d, st, di->sms,
                                   &why, take_armed(OQ_KERNEL_GEMM),
                                   static_cast<unsigned char *>(ws) + have,
                                   oq::noalloc_split_bytes());
        });
    if (e != cudaSuccess)
        return fail_cuda(e, why.c_str());
    return OQ_OK;
}

int oq_quantized_linear(const oq_rpbh *r, const oq_codebook *ca, const oq_codebook *cw,
                        const void *x, int dtype, const uint8_t *W_codes, const float *row_norms,
                        int T, int d, int out_features, void *y, int out_dtype, float *s,
                        int flags, void *stream) {
    const char *who = "oq_quantized_linear";
    if (!r || !ca || !cw)
        return fail(OQ_EINVAL, "%s: null handle", who);
    if (check_dims(d, who) != OQ_OK)
        return OQ_EINVAL;
    if (r->d != d || ca->d != d || cw->d != d)
        return fail(OQ_EINVAL, "%s: d = %d but rotation/codebooks have d = %d / %d / %d", who,
                    d, r->d, ca->d, cw->d);
    if (dtype != OQ_F32 && dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: dtype must be OQ_F32 or OQ_BF16", who);
    if (out_dtype != OQ_F32 && out_dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: out_dtype must be OQ_F32 or OQ_BF16", who);
    if (flags & ~OQ_FORWARD_GELU)
        return fail(OQ_EINVAL, "%s: unknown flags 0x%x", who, flags);
    const bool gelu = (flags & OQ_FORWARD_GELU) != 0;
    if (gelu && dtype != OQ_BF16)
        return fail(OQ_EINVAL, "%s: OQ_FORWARD_GELU takes bf16 input", who);
    if (T < 0 || out_features < 1 || !out_rows_aligned(out_features, out_dtype))
        return fail(OQ_EINVAL, "%s: T = %d must be >= 0 and out_features = %d positive with "
                               "16-byte rows of y (a multiple of 4 for fp32, 8 for bf16)", who,
                    T, out_features);
    if (T == 0)
        return OQ_OK;
    if (!x || !W_codes || !row_norms || !y)
        return fail(OQ_EINVAL, "%s: null data pointer", who);
    if (!aligned16(x) || !aligned16(W_codes) || !aligned16(y) ||
        (reinterpret_cast<uintptr_t>(row_norms) & 3u) || (reinterpret_cast<uintptr_t>(s) & 3u))
        return fail(OQ_EINVAL, "%s: x, W_codes and y must be 16-byte aligned, row_norms and s "
                               "4-byte", who);
    int dev;
    DeviceInfo *di;
    int rc = current_device(&dev, &di);
    if (rc != OQ_OK)
        return rc;
    cudaMemPool_t pool = device_pool(dev, di, &rc);
    if (!pool)
        return rc;
    cudaStream_t side = device_side(di, &rc);
    if (!side)
        return rc;
    // The whole step as one persistent kernel where it applies (OQ_FUSED_STEP=1)
    // (not where the GEMM would split its K loop: few tiles leave the persistent kernel
    // nothing to overlap, and the split form's summation order is the one to match)
    if (fused_step_requested() && !gelu && !tc_k1_requested() &&
        oq::fused_step_supported(d, r->h, ca->bits, dtype == OQ_BF16) &&
        !oq::gemm_splits_k(T, out_features, d, out_dtype == OQ_BF16))
        return fused_step(r, ca, cw, x, W_codes, row_norms, T, d, out_features, y, out_dtype, s,
                          (cudaStream_t)stream, dev, di, pool, who);
    // The activation operand takes one of three forms:
    //   direct: K1 writes each code's fp16 centroid straight into the GEMM's A operand (bf16 x,
    //           2/4/8-bit codes, 32 <= h <= 256);
    //   codes:  K1 writes the packed 4-bit codes and the GEMM decodes them into its shared-
    //           memory A tiles (OQ_LINEAR_PATH=fused; bf16 x, odd-symmetric 4-bit codebook);
    //   else:   K1 writes codes and the decode prepass expands them into the fp16 A operand.
    // The weight operand: decoded into B16 (in K1's tail or on the side stream), or, with
    // OQ_LINEAR_PATH=wcodes, decoded from its codes inside the GEMM.
    // workspace: A16 [T, d] fp16 (direct / prepass) | B16 [N, d] fp16 (not wcodes) | s [T] (if
    // not given) | codes [T, d*ba/8] (codes / prepass)
    uint32_t src_probe[4];
    const bool acodes = fused_requested() && ca->bits == 4 && dtype == OQ_BF16 &&
                        oq::decode8_sources(ca->lut, &src_probe[0], &src_probe[1],
                                            &src_probe[2], &src_probe[3]);
    const bool direct = !acodes && oq::k1_a16_supported(ca->bits, r->h, dtype == OQ_BF16);
    const bool wcodes = !acodes && wcodes_applies(cw, T);
    const size_t a_bytes = acodes ? 0 : align_up((size_t)T * d * 2, 1024);
    const size_t b_bytes = wcodes ? 0 : align_up((size_t)out_features * d * 2, 1024);
    const size_t s_bytes = s ? 0 : align_up((size_t)T * 4, 1024);
    const size_t c_bytes = direct ? 0 : align_up((size_t)T * d * ca->bits / 8, 1024);
    void *ws = nullptr;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaMallocFromPoolAsync(&ws, a_bytes + b_bytes + s_bytes + c_bytes, pool, st);
    if (e != cudaSuccess)
        return fail_cuda(e, "oq_quantized_linear: workspace allocation");
    unsigned char *w8 = static_cast<unsigned char *>(ws);
    uint16_t *A16 = acodes ? nullptr : reinterpret_cast<uint16_t *>(w8);
    uint16_t *B16 = wcodes ? nullptr : reinterpret_cast<uint16_t *>(w8 + a_bytes);
    float *sv = s ? s : reinterpret_cast<float *>(w8 + a_bytes + b_bytes);
    uint8_t *codes = direct ? nullptr : w8 + a_bytes + b_bytes + s_bytes;
    std::string why;
    // 2-bit weights, or 4-bit weights of an odd-symmetric codebook, with the one-CTA-per-SM
    // K1 (direct or codes form): the K1 groups that run out of token pairs decode the weights
    // (no second kernel, no side stream).  Only while the decode is no bigger than K1's own
    // work (N <= T) and K1 holds at least four groups per SM (d <= 5120): a larger weight
    // matrix, or one decoded by a single group per SM, decodes faster beside K1 than in its
    // tail.
    const bool fuse =
        !wcodes && (direct || acodes) && out_features <= T && d <= 5120 && !tc_k1_requested() &&
        oq::k1_named(d, dtype == OQ_BF16) &&
        (cw->bits == 2 || (cw->bits == 4 && oq::decode8_sources(cw->lut, &src_probe[0],
                                                                 &src_probe[1], &src_probe[2],
                                                                 &src_probe[3])));
    auto gemm = [&]() {
        return timed(OQ_KERNEL_GEMM, st, [&] {
            return oq::launch_gemm(A16, codes, ca->lut, B16, W_codes, cw->lut, sv, row_norms,
                                   y, out_dtype == OQ_BF16, T, out_features, d, st, di->sms,
                                   &why, take_armed(OQ_KERNEL_GEMM));
        });
    };
    if (fuse) {
        FusedDecode fd;
        fd.cb = cw;
        fd.codes = W_codes;
        fd.out = B16;
        fd.rows = out_features;
        rc = quantize_rows(r, ca, x, dtype, T, d, codes, sv, st, 1e-8f, who, gelu, A16, &fd);
        if (rc == OQ_OK) {
            e = gemm();
            if (e != cudaSuccess)
                rc = fail_cuda(e, why.c_str());
        }
        cudaError_t e2 = cudaFreeAsync(ws, st);
        if (rc != OQ_OK)
            return rc;
        if (e2 != cudaSuccess)
            return fail_cuda(e2, "oq_quantized_linear: workspace release");
        return OQ_OK;
    }
    if (!wcodes) {
        // the weight decode needs nothing from x: it runs on the side stream beside K1
        std::lock_guard<std::mutex> lk(g_side_mu);
        e = cudaEventRecord(di->fork, st);
        if (e == cudaSuccess)
            e = cudaStreamWaitEvent(side, di->fork, 0);
        if (e == cudaSuccess)
            e = timed(OQ_KERNEL_DECODE, side, [&] {
                return oq::launch_decode(cw->bits, W_codes, B16, out_features, d, cw->lut, side,
                                         di->sms, &why);
            });
        if (e == cudaSuccess)
            e = cudaEventRecord(di->join, side);
    }
    if (e != cudaSuccess) {
        cudaFreeAsync(ws, st);
        return fail_cuda(e, why.empty() ? "oq_quantized_linear: side stream" : why.c_str());
    }
    rc = quantize_rows(r, ca, x, dtype, T, d, codes, sv, st, 1e-8f, who, gelu,
                       direct ? A16 : nullptr);
    if (rc == OQ_OK && !direct && !acodes) {
        e = timed(OQ_KERNEL_DECODE, st, [&] {
            return oq::launch_decode(ca->bits, codes, A16, T, d, ca->lut, st, di->sms, &why);
        });
        if (e != cudaSuccess)
            rc = fail_cuda(e, why.c_str());
    }
    // the GEMM waits for the weight operand (join) whether or not K1 succeeded, so the
    // workspace is released after every use of it
    e = wcodes ? cudaSuccess : cudaStreamWaitEvent(st, di->join, 0);
    if (rc == OQ_OK && e == cudaSuccess) {
        e = gemm();
        if (e != cudaSuccess)
            rc = fail_cuda(e, why.c_str());
    } else if (rc == OQ_OK) {
        rc = fail_cuda(e, "oq_quantized_linear: join");
    }
    cudaError_t e2 = cudaFreeAsync(ws, st);
    if (rc != OQ_OK)
        return rc;
    if (e2 != cudaSuccess)
        return fail_cuda(e2, "oq_quantized_linear: workspace release");
    return OQ_OK;
}

int oq_check(void *stream) {
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess)
        return fail_cuda(e, "oq_check: stream synchronize");
    unsigned w1 = 0, w2 = 0, w3 = 0, w4 = 0;
    if ((e = oq::read_and_clear_k1_error(&w1, st)) != cudaSuccess)
        return fail_cuda(e, "oq_check: read k1 error word");
    if ((e = oq::read_and_clear_k3_error(&w4, st)) != cudaSuccess)
        return fail_cuda(e, "oq_check: read fused-step error word");
    if ((e = oq::read_and_clear_k1tc_error(&w3, st)) != cudaSuccess)
        return fail_cuda(e, "oq_check: read k1 (tensor-core) error word");
    if ((e = oq::read_and_clear_k2_error(&w2, st)) != cudaSuccess)
        return fail_cuda(e, "oq_check: read k2 error word");
    if (w1 || w2 || w3 || w4)
        return fail(OQ_EDEVICE, "device error word: quantize=0x%x quantize_tc=0x%x linear=0x%x "
                                "fused=0x%x (a bounded wait gave up; quantize bits 1/2 = row "
                                "copy/armed test wait; quantize_tc bits 1/2/4/8/16 = "
                                "staging/operand ring/accumulator/norm/code tile; linear bits "
                                "1/2/4/8 = operand stage/ring slot/accumulator/armed test wait; "
                                "fused bits 1/2/4/8/16 = GEMM stage/quantized rows/tile id/row "
                                "copy/armed test wait)",
                    w1, w3, w2, w4);
    return OQ_OK;
}

void oq_free_rpbh(oq_rpbh *r) {
    if (!r)
        return;
    int cur = -1;
    cudaGetDevice(&cur);
    for (int dev = 0; dev < oq::kMaxDevices; ++dev) {
        for (int f = 0; f < 2; ++f)
            if (r->dev_ent[f][dev]) {
                cudaSetDevice(dev);
                cudaFree(r->dev_ent[f][dev]);
            }
        if (r->dev_ent16[dev]) {
            cudaSetDevice(dev);
            cudaFree(r->dev_ent16[dev]);
        }
    }
    if (cur >= 0)
        cudaSetDevice(cur);
    delete r;
}

void oq_free_codebook(oq_codebook *cb) {
    if (!cb)
        return;
    int cur = -1;
    cudaGetDevice(&cur);
    for (int dev = 0; dev < oq::kMaxDevices; ++dev) {
        if (cb->dev_tbl[dev]) {
            cudaSetDevice(dev);
            cudaFree(cb->dev_tbl[dev]);
        }
        if (cb->dev_dec[dev]) {
            cudaSetDevice(dev);
            cudaFree(cb->dev_dec[dev]);
        }
    }
    if (cur >= 0)
        cudaSetDevice(cur);
    delete cb;
}

int oq_debug_arm_wait_timeout(int kernel, long long limit_cycles) {
    if (kernel == 0) {
        g_armed_kernel = 0;
        return OQ_OK;
    }
    if (kernel != OQ_KERNEL_QUANTIZE && kernel != OQ_KERNEL_GEMM)
        return fail(OQ_EINVAL, "oq_debug_arm_wait_timeout: kernel = %d (OQ_KERNEL_QUANTIZE or "
                               "OQ_KERNEL_GEMM, or 0 to disarm)", kernel);
    if (limit_cycles < 1000 || limit_cycles > 1000000000LL)
        return fail(OQ_EINVAL, "oq_debug_arm_wait_timeout: limit_cycles = %lld not in "
                               "[1e3, 1e9]", limit_cycles);
    g_armed_kernel = kernel;
    g_armed_cycles = limit_cycles;
    return OQ_OK;
}

int oq_timing_enable(int on) {
    g_timing = on != 0;
    return OQ_OK;
}

int oq_timing_collect(oq_timing_record *out, int capacity, int *count) {
    if (count)
        *count = 0;
    if (capacity < 0 || (capacity > 0 && !out))
        return fail(OQ_EINVAL, "oq_timing_collect: bad output buffer");
    int n = 0;
    cudaError_t err = cudaSuccess;
    for (const TimedLaunch &t : g_timed) {
        float ms = 0.f;
        cudaError_t e = cudaEventSynchronize(t.stop);
        if (e == cudaSuccess)
            e = cudaEventElapsedTime(&ms, t.start, t.stop);
        if (e != cudaSuccess && err == cudaSuccess)
            err = e;
        if (n < capacity) {
            out[n].kernel = t.kernel;
            out[n].ms = ms;
        }
        ++n;
        g_event_pool.push_back(t.start);
        g_event_pool.push_back(t.stop);
    }
    g_timed.clear();
    if (count)
        *count = n < capacity ? n : capacity;
    if (err != cudaSuccess)
        return fail_cuda(err, "oq_timing_collect");
    return OQ_OK;
}

const char *oq_last_error(void) { return g_last_error.c_str(); }

const char *oq_version(void) { return "liboq 0.1.0 (sm_100a)"; }

}  // extern "C"
