"""ctypes wrapper over liboracle.so (fp64 CPU oracle).  Test infrastructure only.

All arrays are numpy; floating inputs are converted to float64 (exact for bf16/fp32 data).
Citations are to the rcap.io summary "OrbitQuant: Data-Agnostic Quantization for Image and
Video" [RCAP]; each wrapped C function carries its own citation in oracle.c.
"""
import ctypes as C
import math

import numpy as np
from scipy import special

from . import build as _build

_lib = None

_u8p = np.ctypeslib.ndpointer(dtype=np.uint8, flags="C_CONTIGUOUS")
_i8p = np.ctypeslib.ndpointer(dtype=np.int8, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")

EPS_ACT = 1e-8   # eps of the per-token quantizer ([RCAP] pseudocode leaves it open)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        L.orc_splitmix64_next.restype = C.c_uint64
        L.orc_splitmix64_next.argtypes = [C.POINTER(C.c_uint64)]
        L.orc_uniform_below.restype = C.c_uint64
        L.orc_uniform_below.argtypes = [C.POINTER(C.c_uint64), C.c_uint64]
        L.orc_build_rpbh.restype = C.c_int
        L.orc_build_rpbh.argtypes = [C.c_int, C.c_uint64, _i32p, _i8p]
        L.orc_build_block_rht.restype = C.c_int
        L.orc_build_block_rht.argtypes = [C.c_int, C.c_uint64, _i32p, _i8p]
        L.orc_hadamard_entry.restype = C.c_int
        L.orc_hadamard_entry.argtypes = [C.c_int, C.c_int]
        L.orc_rotate_row.restype = C.c_int
        L.orc_rotate_row.argtypes = [C.c_int, C.c_int, _i32p, _i8p, _f64p, _f64p]
        L.orc_lloyd_max_gauss.restype = C.c_int
        L.orc_lloyd_max_gauss.argtypes = [C.c_int, C.c_double, C.c_int, _f64p, _f64p,
                                          C.POINTER(C.c_int), C.POINTER(C.c_double)]
        L.orc_gauss_mse.restype = C.c_double
        L.orc_gauss_mse.argtypes = [C.c_int, _f64p, _f64p]
        L.orc_betainc.restype = C.c_double
        L.orc_betainc.argtypes = [C.c_double, C.c_double, C.c_double]
        L.orc_sphere_cdf.restype = C.c_double
        L.orc_sphere_cdf.argtypes = [C.c_int, C.c_double]
        L.orc_sphere_density.restype = C.c_double
        L.orc_sphere_density.argtypes = [C.c_int, C.c_double]
        L.orc_lloyd_max_sphere.restype = C.c_int
        L.orc_lloyd_max_sphere.argtypes = [C.c_int, C.c_int, C.c_double, C.c_int, _f64p,
                                           _f64p, C.POINTER(C.c_int), C.POINTER(C.c_double)]
        L.orc_code_of.restype = C.c_int
        L.orc_code_of.argtypes = [C.c_double, C.c_int, _f64p, C.c_double]
        L.orc_pack.restype = None
        L.orc_pack.argtypes = [C.c_int, C.c_int, _u8p, _u8p]
        L.orc_unpack.restype = None
        L.orc_unpack.argtypes = [C.c_int, C.c_int, _u8p, _u8p]
        L.orc_quantize_rows_detail.restype = C.c_int
        L.orc_quantize_rows_detail.argtypes = [
            C.c_int, C.c_int, C.c_int, _i32p, _i8p, C.c_int, _f64p, C.c_double, _f64p,
            _u8p, _f64p, C.c_void_p, C.c_void_p]
        L.orc_linear.restype = C.c_int
        L.orc_linear.argtypes = [C.c_int, C.c_int, C.c_int, C.c_int, _f64p, C.c_int, _f64p,
                                 _u8p, _f64p, _u8p, _f64p, _f64p]
        _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


# --- random tables --------------------------------------------------------------------

def splitmix64(seed: int, n: int) -> np.ndarray:
    """First n SplitMix64 outputs from state `seed`."""
    st = C.c_uint64(seed)
    return np.array([lib().orc_splitmix64_next(C.byref(st)) for _ in range(n)], dtype=np.uint64)


def uniform_below(seed: int, n: int, count: int) -> np.ndarray:
    st = C.c_uint64(seed)
    return np.array([lib().orc_uniform_below(C.byref(st), n) for _ in range(count)],
                    dtype=np.uint64)


def build_rpbh(d: int, seed: int):
    """[RCAP] pseudocode build_rpbh(d): (perm int32[d], sign int8[d])."""
    perm = np.empty(d, dtype=np.int32)
    sign = np.empty(d, dtype=np.int8)
    rc = lib().orc_build_rpbh(d, seed, perm, sign)
    if rc != 0:
        raise ValueError(f"orc_build_rpbh({d}) failed: {rc}")
    return perm, sign


def build_block_rht(d: int, seed: int):
    """Block-RHT ablation: the RPBH tables of `seed` with the identity permutation."""
    perm = np.empty(d, dtype=np.int32)
    sign = np.empty(d, dtype=np.int8)
    rc = lib().orc_build_block_rht(d, seed, perm, sign)
    if rc != 0:
        raise ValueError(f"orc_build_block_rht({d}) failed: {rc}")
    return perm, sign


def hadamard(h: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order h as integers."""
    L = lib()
    return np.array([[L.orc_hadamard_entry(i, j) for j in range(h)] for i in range(h)],
                    dtype=np.int64)


def rotate(x, h: int, perm, sign) -> np.ndarray:
    """z = R x for each row of x ([RCAP] RPBH paragraph)."""
    x = _f64(np.atleast_2d(x))
    rows, d = x.shape
    z = np.empty_like(x)
    for r in range(rows):
        rc = lib().orc_rotate_row(d, h, perm, sign, x[r], z[r])
        if rc != 0:
            raise ValueError(f"orc_rotate_row failed: {rc}")
    return z


# --- Lloyd-Max --------------------------------------------------------------------------

def lloyd_max(bits: int, tol: float = 4e-14, max_iter: int = 2_000_000):
    """Unit (N(0,1)) Lloyd-Max quantizer: (centroids[L], bounds[L-1], iters, residual)."""
    L = 1 << bits
    c = np.empty(L, dtype=np.float64)
    t = np.empty(L - 1, dtype=np.float64)
    it = C.c_int(0)
    res = C.c_double(0.0)
    lib().orc_lloyd_max_gauss(bits, tol, max_iter, c, t, C.byref(it), C.byref(res))
    return c, t, it.value, res.value


def betainc(a: float, b: float, x: float) -> float:
    """Regularized incomplete beta I_x(a, b) (continued fraction)."""
    return lib().orc_betainc(a, b, x)


def sphere_cdf(d: int, x: float) -> float:
    """CDF of one coordinate of a uniform unit vector in R^d."""
    return lib().orc_sphere_cdf(d, x)


def sphere_density(d: int, x: float) -> float:
    """f_d(x) = (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2) on [-1, 1]."""
    return lib().orc_sphere_density(d, x)


def lloyd_max_sphere(d: int, bits: int, tol: float = 1e-12, max_iter: int = 2_000_000):
    """Lloyd-Max quantizer for the exact marginal f_d, in the coordinate's own units:
    (centroids[L], bounds[L-1], iters, residual); residual in units of 1/sqrt(d)."""
    L = 1 << bits
    c = np.empty(L, dtype=np.float64)
    t = np.empty(L - 1, dtype=np.float64)
    it = C.c_int(0)
    res = C.c_double(0.0)
    lib().orc_lloyd_max_sphere(d, bits, tol, max_iter, c, t, C.byref(it), C.byref(res))
    return c, t, it.value, res.value


_CB_CACHE = {}


def codebook(bits: int, marginal: str = "gauss", d: int = 0):
    """Cached unit codebook (centroids, bounds) for `bits`: the N(0,1) Lloyd-Max quantizer
    (marginal "gauss"), or sqrt(d) times the Lloyd-Max quantizer of the exact marginal f_d
    (marginal "sphere"), so that both compare against sqrt(d) * x_rot / s."""
    key = (bits, marginal, d if marginal == "sphere" else 0)
    if key not in _CB_CACHE:
        if marginal == "gauss":
            c, t, _, res = lloyd_max(bits)
            if not res <= 1e-12:
                raise RuntimeError(f"Lloyd-Max at {bits} bits did not converge: {res}")
        elif marginal == "sphere":
            tol = 1e-12 if bits <= 4 else 1e-10   # plain Lloyd is slow at 256 levels
            c, t, _, res = lloyd_max_sphere(d, bits, tol=tol)
            if not res <= tol:
                raise RuntimeError(f"f_d Lloyd-Max at d={d}, {bits} bits: {res}")
            c, t = c * np.sqrt(d), t * np.sqrt(d)
        else:
            raise ValueError(marginal)
        _CB_CACHE[key] = (c, t)
    return _CB_CACHE[key]


def gauss_mse(centroids, bounds) -> float:
    c = _f64(centroids)
    t = _f64(bounds)
    return lib().orc_gauss_mse(len(c), c, t)


def code_of(v: float, unit_bounds, sigma: float) -> int:
    t = _f64(unit_bounds)
    return lib().orc_code_of(float(v), len(t) + 1, t, float(sigma))


# --- packing ----------------------------------------------------------------------------

def pack(codes, bits: int) -> np.ndarray:
    """LSB-first packing of each row of `codes` (uint8 [..., n]) into n*bits/8 bytes."""
    codes = np.ascontiguousarray(np.atleast_2d(codes), dtype=np.uint8)
    rows, n = codes.shape
    nb = (n * bits + 7) // 8
    out = np.empty((rows, nb), dtype=np.uint8)
    for r in range(rows):
        lib().orc_pack(n, bits, codes[r], out[r])
    return out


def unpack(packed, n: int, bits: int) -> np.ndarray:
    packed = np.ascontiguousarray(np.atleast_2d(packed), dtype=np.uint8)
    rows = packed.shape[0]
    out = np.empty((rows, n), dtype=np.uint8)
    for r in range(rows):
        lib().orc_unpack(n, bits, packed[r], out[r])
    return out


# --- quantizers and the linear layer ------------------------------------------------------

def quantize_rows(x, h: int, perm, sign, bits: int, eps: float, detail: bool = False,
                  marginal: str = "gauss"):
    """[RCAP] pseudocode per-row quantizer.  Returns (packed codes, norms) and, with
    detail=True, also (z, u) where u = (z/(s+eps)) * sqrt(d) in unit-codebook units.
    marginal: the codebook's target, "gauss" (N(0, 1/d)) or "sphere" (exact f_d)."""
    x = _f64(np.atleast_2d(x))
    rows, d = x.shape
    _, t = codebook(bits, marginal, d)
    packed = np.empty((rows, d * bits // 8), dtype=np.uint8)
    norms = np.empty(rows, dtype=np.float64)
    z = np.empty_like(x) if detail else None
    u = np.empty_like(x) if detail else None
    rc = lib().orc_quantize_rows_detail(
        rows, d, h, perm, sign, bits, t, float(eps), x, packed, norms,
        z.ctypes.data if detail else None, u.ctypes.data if detail else None)
    if rc != 0:
        raise ValueError(f"orc_quantize_rows failed: {rc}")
    if detail:
        return packed, norms, z, u
    return packed, norms


def gelu(x) -> np.ndarray:
    """GELU in its exact (erf) form, x Phi(x), in fp64, with the normal CDF written as
    Phi(x) = erfc(-x / sqrt 2) / 2: the same function as (1 + erf(x / sqrt 2)) / 2, evaluated
    without the cancellation of 1 + erf for negative x (which loses the left tail)."""
    x = np.asarray(x, dtype=np.float64)
    return 0.5 * x * special.erfc(-x / math.sqrt(2.0))


def quantize_act(x, h, perm, sign, bits, detail=False, marginal="gauss", gelu_input=False):
    """Online activation step: eps = EPS_ACT.  gelu_input: quantize GELU(x) (the MLP down
    projection's input formed from the up projection's pre-activation)."""
    if gelu_input:
        x = gelu(_f64(np.atleast_2d(x)))
    return quantize_rows(x, h, perm, sign, bits, EPS_ACT, detail, marginal)


def quantize_weight(W, h, perm, sign, bits, detail=False, marginal="gauss"):
    """Offline weight step: no eps; rows of W are the 'tokens'."""
    return quantize_rows(W, h, perm, sign, bits, 0.0, detail, marginal)


def linear(x_packed, s, w_packed, rn, d: int, bits_a: int, bits_w: int,
           marginal: str = "gauss") -> np.ndarray:
    """y[t,o] = s_t rn_o sum_k sigma ca[xc] sigma cw[wc], naive fp64 triple loop."""
    ca, _ = codebook(bits_a, marginal, d)
    cw, _ = codebook(bits_w, marginal, d)
    xp = np.ascontiguousarray(np.atleast_2d(x_packed), dtype=np.uint8)
    wp = np.ascontiguousarray(np.atleast_2d(w_packed), dtype=np.uint8)
    T, out = xp.shape[0], wp.shape[0]
    y = np.empty((T, out), dtype=np.float64)
    rc = lib().orc_linear(T, d, out, bits_a, ca, bits_w, cw, xp, _f64(s), wp, _f64(rn), y)
    if rc != 0:
        raise ValueError(f"orc_linear failed: {rc}")
    return y


def sigma(d: int) -> float:
    return 1.0 / math.sqrt(d)
