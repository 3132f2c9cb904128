"""liboq host logic on the CPU (no GPU calls): the C ABI loads and exports every symbol of
include/oq.h; its RPBH tables and Lloyd-Max codebooks (independent codings) agree with the
oracle; the quantizer grid table, evaluated with the kernel's integer recipe, reproduces the
oracle's boundary count; argument validation rejects bad input before touching a device.
"""
import ctypes as C

import numpy as np
import pytest

import oracle as O
from calibration_free_bit_b200 import build as B
from calibration_free_bit_b200 import oq


@pytest.fixture(scope="module", autouse=True)
def built():
    B.build()


def test_library_exports_every_header_symbol():
    names = oq.header_functions()
    assert {"oq_build_rpbh", "oq_lloyd_max", "oq_quantize_weight", "oq_quantize_act",
            "oq_linear"} <= set(names)
    L = oq.lib()
    missing = []
    for n in names:
        try:
            getattr(L, n)
        except AttributeError:
            missing.append(n)
    assert not missing, missing
    assert oq.version().startswith("liboq")


def test_binding_constants_match_the_header():
    """Every OQ_* constant the Python binding defines has the value of the header's #define
    (status codes, element types, flags, kernel ids), and every kernel id has a name."""
    import os
    import re
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    hdr = open(os.path.join(root, "include", "oq.h")).read()
    defs = {}
    for name, val in re.findall(r"^#define (OQ_[A-Z0-9_]+)\s+\(?(-?\d+)u?\)?", hdr, re.M):
        defs[name] = int(val)
    bound = {k: getattr(oq, k) for k in dir(oq) if k.startswith("OQ_") and
             isinstance(getattr(oq, k), int)}
    assert bound, "no constants in the binding"
    for k, v in bound.items():
        assert k in defs and defs[k] == v, (k, v, defs.get(k))
    kernel_ids = {v for k, v in defs.items() if k.startswith("OQ_KERNEL_")}
    assert kernel_ids == set(oq.KERNEL_NAMES), (kernel_ids, oq.KERNEL_NAMES)


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (3072, 128, 0), (13824, 128, 7),
                                      (16384, 256, 12345), (1024, 32, 2**63 + 5)])
def test_rpbh_tables_bit_exact_vs_oracle(d, h, seed):
    perm, sign = oq.oq_build_rpbh(d, h, seed).tables()
    operm, osign = O.build_rpbh(d, seed)
    assert np.array_equal(perm, operm)
    assert np.array_equal(sign, osign)


@pytest.mark.parametrize("d,h,seed", [(256, 64, 0), (3072, 128, 9)])
def test_block_rht_tables_bit_exact_vs_oracle(d, h, seed):
    perm, sign = oq.oq_build_block_rht(d, h, seed).tables()
    operm, osign = O.build_block_rht(d, seed)
    assert np.array_equal(perm, operm) and np.array_equal(sign, osign)


@pytest.mark.parametrize("bits,tol", [(2, 1e-11), (3, 1e-11), (4, 1e-11), (6, 1e-10),
                                      (8, 1e-8)])
def test_codebook_matches_oracle(bits, tol):
    """Two independent solvers (liboq: Lloyd warm-up + Newton to a residual < 1e-15; oracle:
    plain Lloyd stopped at a step <= 4e-14).  The oracle's distance to the fixed point is
    step / (1 - contraction): ~1e-12 at 4 bits (contraction ~0.96) and ~1e-10 at 8 bits
    (contraction ~1 - 2e-4), hence the tolerances (unit-codebook units)."""
    d = 3072
    c, t = oq.oq_lloyd_max(d, bits).values()
    oc, ot = O.codebook(bits)
    sig = 1.0 / np.sqrt(d)
    np.testing.assert_allclose(c, sig * oc, rtol=0, atol=tol * sig)
    np.testing.assert_allclose(t, sig * ot, rtol=0, atol=tol * sig)


@pytest.mark.parametrize("d,bits,tol", [(128, 2, 1e-10), (128, 4, 1e-10), (256, 3, 1e-10),
                                        (3072, 4, 1e-10), (16384, 4, 1e-8), (128, 8, 1e-8)])
def test_exact_marginal_codebook_matches_oracle(d, bits, tol):
    """f_d codebook (the f3 variant): liboq solves it by Newton with Gauss-Legendre cell
    probabilities, the oracle by plain Lloyd with a continued-fraction incomplete beta.
    Tolerances in unit-codebook units: the oracle's incomplete beta is good to ~1e-11 in
    absolute probability at d = 16384 (b = 8191.5), and its 8-bit Lloyd stops at a step of
    1e-12 with a contraction close to 1."""
    cb = oq.oq_lloyd_max(d, bits, "exact")
    c, t = cb.values()                                   # the f_d quantizer itself
    if bits == 8:
        oc, ot, _, res = O.lloyd_max_sphere(d, bits, tol=1e-12)
        assert res <= 1e-12
    else:
        oc, ot = (v / np.sqrt(d) for v in O.codebook(bits, "sphere", d))
    sd = 1.0 / np.sqrt(d)
    np.testing.assert_allclose(c, oc, rtol=0, atol=tol * sd)
    np.testing.assert_allclose(t, ot, rtol=0, atol=tol * sd)
    assert np.all(np.abs(c) < 1.0) and np.all(np.diff(c) > 0)


def test_quantized_linear_validation_without_a_gpu():
    L = oq.lib()
    r = oq.oq_build_rpbh(3072, 128)
    ca = oq.oq_lloyd_max(3072, 4)
    c_other = oq.oq_lloyd_max(1024, 4)
    fake = 1 << 20
    args = lambda **kw: dict(dict(r=r.handle, ca=ca.handle, cw=ca.handle, x=fake,    # noqa
                                  dtype=oq.OQ_BF16, wc=fake, rn=fake, T=8, d=3072, N=128,
                                  y=fake, od=oq.OQ_F32, s=None, flags=0), **kw)

    def call(a):
        return L.oq_quantized_linear(a["r"], a["ca"], a["cw"], a["x"], a["dtype"], a["wc"],
                                     a["rn"], a["T"], a["d"], a["N"], a["y"], a["od"], a["s"],
                                     a["flags"], None)
    assert call(args(flags=4)) == oq.OQ_EINVAL                        # unknown flag
    assert call(args(flags=1, dtype=oq.OQ_F32)) == oq.OQ_EINVAL       # GELU needs bf16
    assert call(args(cw=c_other.handle)) == oq.OQ_EINVAL              # d mismatch
    assert call(args(N=102)) == oq.OQ_EINVAL                          # fp32 rows not 16 B
    assert call(args(N=100, od=oq.OQ_BF16)) == oq.OQ_EINVAL           # bf16 rows not 16 B
    assert call(args(x=fake + 4)) == oq.OQ_EINVAL                     # misaligned x
    assert call(args(s=fake + 2)) == oq.OQ_EINVAL                     # misaligned s
    assert call(args(T=0, x=None, wc=None, rn=None, y=None)) == oq.OQ_OK


def test_exact_marginal_rejects_small_d():
    h = C.c_void_p()
    assert oq.lib().oq_lloyd_max_marginal(2, 4, 1, C.byref(h)) == oq.OQ_EINVAL
    assert oq.lib().oq_lloyd_max_marginal(128, 4, 7, C.byref(h)) == oq.OQ_EINVAL


def emulate_kernel_codes(u, G, delta, table):
    """The kernel's code recipe in exact integer arithmetic (documented in include/oq.h):
    a = sat(u/(G delta) + 1/2) in fp32; q = floor(a 2^23); word = table[q >> (23-log2 G)];
    code = (word + (0x3F800000 + q) G) mod 2^32 >> 24."""
    a = np.clip((u / (G * delta) + 0.5).astype(np.float32), 0.0, 1.0).astype(np.float64)
    q = np.floor(a * 2.0**23).astype(np.int64)
    F = 23 - int(np.log2(G))
    word = table[q >> F].astype(np.int64)
    D = (word + (0x3F800000 + q) * G) % (1 << 32)
    return (D >> 24).astype(np.int64)


@pytest.mark.parametrize("bits,marginal", [(2, "gauss"), (3, "gauss"), (4, "gauss"),
                                           (6, "gauss"), (8, "gauss"), (4, "exact"),
                                           (8, "exact")])
def test_quantizer_grid_matches_boundary_count(bits, marginal):
    d = 3072 if marginal == "gauss" else 128
    cb = oq.oq_lloyd_max(d, bits, marginal)
    G, delta, table = cb.grid()
    assert G & (G - 1) == 0 and len(table) == G + 1
    t = cb.values()[1] * np.sqrt(d)                     # unit boundaries the grid encodes
    rng = np.random.default_rng(bits)
    u = np.concatenate([rng.standard_normal(400000) * 1.3,
                        rng.uniform(-60, 60, 20000),
                        t, t + 1e-7, t - 1e-7, t + 3e-6, t - 3e-6,
                        [0.0, -0.0, 1e30, -1e30, 55.4, -55.4]])
    got = emulate_kernel_codes(u, G, delta, table)
    want = np.searchsorted(t, u, side="right")
    bad = np.flatnonzero(got != want)
    # the fixed-point grid moves a boundary by < 2^-23 of the grid span (< 1.2e-6 sigma)
    for i in bad:
        j = np.argmin(np.abs(t - u[i]))
        assert abs(u[i] - t[j]) < 2e-6, (u[i], got[i], want[i])
        assert {got[i], want[i]} == {j, j + 1}
    assert len(bad) <= 8 * len(t)


def test_validation_rejects_bad_arguments_without_a_gpu():
    L = oq.lib()
    h = C.c_void_p()
    assert L.oq_build_rpbh(100, 64, 0, C.byref(h)) == oq.OQ_EINVAL
    assert L.oq_build_rpbh(3072, 48, 0, C.byref(h)) == oq.OQ_EINVAL
    assert L.oq_build_rpbh(3072, 2048, 0, C.byref(h)) == oq.OQ_EINVAL
    assert L.oq_build_rpbh(32768, 128, 0, C.byref(h)) == oq.OQ_EINVAL
    assert L.oq_lloyd_max(3072, 5, C.byref(h)) == oq.OQ_EINVAL
    assert b"bits" in L.oq_last_error()
    r = oq.oq_build_rpbh(3072, 128)
    ca = oq.oq_lloyd_max(3072, 4)
    c_other = oq.oq_lloyd_max(1024, 4)
    fake = 1 << 20        # never dereferenced: validation fails first
    # d mismatch between rotation and codebook
    assert L.oq_quantize_act(r.handle, c_other.handle, fake, oq.OQ_BF16, 8, 3072, fake, fake,
                             None) == oq.OQ_EINVAL
    # bad dtype, negative T, null pointers, misalignment
    assert L.oq_quantize_act(r.handle, ca.handle, fake, 7, 8, 3072, fake, fake,
                             None) == oq.OQ_EINVAL
    assert L.oq_quantize_act(r.handle, ca.handle, fake, oq.OQ_BF16, -1, 3072, fake, fake,
                             None) == oq.OQ_EINVAL
    assert L.oq_quantize_act(r.handle, ca.handle, None, oq.OQ_BF16, 8, 3072, fake, fake,
                             None) == oq.OQ_EINVAL
    assert L.oq_quantize_act(r.handle, ca.handle, fake + 2, oq.OQ_BF16, 8, 3072, fake, fake,
                             None) == oq.OQ_EINVAL
    # T = 0 is a no-op that succeeds without touching a device
    assert L.oq_quantize_act(r.handle, ca.handle, None, oq.OQ_BF16, 0, 3072, None, None,
                             None) == oq.OQ_OK
    # linear: rows of y not a multiple of 16 bytes, unknown output type, d mismatch
    assert L.oq_linear(ca.handle, ca.handle, fake, fake, fake, fake, 8, 3072, 102, fake,
                       oq.OQ_F32, None) == oq.OQ_EINVAL
    assert L.oq_linear(ca.handle, ca.handle, fake, fake, fake, fake, 8, 3072, 128, fake,
                       2, None) == oq.OQ_EINVAL
    assert b"out_dtype" in L.oq_last_error()
    assert L.oq_linear(ca.handle, ca.handle, None, None, None, None, 0, 3072, 128, None,
                       oq.OQ_BF16, None) == oq.OQ_OK
    assert L.oq_linear(ca.handle, c_other.handle, fake, fake, fake, fake, 8, 3072, 128, fake,
                       oq.OQ_F32, None) == oq.OQ_EINVAL
    assert L.oq_linear(ca.handle, ca.handle, None, None, None, None, 0, 3072, 128, None,
                       oq.OQ_F32, None) == oq.OQ_OK


@pytest.mark.parametrize("d,h,ok", [
    (3072, 2, True), (3072, 4, True), (3072, 8, True), (3072, 16, True), (3072, 1024, True),
    (128, 128, True), (16384, 1024, True),
    (3072, 1, False),      # h below 2
    (3072, 2048, False),   # h above 1024
    (3072, 48, False),     # h not a power of two
    (3072, 12, False),
    (2048, 4096, False),   # h larger than d
    (1536, 1024, False),   # h does not divide d
    (100, 4, False),       # d not a multiple of 128 (3-bit code rows would not be 16-byte)
    (3008, 64, False),
    (64, 64, False),       # d below 128
    (16512, 128, False),   # d above 16384 (a bf16 token pair no longer fits shared memory)
])
def test_size_limits_of_the_rotation(d, h, ok):
    """Each size limit of oq_build_rpbh / oq_build_block_rht, accepted or refused with
    OQ_EINVAL before anything touches a device."""
    L = oq.lib()
    for build in (L.oq_build_rpbh, L.oq_build_block_rht):
        hd = C.c_void_p()
        rc = build(d, h, 0, C.byref(hd))
        assert rc == (oq.OQ_OK if ok else oq.OQ_EINVAL), (d, h, L.oq_last_error())
        if ok:
            L.oq_free_rpbh(hd)


@pytest.mark.parametrize("N,out_dtype,ok", [
    (4, oq.OQ_F32, True), (20, oq.OQ_F32, True), (3072, oq.OQ_F32, True),
    (8, oq.OQ_BF16, True), (24, oq.OQ_BF16, True),
    (2, oq.OQ_F32, False), (102, oq.OQ_F32, False),      # fp32 rows of y not 16-byte
    (4, oq.OQ_BF16, False), (20, oq.OQ_BF16, False),     # bf16 rows of y not 16-byte
    (0, oq.OQ_F32, False), (-16, oq.OQ_F32, False),
])
def test_output_row_rule_of_the_linear_calls(N, out_dtype, ok):
    """out_features must give 16-byte rows of y (the TMA store's row-stride rule), checked by
    oq_linear, oq_linear_noalloc and oq_quantized_linear alike.  Calls with T = 0 stop after
    validation, so no device is needed."""
    L = oq.lib()
    r = oq.oq_build_rpbh(1024, 128)
    ca = oq.oq_lloyd_max(1024, 4)
    want = oq.OQ_OK if ok else oq.OQ_EINVAL
    assert L.oq_linear(ca.handle, ca.handle, None, None, None, None, 0, 1024, N, None,
                       out_dtype, None) == want
    assert L.oq_linear_noalloc(ca.handle, ca.handle, None, None, None, None, 0, 1024, N, None,
                               out_dtype, None) == want
    assert L.oq_quantized_linear(r.handle, ca.handle, ca.handle, None, oq.OQ_BF16, None, None,
                                 0, 1024, N, None, out_dtype, None, 0, None) == want
