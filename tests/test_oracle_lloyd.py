"""Pins for the oracle's Lloyd-Max codebook for the Gaussian marginal.

Source: rcap.io summary, change-of-basis paragraph: one "standard Lloyd-Max quantizer"
built offline against the fixed marginal, close to N(0, 1/d) for d > 64.  Pinned against
the textbook optima (Max 1960), closed forms at 1 bit, the two Lloyd conditions evaluated by
numerical quadrature (scipy, independent of the oracle's erfc closed forms), and the
Panter-Dite high-resolution distortion at 8 bits.
"""
import math

import numpy as np
import pytest
from scipy import integrate, stats

import oracle as O
from conftest import golden_rows


def _golden():
    out = {}
    for bits, cents, bounds, mse in golden_rows("lloyd_max_gauss_max1960.txt"):
        out[int(bits)] = ([float(v) for v in cents.split()],
                          [float(v) for v in bounds.split()], float(mse))
    return out


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_textbook_gaussian_optima(bits):
    c, t = O.codebook(bits)
    want_c, want_t, want_mse = _golden()[bits]
    L = 1 << bits
    # 4 significant digits in the table
    np.testing.assert_allclose(c[L // 2:], want_c, rtol=6e-4)
    np.testing.assert_allclose(t[L // 2:], want_t, rtol=6e-4)
    assert O.gauss_mse(c, t) == pytest.approx(want_mse, rel=1e-3)


def test_one_bit_closed_form():
    c, t = O.codebook(1)
    assert c[1] == pytest.approx(math.sqrt(2 / math.pi), abs=1e-13)
    assert c[0] == -c[1] and t[0] == 0.0
    assert O.gauss_mse(c, t) == pytest.approx(1 - 2 / math.pi, abs=1e-13)


def _cell(t, i):
    lo = -np.inf if i == 0 else t[i - 1]
    hi = np.inf if i == len(t) else t[i]
    return lo, hi


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_fixed_point_conditions_by_quadrature(bits):
    c, t = O.codebook(bits)
    L = 1 << bits
    # boundaries are exact midpoints
    np.testing.assert_array_equal(t, 0.5 * (c[:-1] + c[1:]))
    cells = range(L) if bits <= 4 else list(range(0, 8)) + list(range(L // 2 - 4, L // 2 + 4)) + \
        list(range(L - 8, L))
    for i in cells:
        lo, hi = _cell(t, i)
        m0 = integrate.quad(stats.norm.pdf, lo, hi, epsabs=0, epsrel=1e-13)[0]
        m1 = integrate.quad(lambda x: x * stats.norm.pdf(x), lo, hi, epsabs=0,
                            epsrel=1e-13)[0]
        assert c[i] == pytest.approx(m1 / m0, abs=1e-9)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_mse_matches_quadrature(bits):
    c, t = O.codebook(bits)
    total = 0.0
    for i in range(len(c)):
        lo, hi = _cell(t, i)
        total += integrate.quad(lambda x: (x - c[i]) ** 2 * stats.norm.pdf(x), lo, hi,
                                epsabs=1e-15, epsrel=1e-12)[0]
    assert O.gauss_mse(c, t) == pytest.approx(total, rel=1e-9)


@pytest.mark.parametrize("bits", [2, 3, 4, 6, 8])
def test_codebook_is_symmetric_and_sorted(bits):
    c, t = O.codebook(bits)
    np.testing.assert_array_equal(c, -c[::-1])
    assert np.all(np.diff(c) > 0) and np.all(np.diff(t) > 0)
    assert t[len(t) // 2] == 0.0


def test_eight_bit_high_resolution_distortion():
    """Panter-Dite: L^2 * MSE -> sqrt(3) pi / 2 for the unit Gaussian (within 1% at L=256)."""
    c, t = O.codebook(8)
    ratio = O.gauss_mse(c, t) * 4 ** 8 / (math.sqrt(3) * math.pi / 2)
    assert 0.985 < ratio < 1.0


def test_high_resolution_ratio_approaches_panter_dite_monotonically():
    """L^2 * MSE / (sqrt(3) pi / 2) rises towards 1 with the bit width (4, 6, 8 bits): the
    6-bit codebook (the W6A6 setting) sits between its neighbours."""
    r = [O.gauss_mse(*O.codebook(b)) * 4 ** b / (math.sqrt(3) * math.pi / 2) for b in (4, 6, 8)]
    assert r[0] < r[1] < r[2] < 1.0
    assert 0.95 < r[1] < 0.99
