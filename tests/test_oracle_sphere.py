"""Pins of the oracle's exact-marginal codebook (the f3 variant): Lloyd-Max for
f_d(x) = (1 - x^2)^((d-3)/2) / B(1/2, (d-1)/2), the law of one coordinate of a uniformly
random unit vector in R^d (rcap.io OrbitQuant summary, change-of-basis paragraph: the fixed
marginal that depends only on d, close to N(0, 1/d) above d = 64).

Pinned against: a library incomplete beta (scipy), quadrature of the density, closed forms
(d = 3 is the uniform law, whose Lloyd-Max quantizer is the uniform quantizer; at one bit the
centroid is E|X| = Gamma(d/2) / (sqrt(pi) Gamma((d+1)/2))), the Lloyd conditions checked by
independent quadrature, and the Gaussian limit for large d."""
import math

import numpy as np
import pytest
from scipy import integrate, special

import oracle as O


@pytest.mark.parametrize("a,b", [(0.5, 1.0), (0.5, 63.5), (0.5, 1535.5), (1535.5, 0.5),
                                 (2.0, 3.0), (0.5, 8191.5)])
def test_betainc_matches_library(a, b):
    for x in [1e-9, 1e-6, 1e-3, 0.01, 0.1, 0.3, 0.5, 0.9, 0.999, 1 - 1e-9]:
        assert abs(O.betainc(a, b, x) - special.betainc(a, b, x)) <= 1e-11, (a, b, x)


@pytest.mark.parametrize("d", [3, 4, 7, 64, 128, 3072])
def test_sphere_cdf_and_density_agree(d):
    assert O.sphere_cdf(d, 0.0) == pytest.approx(0.5, abs=1e-15)
    assert O.sphere_cdf(d, 1.0) == 1.0 and O.sphere_cdf(d, -1.0) == 0.0
    sd = 1 / math.sqrt(d)
    for x in [0.3 * sd, sd, 2.5 * sd, min(0.9, 6 * sd)]:
        area, _ = integrate.quad(lambda v: O.sphere_density(d, v), 0.0, x, epsabs=1e-14,
                                 epsrel=1e-13, limit=200)
        assert O.sphere_cdf(d, x) - 0.5 == pytest.approx(area, abs=1e-12)
        assert O.sphere_cdf(d, -x) == pytest.approx(1.0 - O.sphere_cdf(d, x), abs=1e-15)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_d3_is_the_uniform_quantizer(bits):
    c, t, _, res = O.lloyd_max_sphere(3, bits)
    L = 1 << bits
    assert res <= 1e-12
    np.testing.assert_allclose(c, -1 + (2 * np.arange(L) + 1) / L, atol=1e-10)
    np.testing.assert_allclose(t, -1 + 2 * np.arange(1, L) / L, atol=1e-10)


@pytest.mark.parametrize("d", [3, 4, 5, 10, 64, 128, 1000, 16384])
def test_one_bit_centroid_is_mean_absolute_coordinate(d):
    c, t, _, _ = O.lloyd_max_sphere(d, 1)
    exact = math.exp(math.lgamma(d / 2) - math.lgamma((d + 1) / 2)) / math.sqrt(math.pi)
    assert c[1] == pytest.approx(exact, rel=1e-12)
    assert c[0] == -c[1] and t[0] == 0.0


@pytest.mark.parametrize("d,bits", [(64, 3), (128, 2), (9, 4)])
def test_lloyd_conditions_by_quadrature(d, bits):
    c, t, _, res = O.lloyd_max_sphere(d, bits)
    assert res <= 1e-12
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), atol=1e-15)
    edges = np.concatenate([[-1.0], t, [1.0]])
    f = lambda v: O.sphere_density(d, v)                          # noqa: E731
    for i in range(len(c)):
        P, _ = integrate.quad(f, edges[i], edges[i + 1], epsabs=1e-15, epsrel=1e-13)
        M, _ = integrate.quad(lambda v: v * f(v), edges[i], edges[i + 1], epsabs=1e-15,
                              epsrel=1e-13)
        assert c[i] == pytest.approx(M / P, abs=1e-9 / math.sqrt(d))


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_gaussian_limit(bits):
    g, _ = O.codebook(bits)
    gaps = []
    for d in [256, 4096, 16384]:
        c, _, _, _ = O.lloyd_max_sphere(d, bits)
        gaps.append(np.max(np.abs(c * math.sqrt(d) - g)))
    assert gaps[0] > gaps[1] > gaps[2]                      # shrinks as d grows ...
    assert gaps[2] < 2e-3                                   # ... towards the N(0,1) codebook
    assert gaps[0] / gaps[2] == pytest.approx(16384 / 256, rel=0.2)   # at rate O(1/d)


def test_exact_codebook_beats_gaussian_codebook_under_f_d():
    """At d = 128 the f_d codebook has the lower expected error under f_d (the reason for
    the variant); the N(0, 1/d) codebook is the one the path uses by default."""
    d, bits = 128, 3
    cs, ts = O.codebook(bits, "sphere", d)
    cg, tg = O.codebook(bits)

    def mse(c_unit, t_unit):
        c, t = c_unit / math.sqrt(d), t_unit / math.sqrt(d)
        edges = np.concatenate([[-1.0], t, [1.0]])
        total = 0.0
        for i in range(len(c)):
            v, _ = integrate.quad(lambda x: (x - c[i]) ** 2 * O.sphere_density(d, x),
                                  edges[i], edges[i + 1], epsabs=1e-16, epsrel=1e-12)
            total += v
        return total

    assert mse(cs, ts) < mse(cg, tg)
