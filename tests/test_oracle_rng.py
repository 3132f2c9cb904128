"""Pins for the oracle's random tables (SplitMix64, bounded integers, RPBH perm/sign).

The OrbitQuant summary (rcap.io, RPBH paragraph) asks for a uniform random permutation and
random sign flips; the generator, draw order and bounded-integer method are a reading.
These tests pin that reading to things outside the oracle: published generator outputs, a
hand-worked tiny case, and the statistics a uniform permutation / fair signs must show.
"""
import itertools

import numpy as np
import pytest
from scipy import stats

import oracle as O
from conftest import golden_rows


def test_splitmix64_published_vector():
    """First outputs from state 1234567 equal the published reference outputs."""
    lines = golden_rows("splitmix64_reference.txt")
    seed = int(lines[0][0].split()[1])
    expected = [int(r[0]) for r in lines[1:]]
    got = [int(v) for v in O.splitmix64(seed, len(expected))]
    assert got == expected


def test_uniform_below_power_of_two_takes_low_bits():
    """n = 2^k has no rejected range, so the result is r mod n of the pinned outputs."""
    raw = [int(v) for v in O.splitmix64(42, 50)]
    for k in (1, 3, 17, 63):
        n = 1 << k
        got = [int(v) for v in O.uniform_below(42, n, 50)]
        assert got == [r % n for r in raw]


def test_uniform_below_rejects_the_partial_top_range():
    """n = 2^63 + 1: 2^64 mod n = 2^63 - 1, so draws >= 2^63 + 1 are skipped and kept
    draws are returned unchanged (they are already < n)."""
    n = (1 << 63) + 1
    raw = [int(v) for v in O.splitmix64(7, 400)]
    kept = [r for r in raw if r < n]
    got = [int(v) for v in O.uniform_below(7, n, 100)]
    assert got == kept[:100]
    assert len(kept) >= 100


@pytest.mark.parametrize("n", [3, 5, 7, 10])
def test_uniform_below_is_uniform(n):
    draws = O.uniform_below(2024 + n, n, 30000).astype(np.int64)
    assert draws.min() >= 0 and draws.max() < n
    counts = np.bincount(draws, minlength=n)
    assert stats.chisquare(counts).pvalue > 1e-4


def test_rpbh_handworked_tiny_cases():
    for head, perm_s, sign_s in golden_rows("rpbh_tiny_handworked.txt"):
        d, seed = (int(v) for v in head.split())
        perm, sign = O.build_rpbh(d, seed)
        assert perm.tolist() == [int(v) for v in perm_s.split()]
        assert sign.tolist() == [int(v) for v in sign_s.split()]


@pytest.mark.parametrize("d", [256, 3072, 16384])
def test_rpbh_is_a_bijection_with_fair_signs(d):
    perm, sign = O.build_rpbh(d, 0)
    assert np.array_equal(np.sort(perm), np.arange(d))
    assert set(np.unique(sign).tolist()) <= {-1, 1}
    plus = int((sign == 1).sum())
    # binomial(d, 1/2): 5 standard deviations
    assert abs(plus - d / 2) < 5 * np.sqrt(d) / 2


def test_rpbh_permutations_are_uniform_over_seeds():
    """Every one of the 24 permutations of 4 elements appears equally often."""
    index = {p: i for i, p in enumerate(itertools.permutations(range(4)))}
    counts = np.zeros(24, dtype=np.int64)
    for seed in range(24000):
        perm, _ = O.build_rpbh(4, seed)
        counts[index[tuple(perm.tolist())]] += 1
    assert counts.min() > 0
    assert stats.chisquare(counts).pvalue > 1e-4


def test_rpbh_first_entry_uniform_and_seeds_differ():
    d = 64
    first = np.array([O.build_rpbh(d, s)[0][0] for s in range(6400)])
    assert stats.chisquare(np.bincount(first, minlength=d)).pvalue > 1e-4
    a, _ = O.build_rpbh(3072, 0)
    b, _ = O.build_rpbh(3072, 1)
    assert not np.array_equal(a, b)
