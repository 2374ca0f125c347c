"""Pins for the oracle's temperature softmax, top-p truncation and draw.

Checked against scipy's softmax, closed forms, brute-force subset search on
tiny vocabularies and exact rational arithmetic for the inverse-CDF draw.
"""
import itertools
import json
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy.special import softmax

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_claims.json")))
T_PAGES = GOLDEN["temperature"]["value"]
TOPP_PAGES = GOLDEN["top_p"]["value"]


@pytest.mark.parametrize("T", [0.6, 1.0, 2.5])
def test_top_p_one_is_plain_softmax(T):
    rng = np.random.default_rng(10)
    l = 1.4 * rng.standard_normal(1000)
    p, info = oracle.warp(l, T, 1.0)
    np.testing.assert_allclose(p, softmax(l / T), rtol=1e-12, atol=1e-300)
    assert info["kept"] == 1000


def test_two_token_closed_form():
    # p0 = 1 / (1 + exp(-(l0 - l1)/T))
    for d in [0.0, 0.3, 2.0, -1.7]:
        p, _ = oracle.warp(np.array([d, 0.0]), 0.6, 1.0)
        assert abs(p[0] - 1.0 / (1.0 + np.exp(-d / 0.6))) < 1e-15
        assert abs(p.sum() - 1.0) < 1e-15


def test_shift_invariance_and_normalisation():
    rng = np.random.default_rng(11)
    l = rng.standard_normal(4096)
    p1, _ = oracle.warp(l, T_PAGES, TOPP_PAGES)
    p2, _ = oracle.warp(l + 37.25, T_PAGES, TOPP_PAGES)
    np.testing.assert_allclose(p1, p2, rtol=1e-12, atol=1e-300)
    assert abs(p1.sum() - 1.0) < 1e-12


def test_greedy_one_hot_with_lowest_index_tie_rule():
    l = np.array([0.5, 2.0, -1.0, 2.0, 1.9])
    p, info = oracle.warp(l, 0.0, TOPP_PAGES)
    assert list(p) == [0, 1, 0, 0, 0]
    assert info["kept"] == 1


def test_small_temperature_tends_to_greedy():
    rng = np.random.default_rng(12)
    l = rng.standard_normal(300)
    p, _ = oracle.warp(l, 1e-3, TOPP_PAGES)
    assert p[np.argmax(l)] == 1.0 and p.sum() == 1.0


def _brute_force_top_p(p, top_p, l):
    """Smallest-cardinality subset with mass >= top_p; among those the
    largest mass; among equal masses the lexicographically smallest index set.
    """
    V = len(p)
    for size in range(1, V + 1):
        best = None
        for sub in itertools.combinations(range(V), size):
            mass = sum(p[j] for j in sub)
            if mass >= top_p - 1e-15:
                key = (-round(mass, 14), sub)
                if best is None or key < best[0]:
                    best = (key, sub)
        if best is not None:
            return set(best[1])
    return set(range(V))


@pytest.mark.parametrize("seed", range(40))
def test_top_p_matches_brute_force_subset_search(seed):
    rng = np.random.default_rng(100 + seed)
    V = int(rng.integers(2, 9))
    # coarse grid -> frequent exact ties in logits (and hence in p)
    l = np.round(rng.standard_normal(V) * 2) / 2 if seed % 2 else rng.standard_normal(V)
    top_p = float(rng.choice([0.5, 0.8, TOPP_PAGES, 0.3]))
    T = float(rng.choice([0.6, 1.0]))
    p_full = softmax(l / T)
    kept_expected = _brute_force_top_p(p_full, top_p, l)
    p, info = oracle.warp(l, T, top_p)
    kept = set(np.nonzero(p)[0].tolist())
    # skip cases where the crossing is within rounding of top_p
    cums = np.cumsum(sorted(p_full, reverse=True))
    if np.min(np.abs(cums - top_p)) < 1e-12:
        pytest.skip("crossing within rounding of top_p")
    assert kept == kept_expected
    ref = np.zeros(V)
    for j in kept_expected:
        ref[j] = p_full[j]
    np.testing.assert_allclose(p, ref / ref.sum(), rtol=1e-12, atol=1e-300)


def test_top_p_tie_keeps_lower_indices():
    # four equal logits: 0.5 mass needs exactly two of them: indices 0 and 1
    p, info = oracle.warp(np.array([1.0, 1.0, 1.0, 1.0]), 1.0, 0.5)
    assert list(p) == [0.5, 0.5, 0.0, 0.0]
    # order by logit first: index 2 has the largest logit, then ties 0 < 3
    # p = (0.0453, 0.0003, 0.9094, 0.0453): 0.9094 < 0.93 <= 0.9547
    p, info = oracle.warp(np.array([0.0, -5.0, 3.0, 0.0]), 1.0, 0.93)
    assert p[2] > 0 and p[0] > 0 and p[3] == 0 and p[1] == 0


def test_top_p_mass_properties():
    rng = np.random.default_rng(13)
    l = 1.43 * rng.standard_normal(20000)
    p_full = softmax(l / T_PAGES)
    p, info = oracle.warp(l, T_PAGES, TOPP_PAGES)
    kept = p > 0
    # kept set is a prefix in descending logit order
    assert l[kept].min() >= l[~kept].max()
    # its mass reaches top_p, and dropping its smallest member falls below
    mass = p_full[kept].sum()
    assert mass >= TOPP_PAGES - 1e-12
    assert mass - p_full[kept].min() < TOPP_PAGES + 1e-12
    assert abs(info["kept_sum"] - mass) < 1e-12


def test_non_finite_logit_is_reported():
    _, info = oracle.warp(np.array([0.0, np.nan, 1.0]), 1.0, 0.9)
    assert info["status"] == 2
    _, info = oracle.warp(np.array([0.0, np.inf]), 1.0, 0.9)
    assert info["status"] == 2


def test_draw_is_exact_inverse_cdf():
    """Every 2**-24-grid uniform lands in the bin that exact rational
    arithmetic assigns it; zero-weight bins are never chosen."""
    rng = np.random.default_rng(14)
    for trial in range(30):
        V = int(rng.integers(1, 9))
        w = rng.random(V)
        w[rng.random(V) < 0.3] = 0.0
        if w.sum() == 0:
            w[0] = 0.25
        total = sum(Fraction(float(x)) for x in w)
        for k in rng.integers(0, 2 ** 24, size=200):
            u = float(k) * 2.0 ** -24
            x, _ = oracle.draw(w, u)
            target = Fraction(int(k), 2 ** 24) * total
            c = Fraction(0)
            expect = None
            for j in range(V):
                c += Fraction(float(w[j]))
                if c > target:
                    expect = j
                    break
            # exact and rounded cumulative sums agree away from a bin edge
            edge_gap = min(abs(float(sum(Fraction(float(x)) for x in w[:j + 1]) - target))
                           for j in range(V))
            if edge_gap > 1e-12:
                assert x == expect
            assert w[x] > 0


def test_draw_counts_on_the_full_uniform_grid():
    # bin x receives exactly ceil(C_x * 2^24 / total) - ceil(C_{x-1} * 2^24 / total)
    # grid points (power-of-two weights make every edge exact).
    w = np.array([0.25, 0.0, 0.125, 0.5, 0.125])
    total = w.sum()
    edges = np.concatenate([[0.0], np.cumsum(w)]) / total
    ks = np.arange(0, 2 ** 24, 997)
    counts = np.zeros(5, dtype=np.int64)
    for k in ks:
        x, _ = oracle.draw(w, float(k) * 2.0 ** -24)
        counts[x] += 1
    expect = np.zeros(5, dtype=np.int64)
    for k in ks:
        u = k * 2.0 ** -24
        expect[int(np.searchsorted(edges, u, side="right")) - 1] += 1
    assert np.array_equal(counts, expect)
    assert counts[1] == 0


def test_draw_exact_edges_and_leading_zeros():
    # x = min{k : C_k > u * total}: a uniform exactly on an edge belongs to the
    # next bin, and u = 0 skips leading zero-weight bins.
    w = np.array([0.0, 0.25, 0.0, 0.75])
    assert oracle.draw(w, 0.0)[0] == 1
    assert oracle.draw(w, 0.25)[0] == 3
    assert oracle.draw(w, 0.25 - 2.0 ** -24)[0] == 1
    assert oracle.draw(w, 1.0 - 2.0 ** -24)[0] == 3
    # rounding leaves no crossing (u*total == total cannot happen for u < 1,
    # so emulate with u = 1): the last positive bin is returned
    assert oracle.draw(np.array([0.5, 0.5, 0.0]), 1.0)[0] == 1
