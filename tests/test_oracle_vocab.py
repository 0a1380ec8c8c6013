"""Pins for the oracle's softmax statistics and inverse CDF (CPU only)."""

import numpy as np
import pytest
from scipy.special import logsumexp, softmax

from oracle import vocab


def test_row_stats_match_logsumexp():
    rng = np.random.default_rng(0)
    for V in (1, 7, 1024, 151936):
        x = rng.normal(0.0, 3.0, V)
        m, s = vocab.row_stats(x)
        assert m == x.max()
        assert m + np.log(s) == pytest.approx(logsumexp(x), rel=1e-13)
        np.testing.assert_allclose(vocab.probs(x), softmax(x), rtol=1e-12)


def test_prob_of_matches_softmax_entry():
    x = np.array([0.5, -1.0, 2.0, 2.0, -30.0])
    m, s = vocab.row_stats(x)
    for v in range(5):
        assert vocab.prob_of(x, v, m, s) == pytest.approx(softmax(x)[v],
                                                          rel=1e-14)


def test_inverse_cdf_brute_force_against_searchsorted():
    rng = np.random.default_rng(1)
    for V in range(1, 9):
        for _ in range(30):
            w = rng.random(V)
            w[rng.random(V) < 0.3] = 0.0
            if w.sum() == 0:
                w[rng.integers(V)] = 1.0
            c = np.cumsum(w)
            for u in np.linspace(0.0, 1.0 - 2.0 ** -24, 97):
                v, _ = vocab.inverse_cdf(w, u)
                ref = int(np.searchsorted(c, u * c[-1], side="right"))
                ref = min(ref, int(np.nonzero(w > 0)[0][-1]))
                assert v == ref
                assert w[v] > 0


def test_single_positive_entry_is_deterministic():
    w = np.zeros(8)
    w[5] = 0.25
    for u in (0.0, 0.3, 0.999999):
        assert vocab.inverse_cdf(w, u)[0] == 5


def test_zero_mass_prefix_and_u_zero():
    w = np.array([0.0, 0.0, 0.5, 0.0, 0.5])
    assert vocab.inverse_cdf(w, 0.0)[0] == 2
    assert vocab.inverse_cdf(w, 0.5)[0] == 4
    assert vocab.inverse_cdf(w, 0.4999)[0] == 2


def test_near_tie_flag():
    w = np.array([0.25, 0.25, 0.25, 0.25])
    assert vocab.inverse_cdf(w, 0.5)[1]             # exactly on a boundary
    assert vocab.inverse_cdf(w, 0.5 + 4e-7)[1]
    assert not vocab.inverse_cdf(w, 0.5 + 4e-6)[1]
    assert not vocab.inverse_cdf(w, 0.6)[1]


def test_empirical_distribution():
    rng = np.random.default_rng(2)
    w = np.array([0.1, 0.0, 0.4, 0.2, 0.3])
    u = (rng.integers(0, 2 ** 24, 200000) * 2.0 ** -24)
    draws = np.array([vocab.inverse_cdf(w, x)[0] for x in u[:40000]])
    freq = np.bincount(draws, minlength=5) / draws.size
    np.testing.assert_allclose(freq, w, atol=0.01)


def test_tie_alternatives_cross_only_the_near_boundary():
    # Masses 0.25 each with a zero entry between indices 1 and 3: the
    # positive-mass neighbour across the boundary at 0.5 is 3, not 2.
    w = np.array([0.25, 0.25, 0.0, 0.25, 0.25])
    total = w.sum()
    # Just below the boundary c[1] = 0.5: the draw is 1, the other side 3.
    u = (0.5 - 3e-7) / total
    assert vocab.inverse_cdf(w, u) == (1, True)
    assert vocab.tie_alternatives(w, u) == [1, 3]
    # Just above it: the draw is 3, the other side 1.
    u = (0.5 + 3e-7) / total
    assert vocab.inverse_cdf(w, u) == (3, True)
    assert vocab.tie_alternatives(w, u) == [1, 3]
    # Far from every boundary: the draw alone.
    assert vocab.tie_alternatives(w, 0.6) == [vocab.inverse_cdf(w, 0.6)[0]]
    # The first boundary has nothing before index 0.
    assert vocab.tie_alternatives(w, 1e-9) == [0]


def test_tie_alternatives_brute_force():
    # The alternatives are exactly the draws an inverse CDF makes for every
    # target within the band, on small vectors with clusters of tiny masses.
    rng = np.random.default_rng(4)
    band = 1e-6
    for _ in range(300):
        V = int(rng.integers(2, 10))
        w = rng.random(V)
        w[rng.random(V) < 0.3] = 0.0
        tiny = rng.random(V) < 0.3
        w[tiny] *= 1e-8                     # intervals narrower than the band
        if w.sum() == 0:
            w[0] = 1.0
        c = np.cumsum(w)
        k = int(rng.integers(0, V))
        u = float(np.clip((c[k] + rng.uniform(-5e-7, 5e-7) * c[-1]) / c[-1],
                          0.0, 1.0 - 2.0 ** -24))
        alts = vocab.tie_alternatives(w, u, band)
        # Targets across the band: a dense grid plus both sides of every
        # running-sum boundary inside it (intervals far narrower than any
        # grid step are still visited).
        total = c[-1]
        xs = list(u + np.linspace(-band, band, 401)[1:-1])
        for cj in c:
            for x in (cj / total * (1 - 1e-15), cj / total * (1 + 1e-15)):
                if abs(x - u) < band:
                    xs.append(x)
        seen = {vocab.inverse_cdf(w, u)[0]}
        for x in xs:
            if 0.0 <= x < 1.0:
                seen.add(vocab.inverse_cdf(w, float(x))[0])
        assert set(alts) == seen, (w, u, alts, seen)
        assert all(w[a] > 0 for a in alts)


def test_log_normaliser_is_logsumexp():
    rng = np.random.default_rng(5)
    for V in (1, 9, 151936):
        x = rng.normal(0.0, 3.0, V)
        x[int(rng.integers(V))] += 18.6
        assert vocab.log_normaliser(x) == pytest.approx(logsumexp(x),
                                                        rel=1e-14)
