"""Pins for the oracle's Philox4x32-10 and uniform stream (CPU only)."""

import os

import numpy as np
import pytest
from scipy import stats

from oracle import philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "philox4x32_10_kat.txt")


def _kat_rows():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            words = [int(w, 16) for w in line.split()]
            rows.append((words[0:4], words[4:6], words[6:10]))
    return rows


@pytest.mark.parametrize("ctr,key,expect", _kat_rows())
def test_known_answer_vectors(ctr, key, expect):
    assert list(philox.philox4x32_10(ctr, key)) == expect


@pytest.mark.parametrize("ctr,key,expect", _kat_rows())
def test_known_answer_vectors_vectorised(ctr, key, expect):
    out = philox.philox4x32_10_np(*ctr, *key)
    assert [int(v) for v in out] == expect


def test_vectorised_matches_scalar():
    rng = np.random.default_rng(1)
    c = rng.integers(0, 2 ** 32, size=(6, 200), dtype=np.uint64)
    out = philox.philox4x32_10_np(c[0], c[1], c[2], c[3], c[4], c[5])
    for i in range(200):
        ref = philox.philox4x32_10([int(c[k, i]) for k in range(4)],
                                   [int(c[4, i]), int(c[5, i])])
        assert tuple(int(o[i]) for o in out) == ref


def test_uniform_grid_and_range():
    u = philox.uniform_np(0, np.arange(4096), 7, 123, 0)
    assert u.min() >= 0.0 and u.max() <= 1.0 - 2.0 ** -24
    k = u * 2.0 ** 24
    assert np.all(k == np.floor(k))
    assert philox.uniform(0, 5, 7, 123, 0) == u[5]


def test_uniform_depends_on_every_counter_word_and_the_seed():
    base = philox.uniform(3, 1, 2, 3, 0)
    assert philox.uniform(4, 1, 2, 3, 0) != base
    assert philox.uniform(3 + (1 << 32), 1, 2, 3, 0) != base
    assert philox.uniform(3, 2, 2, 3, 0) != base
    assert philox.uniform(3, 1, 3, 3, 0) != base
    assert philox.uniform(3, 1, 2, 4, 0) != base
    assert philox.uniform(3, 1, 2, 3, 1) != base


def test_uniform_chi_square():
    n = 1 << 16
    seq = np.arange(n) % 64
    pos = np.arange(n) // 64
    u = philox.uniform_np(0, seq, 11, pos, 2)
    counts = np.bincount((u * 64).astype(np.int64), minlength=64)
    assert stats.chisquare(counts).pvalue > 1e-4
