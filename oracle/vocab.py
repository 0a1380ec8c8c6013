"""Vocabulary softmax statistics, probabilities and the inverse CDF (fp64).

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix: the model proposes tokens from q at MASK positions and
verifies them with p at clean positions ("Inference & ISD" on the hada.io
summary).  Both are the softmax of a logits row over the vocabulary.
Temperature 1 and no truncation (the pages name neither).

Readings for the sampler (the pages print no sampler):
* a draw from an unnormalised non-negative mass vector w with uniform u
  returns the smallest index v (ascending vocabulary order) whose running
  sum exceeds u * sum(w) -- strictly greater, so entries of zero mass are
  never chosen;
* if rounding leaves u * sum(w) at or above every running sum, the last
  index with positive mass is returned;
* a draw is a near-tie when u * sum(w) lies within ``tie_band * sum(w)``
  of either end of the chosen index's interval; fp32 and fp64 may then
  legitimately choose neighbouring indices: the positive-mass index on the
  other side of each boundary the target is that close to
  (``tie_alternatives``).
"""

import numpy as np

TIE_BAND = 1e-6


def row_stats(logits):
    """(m, s): the row maximum and sum_v exp(l_v - m), in float64."""
    x = np.asarray(logits, dtype=np.float64)
    m = float(np.max(x))
    s = float(np.sum(np.exp(x - m)))
    return m, s


def probs(logits):
    """Softmax of one logits row: exp(l_v - m) / s."""
    x = np.asarray(logits, dtype=np.float64)
    m, s = row_stats(x)
    return np.exp(x - m) / s


def prob_of(logits, x, m, s):
    """p(x) = exp(l_x - m) / s for given row statistics."""
    return float(np.exp(float(logits[x]) - m) / s)


def inverse_cdf(mass, u, tie_band=TIE_BAND):
    """Inverse-CDF draw from an unnormalised mass vector.

    Returns (index, near_tie).  ``mass`` must be non-negative with a
    positive sum.
    """
    w = np.asarray(mass, dtype=np.float64)
    c = np.cumsum(w)
    total = float(c[-1])
    t = u * total
    above = np.nonzero(c > t)[0]
    if above.size:
        v = int(above[0])
    else:
        v = int(np.nonzero(w > 0)[0][-1])
    hi = float(c[v])
    band = tie_band * total
    near = (hi - t) < band
    if v > 0:
        near = near or (t - float(c[v - 1])) < band
    return v, bool(near)


def tie_alternatives(mass, u, tie_band=TIE_BAND):
    """Every index a near-tie draw may legitimately return.

    The target is t = u * sum(w); a draw whose running sums carry an error
    below ``tie_band * sum(w)`` may land anywhere within that distance of
    t.  Returned: every positive-mass index whose interval
    [c[v - 1], c[v]) meets (t - band, t + band) -- the draw's own index and,
    across each boundary that close, as many neighbours as lie in the band
    (tiny masses can put several there).  Sorted.
    """
    w = np.asarray(mass, dtype=np.float64)
    c = np.cumsum(w)
    total = float(c[-1])
    t = u * total
    band = tie_band * total
    v, _ = inverse_cdf(w, u, tie_band)
    lo = np.concatenate([[0.0], c[:-1]])
    hit = (w > 0) & (lo < t + band) & (c > t - band)
    return sorted(set(np.nonzero(hit)[0].tolist()) | {v})


def log_normaliser(logits):
    """ln sum_v exp(l_v) = m + ln s (the log-partition function of a row)."""
    m, s = row_stats(logits)
    return m + float(np.log(s))
