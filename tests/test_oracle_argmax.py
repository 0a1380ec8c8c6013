"""Pins for the oracle's argmax-proposal variant (CPU only).

Drafts are x = argmax q (first maximal index), accepted with probability
p(x), and a rejection resamples from p with x removed.  Fixed by the
mathematics of speculative sampling with a point-mass proposal:

* the token decided at a verified position is distributed as p (chi-square);
* the acceptance rate is p(argmax q) (binomial band);
* the replacement never equals the rejected draft and follows p without x;
* exact ties at the maximum of q resolve to the lowest index.
"""

import numpy as np
import pytest
from scipy import stats
from scipy.special import softmax

from oracle import step as ostep


def _two_step_case(B, V, P1, Q2, P2, seed, proposal="argmax"):
    """R step proposing one draft from Q2, then an S step verifying it with
    P2 (N = 2, K = 4).  Returns the oracle outputs of both steps."""
    N, K = 2, 4
    L0 = np.full(B, 10)
    pending = np.full((B, N), -1)
    pending[:, 0] = 3
    n = np.ones(B, dtype=np.int64)
    q_row = np.full((B, N), -1)
    lc0 = np.zeros((B, K, V))
    lc0[:, 0] = P1
    lc0[:, 1] = Q2
    s0 = ostep.accept_resample(lc0, lc0, pending, n, q_row, L0, seed, 0, N,
                               proposal=proposal)
    L1 = L0 + s0["n_commit"]
    lc1 = np.zeros((B, K, V))
    lc1[:, 0] = P2
    s1 = ostep.accept_resample(lc1, lc0, s0["next_pending"], s0["next_n"],
                               s0["next_q_row"], L1, seed, 1, N,
                               proposal=proposal)
    return s0, s1


def _chi2_pvalue(samples, probs):
    counts = np.bincount(samples, minlength=len(probs))
    keep = probs > 0
    return stats.chisquare(counts[keep], probs[keep] * counts.sum()).pvalue


@pytest.fixture(scope="module")
def case():
    rng = np.random.default_rng(11)
    V, B = 8, 30000
    P1 = rng.normal(0, 1.0, V)
    Q2 = rng.normal(0, 1.5, V)
    P2 = rng.normal(0, 1.0, V)
    s0, s1 = _two_step_case(B, V, P1, Q2, P2, seed=2024)
    return dict(V=V, B=B, P1=P1, Q2=Q2, P2=P2, s0=s0, s1=s1,
                x=int(np.argmax(Q2)))


def test_draft_is_argmax_of_q(case):
    assert np.all(case["s0"]["next_pending"][:, 1] == case["x"])


def test_verified_token_is_distributed_as_p(case):
    s1 = case["s1"]
    tok = np.where(s1["rejected"], s1["next_pending"][:, 0],
                   s1["commit_tokens"][:, 1])
    assert _chi2_pvalue(tok, softmax(case["P2"])) > 1e-4


def test_acceptance_rate_is_p_of_the_draft(case):
    p_x = softmax(case["P2"])[case["x"]]
    rate = 1.0 - case["s1"]["rejected"].mean()
    sigma = np.sqrt(p_x * (1 - p_x) / case["B"])
    assert abs(rate - p_x) < 4.5 * sigma
    # the ratio reported is p(x) itself (q(x) = 1)
    r = case["s1"]["ratio"][:, 1]
    assert np.allclose(r, p_x, rtol=1e-12)


def test_residual_is_p_without_the_draft(case):
    s1, x = case["s1"], case["x"]
    rej = s1["rejected"]
    tok = s1["next_pending"][rej, 0]
    assert not np.any(tok == x)
    w = softmax(case["P2"]).copy()
    w[x] = 0.0
    assert _chi2_pvalue(tok, w / w.sum()) > 1e-4
    # a residual that kept x (plain p) would be seen
    assert _chi2_pvalue(tok, softmax(case["P2"])) < 1e-6


def test_ties_at_the_maximum_take_the_lowest_index():
    V = 6
    Q2 = np.array([0.0, 5.0, 1.0, 5.0, -2.0, 5.0])
    s0, _ = _two_step_case(10, V, np.zeros(V), Q2, np.zeros(V), seed=5)
    assert np.all(s0["next_pending"][:, 1] == 1)
