"""Tokens per forward (TPF) of the ISD stride schedule.

Test infrastructure only (see ``oracle/__init__.py``).

The pages print one closed form (hada.io summary, "Speedup Factor
Explorer", memory-bound case):

    TPF = (2 + p + p^2 + ... + p^(N-2)) / (2 - p^(N-1))

with per-token acceptance probability p and stride N, and, under
"Throughput", the efficiency TPF^2 / query_size with I-DLM (N=4, p=0.9)
at TPF ~ 2.9, efficiency 1.22 and SDAR (N=4, p=0.5) at TPF ~ 1.1,
efficiency 0.31.

``tpf_closed_form`` is that formula.  ``tpf_markov`` computes the same
quantity from the schedule itself (the two-state chain of
``oracle/step.py``), with no algebra shared with the closed form, so the
two agreeing pins the schedule reading.  ``expected_tokens`` is the exact
finite-horizon expectation from a given start state.
"""

import numpy as np


def tpf_closed_form(p, N):
    """The pages' memory-bound TPF formula."""
    num = 2.0 + sum(p ** k for k in range(1, N - 1))
    return num / (2.0 - p ** (N - 1))


def efficiency(tpf, query_size):
    """TPF^2 / query_size, the pages' compute-efficiency measure."""
    return tpf * tpf / query_size


def schedule_chain(p, N):
    """Transition matrix and expected yields of the stride schedule.

    States: 0 = S (N - 1 drafts pending), 1 = R (only the exact token).
    In S, a drafts are accepted before the first rejection with
    probability p^a (1 - p) for a < N - 1, and all N - 1 with probability
    p^(N-1); the step decides a + 1 tokens and goes to S only if all were
    accepted.  R decides one token (the bonus) and goes to S.
    Returns (P [2][2], yields [2], yield_sq [2]) with the first and second
    moments of the tokens decided per step in each state.
    """
    probs_a = [p ** a * (1.0 - p) for a in range(N - 1)] + [p ** (N - 1)]
    y_s = sum(pa * (a + 1) for a, pa in enumerate(probs_a))
    y2_s = sum(pa * (a + 1) ** 2 for a, pa in enumerate(probs_a))
    stay = probs_a[-1]
    P = np.array([[stay, 1.0 - stay], [1.0, 0.0]])
    return P, np.array([y_s, 1.0]), np.array([y2_s, 1.0])


def tpf_markov(p, N):
    """Stationary tokens per forward of the schedule chain."""
    P, y, _ = schedule_chain(p, N)
    # Stationary distribution: left eigenvector of P for eigenvalue 1.
    A = np.vstack([P.T - np.eye(2), np.ones((1, 2))])
    rhs = np.array([0.0, 0.0, 1.0])
    pi = np.linalg.lstsq(A, rhs, rcond=None)[0]
    return float(pi @ y)


def expected_tokens(p, N, steps, start=1):
    """Exact expected tokens decided in ``steps`` steps from ``start``."""
    P, y, _ = schedule_chain(p, N)
    dist = np.zeros(2)
    dist[start] = 1.0
    total = 0.0
    for _ in range(steps):
        total += float(dist @ y)
        dist = dist @ P
    return total
