"""Pins for the oracle's accept / resample step and KV commit (CPU only).

* the speculative-sampling identity: the token decided at a verified
  position is distributed as p whatever q was (the pages' claim that
  min(1, p/q) keeps the AR distribution), by chi-square;
* the acceptance rate equals sum_v min(p_v, q_v), the draft distribution
  is q and the bonus distribution is p;
* the tokens decided per step match the exact finite-horizon expectation
  of the pages' TPF chain;
* the commit keeps the page pool consistent and writes exactly the
  accepted prefix.
"""

import numpy as np
import pytest
from scipy import stats
from scipy.special import softmax

from oracle import step as ostep
from oracle import tpf


def _two_step_case(B, V, P1, Q2, P2, seed):
    """R step drafting one token from Q2, then an S step verifying it with P2.

    Returns the oracle outputs of both steps.
    """
    N, K = 2, 4
    L0 = np.full(B, 10)
    pending = np.full((B, N), -1)
    pending[:, 0] = 3
    n = np.ones(B, dtype=np.int64)
    q_row = np.full((B, N), -1)
    lc0 = np.zeros((B, K, V))
    lc0[:, 0] = P1
    lc0[:, 1] = Q2
    s0 = ostep.accept_resample(lc0, lc0, pending, n, q_row, L0, seed, 0, N)
    L1 = L0 + s0["n_commit"]
    lc1 = np.zeros((B, K, V))
    lc1[:, 0] = P2
    s1 = ostep.accept_resample(lc1, lc0, s0["next_pending"], s0["next_n"],
                               s0["next_q_row"], L1, seed, 1, N)
    return s0, s1


def _chi2_pvalue(samples, probs):
    counts = np.bincount(samples, minlength=len(probs))
    return stats.chisquare(counts, probs * counts.sum()).pvalue


@pytest.fixture(scope="module")
def identity_case():
    rng = np.random.default_rng(7)
    V, B = 8, 30000
    P1 = rng.normal(0, 1.0, V)
    Q2 = rng.normal(0, 1.5, V)
    P2 = rng.normal(0, 1.5, V)
    s0, s1 = _two_step_case(B, V, P1, Q2, P2, seed=12345)
    return dict(V=V, B=B, P1=P1, Q2=Q2, P2=P2, s0=s0, s1=s1)


def test_verified_token_is_distributed_as_p(identity_case):
    c = identity_case
    s1 = c["s1"]
    # Token at position L0 + 2: the draft if accepted, else the replacement.
    tok = np.where(s1["rejected"], s1["next_pending"][:, 0],
                   s1["commit_tokens"][:, 1])
    p2 = softmax(c["P2"])
    q2 = softmax(c["Q2"])
    assert np.abs(p2 - q2).sum() > 0.3     # q is far from p
    assert _chi2_pvalue(tok, p2) > 1e-4
    # A wrong residual (plain p instead of max(0, p - q)) would be seen:
    wrong = np.where(s1["rejected"], s1["next_pending"][:, 0], -1)
    assert _chi2_pvalue(wrong[wrong >= 0], p2) < 1e-6


def test_acceptance_rate_is_overlap(identity_case):
    c = identity_case
    s1 = c["s1"]
    alpha = np.minimum(softmax(c["P2"]), softmax(c["Q2"])).sum()
    rate = 1.0 - s1["rejected"].mean()
    sigma = np.sqrt(alpha * (1 - alpha) / c["B"])
    assert abs(rate - alpha) < 4.5 * sigma


def test_draft_is_q_and_bonus_is_p(identity_case):
    c = identity_case
    s0 = c["s0"]
    assert np.all(s0["next_n"] == 2) and not s0["rejected"].any()
    assert _chi2_pvalue(s0["next_pending"][:, 1], softmax(c["Q2"])) > 1e-4
    assert _chi2_pvalue(s0["next_pending"][:, 0], softmax(c["P1"])) > 1e-4


def test_residual_formula_on_forced_reject():
    # p puts no mass where q does: every draft from q is rejected and the
    # replacement comes from max(0, p - q) = p restricted to p's support.
    V, B = 4, 3000
    P1 = np.zeros(V)
    Q2 = np.log(np.array([1e-12, 1e-12, 0.5, 0.5]))
    P2 = np.log(np.array([0.7, 0.3, 1e-12, 1e-12]))
    _, s1 = _two_step_case(B, V, P1, Q2, P2, seed=9)
    assert s1["rejected"].all()
    assert np.all(s1["n_commit"] == 1)
    tok = s1["next_pending"][:, 0]
    assert set(np.unique(tok)) <= {0, 1}
    assert abs((tok == 0).mean() - 0.7) < 4.5 * np.sqrt(0.21 / B)


def test_identical_p_and_q_always_accept():
    # With p == q the ratio is 1 and u < 1 always accepts; the residual's
    # zero-mass fallback to p is therefore unreachable in exact arithmetic.
    V = 5
    row = np.log(np.array([0.1, 0.2, 0.3, 0.25, 0.15]))
    _, s1 = _two_step_case(200, V, row, row, row, seed=3)
    assert not s1["rejected"].any()      # ratio 1 > u always


def test_schedule_fields():
    V, B = 6, 50
    rng = np.random.default_rng(3)
    P1, Q2, P2 = (rng.normal(0, 1, V) for _ in range(3))
    s0, s1 = _two_step_case(B, V, P1, Q2, P2, seed=1)
    # R step: commits row 0 only, drafts one token from row 1.
    assert np.all(s0["n_commit"] == 1)
    assert np.all(s0["commit_tokens"][:, 0] == 3)
    assert np.all(s0["next_q_row"][:, 1] == 1)
    # S step: accepted -> commits 2 and goes back to S; rejected -> 1 and R.
    acc = ~s1["rejected"]
    assert np.all(s1["n_commit"][acc] == 2) and np.all(s1["next_n"][acc] == 2)
    assert np.all(s1["n_commit"][~acc] == 1)
    assert np.all(s1["next_n"][~acc] == 1)


@pytest.mark.parametrize("N,alpha", [(4, 0.9), (3, 0.7)])
def test_tokens_per_forward_matches_chain(N, alpha):
    """Constant per-draft acceptance alpha: decided tokens per step follow
    the finite-horizon expectation of the pages' TPF chain."""
    V, K, B, T = 2, 2 * N, 1500, 16
    p = np.array([0.5 + (1 - alpha), 0.5 - (1 - alpha)])
    q = np.array([0.5, 0.5])
    assert np.minimum(p, q).sum() == pytest.approx(alpha)
    lp, lq = np.log(p), np.log(q)
    L = np.zeros(B, dtype=np.int64)
    pending = np.full((B, N), -1)
    pending[:, 0] = 0
    n = np.ones(B, dtype=np.int64)
    q_row = np.full((B, N), -1)
    prev = np.zeros((B, K, V))
    total = np.zeros(B)
    for s in range(T):
        cur = np.where((np.arange(K)[None, :] < n[:, None])[..., None],
                       lp[None, None, :], lq[None, None, :])
        o = ostep.accept_resample(cur, prev, pending, n, q_row, L, 77, s, N)
        total += o["n_commit"]
        L = L + o["n_commit"]
        pending, n, q_row, prev = (o["next_pending"], o["next_n"],
                                   o["next_q_row"], cur)
    expect = tpf.expected_tokens(alpha, N, T, start=1)
    se = total.std(ddof=1) / np.sqrt(B)
    assert abs(total.mean() - expect) < 4.5 * se


def _commit_case(rng, B, N, extra_pages):
    Hkv, d, ps = 2, 4, 16
    L = rng.integers(0, 40, B)
    owned = (L + ps - 1) // ps
    max_pages = int(((L + N + ps - 1) // ps).max()) + 1
    grow = int((((L + N + ps - 1) // ps) - owned).sum())
    P = int(owned.sum()) + grow + extra_pages
    perm = rng.permutation(P)
    pt = np.full((B, max_pages), -1)
    at = 0
    for b in range(B):
        pt[b, :owned[b]] = perm[at:at + owned[b]]
        at += owned[b]
    free = perm[at:][::-1].copy()
    fs = np.full(P, -1)
    fs[:free.size] = free
    kc = rng.normal(size=(P, Hkv, ps, d))
    vc = rng.normal(size=(P, Hkv, ps, d))
    kn = rng.normal(size=(B, 2 * N, Hkv, d))
    vn = rng.normal(size=(B, 2 * N, Hkv, d))
    nc = rng.integers(1, N + 1, B)
    return kn, vn, kc, vc, pt, L, nc, fs, free.size


def test_commit_invariants():
    rng = np.random.default_rng(11)
    for trial in range(20):
        B, N = int(rng.integers(1, 9)), int(rng.integers(2, 9))
        kn, vn, kc, vc, pt, L, nc, fs, top = _commit_case(rng, B, N, 3)
        kc2, vc2, pt2, L2, top2, st = ostep.kv_commit(kn, vn, kc, vc, pt, L,
                                                      nc, fs, top)
        assert st == ostep.STATUS_OK
        assert np.array_equal(L2, L + nc)
        owned = [p for b in range(B) for p in pt2[b] if p >= 0]
        free = list(fs[:top2])
        assert len(owned) == len(set(owned))
        assert sorted(owned + free) == list(range(kc.shape[0]))
        for b in range(B):
            assert np.count_nonzero(pt2[b] >= 0) == (L2[b] + 15) // 16
            for r in range(nc[b]):
                pos = L[b] + r
                ph = pt2[b, pos // 16]
                assert np.array_equal(kc2[ph, :, pos % 16], kn[b, r])
                assert np.array_equal(vc2[ph, :, pos % 16], vn[b, r])
        # Nothing outside the committed slots changed.
        changed = np.argwhere(np.any(kc2 != kc, axis=(1, 3)))
        assert len(changed) <= int(nc.sum()) * kc.shape[1]
        # Pages are handed out top of stack first, sequence 0 first.
        popped = [p for b in range(B) for p in pt2[b] if p >= 0
                  and p not in pt[b]]
        assert popped == list(fs[top2:top][::-1])


def test_commit_pool_exhausted_is_all_or_nothing():
    rng = np.random.default_rng(5)
    for _ in range(10):
        kn, vn, kc, vc, pt, L, nc, fs, top = _commit_case(rng, 6, 4, 0)
        L[:] = 15                         # everyone crosses a page boundary
        nc[:] = 2
        owned = (L + 15) // 16
        pt[:, :] = -1
        for b in range(6):
            pt[b, 0] = b
        res = ostep.kv_commit(kn, vn, kc, vc, pt, L, nc, fs, 5)
        assert res[5] == ostep.STATUS_POOL_EXHAUSTED
        assert np.array_equal(res[2], pt) and np.array_equal(res[3], L)
        assert res[4] == 5 and np.array_equal(res[0], kc)
        del owned


def test_commit_page_table_full():
    rng = np.random.default_rng(6)
    kn, vn, kc, vc, pt, L, nc, fs, top = _commit_case(rng, 3, 4, 5)
    L[1] = pt.shape[1] * 16 - 1
    nc[1] = 2
    res = ostep.kv_commit(kn, vn, kc, vc, pt, L, nc, fs, top)
    assert res[5] == ostep.STATUS_PAGE_TABLE_FULL
    assert np.array_equal(res[3], L)


def test_flip_takes_the_other_branch_of_a_ratio_test():
    """flip decides one ratio test the other way and everything after it
    follows that decision: flipping the first rejection accepts that draft
    (and goes on testing), flipping an accepted draft rejects there."""
    rng = np.random.default_rng(11)
    V, B, N = 12, 400, 4
    K = 2 * N
    lc0 = rng.normal(0.0, 1.0, (B, K, V))
    pending = np.full((B, N), -1)
    pending[:, 0] = rng.integers(0, V, B)
    L0 = np.full(B, 40)
    s0 = ostep.accept_resample(lc0, lc0, pending, np.ones(B, dtype=np.int64),
                               np.full((B, N), -1), L0, 3, 0, N)
    lc1 = rng.normal(0.0, 1.0, (B, K, V))
    L1 = L0 + s0["n_commit"]
    args = (lc1, lc0, s0["next_pending"], s0["next_n"], s0["next_q_row"], L1,
            3, 1, N)
    base = ostep.accept_resample(*args)
    flips = []
    for b in range(B):
        a = int(base["accepted"][b])
        if base["rejected"][b]:
            flips.append((b, a + 1, "to_accept"))
        elif a >= 1:
            flips.append((b, a, "to_reject"))
    assert len(flips) > 50
    alt = ostep.accept_resample(*args, flip=[(b, i) for b, i, _ in flips])
    for b, i, kind in flips:
        if kind == "to_accept":
            assert alt["accepted"][b] >= i           # draft i now passes
            assert alt["n_commit"][b] >= i + 1
        else:
            assert alt["rejected"][b] and alt["accepted"][b] == i - 1
            assert alt["n_commit"][b] == i
            # Decided the same way before the flipped test: same prefix.
            assert np.array_equal(alt["commit_tokens"][b, :i],
                                  base["commit_tokens"][b, :i])
    # Untouched sequences are unchanged.
    touched = {b for b, _, _ in flips}
    for b in range(B):
        if b not in touched:
            assert alt["n_commit"][b] == base["n_commit"][b]
            assert np.array_equal(alt["next_pending"][b],
                                  base["next_pending"][b])


def test_next_q_logz_is_the_draft_rows_logsumexp():
    from scipy.special import logsumexp
    rng = np.random.default_rng(12)
    V, B, N = 50, 20, 3
    lc = rng.normal(0.0, 2.0, (B, 2 * N, V))
    pending = np.full((B, N), -1)
    pending[:, 0] = 1
    o = ostep.accept_resample(lc, lc, pending, np.ones(B, dtype=np.int64),
                              np.full((B, N), -1), np.full(B, 5), 0, 0, N)
    for b in range(B):
        for j in range(1, N):
            row = int(o["next_q_row"][b, j])
            assert row == j                       # R mode: n = 1
            assert o["next_q_logz"][b, j] == pytest.approx(
                logsumexp(lc[b, row]), rel=1e-14)
