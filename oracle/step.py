"""One ISD accept / resample step and the KV commit, in fp64.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix (hada.io summary of "Introspective Diffusion Language
Models"): one forward pass both verifies the previously generated tokens
and advances new ones ("Introspective Strided Decoding"); new tokens are
proposed from q at MASK positions and checked with p at clean positions,
and a proposal x is kept with probability min(1, p(x) / q(x)), which keeps
the autoregressive distribution ("Inference & ISD"); the KV cache is paged
("Serving (SGLang)"); the model has strict causal attention and a logit
shift, so the output at position t scores token t + 1 ("Méthodologie").

Readings taken where the pages are silent (each pinned by a test):

Stride schedule.  A stride advances N tokens: one exact token, already
final, followed by N - 1 drafts.  Sequence b holds n_b pending tokens at
absolute positions L_b .. L_b + n_b - 1 (rows 0 .. n_b - 1 of the stride);
rows n_b .. K - 1 (K = 2N) are MASK.  n_b = N after a step whose drafts
were all accepted ("S" mode) and n_b = 1 after a rejection ("R" mode:
the drafts that followed a rejected token are discarded).  Under the logit
shift, row r scores position L_b + r + 1, so
  * draft i (row i) is verified with p from row i - 1,
  * the bonus token comes from p of row n_b - 1,
  * the next drafts come from q of MASK rows n_b .. n_b + N - 2,
  * any remaining rows are spare and ignored.
This realises the pages' tokens-per-forward closed form exactly (see
``oracle/tpf.py``): S -> S with probability p^(N-1) yielding N tokens,
otherwise S -> R; R -> S yielding one token; and 2N - 1 query rows in
S mode, the query size behind the printed efficiency 1.22.

Acceptance.  Drafts are tested in order i = 1 .. n_b - 1 with
u_i = U(seed, b, step, L_b + i, ACCEPT); draft i is accepted iff
u_i < p_i(x_i) / q_i(x_i); a_b counts the accepted drafts before the first
rejection.  A draft whose |u_i - ratio| < 1e-6 is a near-tie.

Resample.  At the first rejection (draft a_b + 1) the replacement at
position L_b + a_b + 1 is drawn from normalise(max(0, p - q)) with p from
row a_b and q the stored draft distribution of draft a_b + 1 (the standard
speculative-sampling residual; it is what makes the min(1, p/q) rule keep
the distribution p).  If that residual has zero total mass, the draw is
taken from p.  Stream RESAMPLE.

Bonus and drafts.  If every draft is accepted, the token at L_b + n_b is
drawn from p of row n_b - 1 (stream BONUS) and becomes the next exact
token, and the next drafts at L_b + n_b + j (j = 1 .. N - 1) are drawn
from q of rows n_b + j - 1 (stream DRAFT).  Their q rows (this step's
logits buffer, the next step's "previous" buffer) are remembered.

Argmax proposals (the pages' serving option of proposing the most likely
token at each MASK position).  Drafts are x = argmax q (lowest index among
exact ties) instead of draws from q: the proposal is a point mass at x, so
q(x) = 1 and the ratio test accepts x with probability min(1, p(x)) =
p(x); the speculative-sampling residual max(0, p - delta_x) is p with x
removed (renormalised).  The verified token is still distributed as p.
The bonus and the replacement are drawn as before.

KV commit and rollback.  The pending rows 0 .. a_b (the exact token and
the accepted drafts) are committed: n_commit_b = 1 + a_b.  Their staged
K/V rows are copied to cache positions L_b .. L_b + n_commit_b - 1 and
L_b grows by n_commit_b.  Rejected drafts and MASK rows are never written,
which is the rollback.  Pages are taken from a free stack only when a
committed position enters a new page, in ascending sequence order; no page
is freed.  The new exact token's KV is produced by the next step's row 0.
"""

import numpy as np

from . import philox
from .vocab import (TIE_BAND, inverse_cdf, log_normaliser, prob_of, probs,
                    row_stats, tie_alternatives)

STATUS_OK = "ok"
STATUS_POOL_EXHAUSTED = "pool_exhausted"
STATUS_PAGE_TABLE_FULL = "page_table_full"


def accept_resample(logits_cur, logits_prev, pending, n_pending, q_row,
                    seq_len, seed, step, N, tie_band=TIE_BAND,
                    proposal="sample", flip=()):
    """One accept / resample / bonus / draft step for every sequence.

    logits_cur  [B][K][V]  this forward pass's logits (fp64 copy)
    logits_prev [B][K][V]  the previous pass's logits (holds the q rows)
    pending     int [B][N] pending tokens (row 0 exact, rows 1.. drafts)
    n_pending   int [B]    1 or N
    q_row       int [B][N] row of logits_prev that drafted pending[b][i]
    seq_len     int [B]    committed length L_b
    proposal    "sample" (drafts drawn from q) or "argmax" (x = argmax q)
    flip        (b, i) pairs whose ratio test is decided the other way: the
                alternative branch of a near-tie ratio test, which a checker
                may need because two roundings can legitimately decide it
                either way

    Returns a dict of numpy arrays (padding -1 / NaN), ``ties``, a list of
    (b, kind, index) naming every near-tie decision, and ``tie_alts``,
    mapping (b, slot of next_pending) of every near-tie draw to the sorted
    tokens it may legitimately yield.  ``next_q_logz`` holds the natural-log
    normaliser ln sum_v exp(l_v) of each next draft's q row.
    """
    flip = set(flip)
    if proposal not in ("sample", "argmax"):
        raise ValueError(proposal)
    argmax = proposal == "argmax"
    B, K, V = logits_cur.shape
    out = {
        "accepted": np.zeros(B, dtype=np.int64),
        "rejected": np.zeros(B, dtype=bool),
        "n_commit": np.zeros(B, dtype=np.int64),
        "commit_tokens": np.full((B, N), -1, dtype=np.int64),
        "next_pending": np.full((B, N), -1, dtype=np.int64),
        "next_n": np.zeros(B, dtype=np.int64),
        "next_q_row": np.full((B, N), -1, dtype=np.int64),
        "next_q_logz": np.full((B, N), np.nan),
        "ratio": np.full((B, N), np.nan),
        "u_accept": np.full((B, N), np.nan),
        "exact_token": np.full(B, -1, dtype=np.int64),
    }
    ties = []
    tie_alts = {}
    for b in range(B):
        n = int(n_pending[b])
        L = int(seq_len[b])
        lc = logits_cur[b]
        # Verification of drafts 1 .. n - 1 in order.
        a = 0
        rejected = False
        for i in range(1, n):
            x = int(pending[b][i])
            m_p, s_p = row_stats(lc[i - 1])
            p_x = prob_of(lc[i - 1], x, m_p, s_p)
            if argmax:
                q_x = 1.0          # the proposal is a point mass at x
            else:
                q_src = logits_prev[b][int(q_row[b][i])]
                m_q, s_q = row_stats(q_src)
                q_x = prob_of(q_src, x, m_q, s_q)
            r = p_x / q_x
            u = philox.uniform(seed, b, step, L + i, philox.STREAM_ACCEPT)
            out["ratio"][b, i] = r
            out["u_accept"][b, i] = u
            if abs(u - r) < tie_band:
                ties.append((b, "accept", i))
            if (u < r) != ((b, i) in flip):
                a += 1
            else:
                rejected = True
                break
        out["accepted"][b] = a
        out["rejected"][b] = rejected
        out["n_commit"][b] = 1 + a
        out["commit_tokens"][b, 0:1 + a] = pending[b][0:1 + a]
        if rejected:
            p = probs(lc[a])
            if argmax:
                q = np.zeros(V)
                q[int(pending[b][a + 1])] = 1.0
            else:
                q = probs(logits_prev[b][int(q_row[b][a + 1])])
            w = np.maximum(0.0, p - q)
            if not np.sum(w) > 0.0:
                w = p
            u = philox.uniform(seed, b, step, L + a + 1,
                               philox.STREAM_RESAMPLE)
            tok, near = inverse_cdf(w, u, tie_band)
            if near:
                ties.append((b, "resample", 0))
                tie_alts[(b, 0)] = tie_alternatives(w, u, tie_band)
            out["next_pending"][b, 0] = tok
            out["next_n"][b] = 1
            out["exact_token"][b] = tok
        else:
            u = philox.uniform(seed, b, step, L + n, philox.STREAM_BONUS)
            tok, near = inverse_cdf(probs(lc[n - 1]), u, tie_band)
            if near:
                ties.append((b, "bonus", 0))
                tie_alts[(b, 0)] = tie_alternatives(probs(lc[n - 1]), u,
                                                    tie_band)
            out["next_pending"][b, 0] = tok
            out["exact_token"][b] = tok
            for j in range(1, N):
                row = n + j - 1
                if argmax:
                    xj = int(np.argmax(lc[row]))   # first maximal index
                else:
                    u = philox.uniform(seed, b, step, L + n + j,
                                       philox.STREAM_DRAFT)
                    xj, near = inverse_cdf(probs(lc[row]), u, tie_band)
                    if near:
                        ties.append((b, "draft", j))
                        tie_alts[(b, j)] = tie_alternatives(probs(lc[row]),
                                                            u, tie_band)
                out["next_pending"][b, j] = xj
                out["next_q_row"][b, j] = row
                out["next_q_logz"][b, j] = log_normaliser(lc[row])
            out["next_n"][b] = N
    out["ties"] = ties
    out["tie_alts"] = tie_alts
    return out


def pages_for(length, page_size):
    """Pages a sequence of ``length`` committed tokens owns."""
    return (length + page_size - 1) // page_size


def kv_commit(k_new, v_new, k_cache, v_cache, page_table, seq_len, n_commit,
              free_stack, free_top, page_size=16):
    """Commit the accepted prefix of every stride into the paged cache.

    Works on copies and returns (k_cache, v_cache, page_table, seq_len,
    free_top, status).  Pages are popped from the top of ``free_stack``
    (entries [0, free_top) are free, the top is free_stack[free_top - 1]),
    sequence 0 first.  The commit is all-or-nothing: if the pool or a
    page-table row is too small nothing changes and the status says why.
    """
    k_cache = k_cache.copy()
    v_cache = v_cache.copy()
    page_table = page_table.copy()
    seq_len = np.array(seq_len, dtype=np.int64).copy()
    B = len(seq_len)
    max_pages = page_table.shape[1]
    need = []
    for b in range(B):
        old = pages_for(int(seq_len[b]), page_size)
        new = pages_for(int(seq_len[b]) + int(n_commit[b]), page_size)
        if new > max_pages:
            return (k_cache, v_cache, page_table, seq_len, free_top,
                    STATUS_PAGE_TABLE_FULL)
        need.append(new - old)
    if sum(need) > free_top:
        return (k_cache, v_cache, page_table, seq_len, free_top,
                STATUS_POOL_EXHAUSTED)
    top = int(free_top)
    for b in range(B):
        old = pages_for(int(seq_len[b]), page_size)
        for k in range(need[b]):
            top -= 1
            page_table[b, old + k] = free_stack[top]
    Hkv = k_new.shape[2]
    for b in range(B):
        L = int(seq_len[b])
        for r in range(int(n_commit[b])):
            pos = L + r
            phys = int(page_table[b, pos // page_size])
            for h in range(Hkv):
                k_cache[phys, h, pos % page_size] = k_new[b, r, h]
                v_cache[phys, h, pos % page_size] = v_new[b, r, h]
        seq_len[b] = L + int(n_commit[b])
    return k_cache, v_cache, page_table, seq_len, top, STATUS_OK
