"""Helpers shared by the GPU parity tests.

Every expected value comes from ``oracle/`` run on the same seeded inputs
the CUDA path receives; nothing computed by the CUDA path is fed to the
oracle.  Inputs flow one way: synth -> (GPU, oracle).
"""

import math

import numpy as np
import torch

from introspective_strided_decoding_b200 import isd, synth
from oracle import attention as oattn
from oracle import step as ostep
from oracle.vocab import row_stats

TOL = {"bf16": 2e-2, "f32": 1e-5}


def f64(t):
    return t.detach().float().cpu().double().numpy()


def f32(t):
    return t.detach().float().cpu().numpy()


def i64(t):
    return t.detach().cpu().long().numpy()


# ---------------------------------------------------------------- attention
def gpu_attention(w, cache, q, k, v, num_ctas=0, lse=True, status=None):
    out = torch.empty_like(q)
    lse_t = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device) \
        if lse else None
    isd.attn_strided(q, k, v, cache["k_cache"], cache["v_cache"],
                     cache["page_table"], cache["seq_len"], out=out,
                     lse=lse_t, status=status,
                     softmax_scale=1.0 / math.sqrt(w.d), num_ctas=num_ctas)
    return out, lse_t


def oracle_attention(w, cache, q, k, v, pairs=None, page_table=None,
                     seq_len=None):
    """Oracle attention on host copies of the synth inputs."""
    pt = page_table if page_table is not None else i64(cache["page_table"])
    sl = seq_len if seq_len is not None else i64(cache["seq_len"])
    return oattn.attn_strided(f64(q), f64(k), f64(v), f64(cache["k_cache"]),
                              f64(cache["v_cache"]), pt, sl,
                              1.0 / math.sqrt(w.d), pairs=pairs)


def oracle_attention_pairs(w, cache, q, k, v, pairs, page_table, seq_len):
    """Oracle attention for a few (b, h) pairs: only the pages those pairs
    touch are copied to the host (as float32, exact for bf16)."""
    qh, kh, vh = f64(q), f64(k), f64(v)
    out = np.full(qh.shape, np.nan)
    lse = np.full(qh.shape[:3], np.nan)
    g = w.Hq // w.Hkv
    for b, h in pairs:
        L = int(seq_len[b])
        npg = (L + 15) // 16
        phys = torch.as_tensor(page_table[b, :npg], dtype=torch.long,
                               device=cache["k_cache"].device)
        sub_k = f64(cache["k_cache"][phys])
        sub_v = f64(cache["v_cache"][phys])
        pt = np.arange(npg)[None, :]
        o, l = oattn.attn_strided(qh[b:b + 1], kh[b:b + 1], vh[b:b + 1],
                                  sub_k, sub_v, pt, np.array([L]),
                                  1.0 / math.sqrt(w.d), pairs=[(0, h)])
        sl = slice(h * g, (h + 1) * g)
        out[b, :, sl] = o[0, :, sl]
        lse[b, :, sl] = l[0, :, sl]
    return out, lse


# ------------------------------------------------------------------ accept
def q_pair(logz):
    """The q_stats layout of a log-normaliser: fp32 hi and the fp32 rest."""
    logz = np.nan_to_num(np.asarray(logz, dtype=np.float64))
    hi = logz.astype(np.float32)
    lo = (logz - hi.astype(np.float64)).astype(np.float32)
    return np.stack([hi, lo], axis=-1)


def gpu_state_from(ostate, device):
    return dict(
        pending=torch.as_tensor(ostate["pending"], dtype=torch.int32,
                                device=device).contiguous(),
        n_pending=torch.as_tensor(ostate["n_pending"], dtype=torch.int32,
                                  device=device).contiguous(),
        q_row=torch.as_tensor(ostate["q_row"], dtype=torch.int32,
                              device=device).contiguous(),
        q_stats=torch.as_tensor(q_pair(ostate["q_logz"]),
                                dtype=torch.float32, device=device)
        .contiguous())


def oracle_initial_state(st):
    B, N = st["pending"].shape
    return dict(pending=i64(st["pending"]), n_pending=i64(st["n_pending"]),
                q_row=i64(st["q_row"]), q_logz=np.full((B, N), np.nan))


def next_oracle_state(ref):
    return dict(pending=ref["next_pending"], n_pending=ref["next_n"],
                q_row=ref["next_q_row"], q_logz=ref["next_q_logz"])


class AcceptStep:
    """GPU outputs of one isd_accept_resample call."""

    def __init__(self, B, N, K, device):
        self.state_out = isd.new_state(B, N, device)
        self.n_commit = torch.zeros(B, dtype=torch.int32, device=device)
        self.commit_tokens = torch.zeros((B, N), dtype=torch.int32,
                                         device=device)
        self.row_stats = torch.full((B, K, 2), float("nan"),
                                    dtype=torch.float32, device=device)
        self.ratio = torch.full((B, N), float("nan"), dtype=torch.float32,
                                device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)


def gpu_accept(lc, lp, seq_len, state_in, seed, step, proposal=None,
               vocab_stats=None):
    B, K, V = lc.shape
    N = K // 2
    o = AcceptStep(B, N, K, lc.device)
    isd.accept_resample(lc, lp, seq_len, state_in, o.state_out, o.n_commit,
                        o.commit_tokens, seed, step, row_stats=o.row_stats,
                        ratio=o.ratio, status=o.status, proposal=proposal,
                        vocab_stats=vocab_stats)
    return o


class _Host:
    """Host copies of a GPU accept step's outputs."""

    def __init__(self, o):
        self.nc = i64(o.n_commit)
        self.ct = i64(o.commit_tokens)
        self.pend = i64(o.state_out["pending"])
        self.n_out = i64(o.state_out["n_pending"])
        self.qr = i64(o.state_out["q_row"])
        qs = o.state_out["q_stats"].cpu().double().numpy()
        self.logz = qs[..., 0] + qs[..., 1]
        self.rs = o.row_stats.cpu().double().numpy()
        self.ratio = o.ratio.cpu().double().numpy()


def _branch_mismatch(g, r, b, N, tol_rel):
    """Why sequence b of the GPU outputs ``g`` differs from oracle branch
    ``r`` (None when it matches).  Draws that are near-ties in that branch
    must land on one of their legitimate tokens; everything else is exact
    (log-normalisers and ratios within ``tol_rel``)."""
    if g.nc[b] != r["n_commit"][b]:
        return f"n_commit {g.nc[b]} != {r['n_commit'][b]}"
    if not np.array_equal(g.ct[b], r["commit_tokens"][b]):
        return "commit_tokens"
    if g.n_out[b] != r["next_n"][b]:
        return "next n"
    if not np.array_equal(g.qr[b], r["next_q_row"][b]):
        return "next q rows"
    for j in range(N):
        alts = r["tie_alts"].get((b, j))
        if alts is not None:
            if g.pend[b, j] not in alts:
                return f"tie draw slot {j}: {g.pend[b, j]} not in {alts}"
        elif g.pend[b, j] != r["next_pending"][b, j]:
            return f"pending slot {j}: {g.pend[b, j]} != " \
                   f"{r['next_pending'][b, j]}"
    for j in range(1, N):
        if r["next_q_row"][b, j] >= 0:
            if abs(g.logz[b, j] - r["next_q_logz"][b, j]) > tol_rel:
                return f"q log-normaliser slot {j}"
    for i in range(1, N):
        if not np.isnan(r["ratio"][b, i]):
            if abs(g.ratio[b, i] - r["ratio"][b, i]) > \
                    tol_rel * r["ratio"][b, i]:
                return f"ratio of draft {i}"
    return None


def compare_accept(o, ref, n_in, rows_cur_f64, rerun, pending_in,
                   tol_rel=1e-5):
    """Compare GPU accept outputs with the oracle's, decision by decision.

    ``rerun(flip)`` re-runs the oracle on the same inputs with the ratio
    tests named in ``flip`` decided the other way; ``pending_in`` is the
    step's input pending tokens.

    * A sequence without a ratio-test near-tie must match the oracle
      exactly, except draws that are near-ties, whose token must be one of
      the oracle's legitimate alternatives (the oracle's index or the
      positive-mass index across the tied boundary).
    * A sequence with a ratio-test near-tie must match exactly one branch
      of the oracle (the tied tests decided either way, every combination),
      with the same draw allowance; and the GPU's own decisions must agree
      with the ratios it reports (accepted drafts have u <= ratio, a
      rejected one u >= ratio).

    Returns counters: sequence-steps compared exactly, near-ties, and
    near-ties on which the GPU chose differently from the oracle's primary
    branch.
    """
    B, N = ref["next_pending"].shape
    g = _Host(o)
    accept_ties = {}
    for b, kind, i in ref["ties"]:
        if kind == "accept":
            accept_ties.setdefault(b, []).append(i)
    out = dict(exact=0, ties=len(ref["ties"]), tie_differs=0)
    branches = {}
    for b in range(B):
        n = int(n_in[b])
        for r in range(n + N - 1):
            m_ref, s_ref = row_stats(rows_cur_f64(b, r))
            assert g.rs[b, r, 0] == m_ref, (b, r)
            assert abs(g.rs[b, r, 1] - s_ref) <= tol_rel * s_ref, (b, r)
        # The committed tokens are the step's own pending prefix.
        nc = int(g.nc[b])
        assert 1 <= nc <= n, (b, nc)
        assert np.array_equal(g.ct[b, :nc], pending_in[b, :nc]), b
        assert (g.ct[b, nc:] == -1).all(), b
        if b not in accept_ties:
            why = _branch_mismatch(g, ref, b, N, tol_rel)
            assert why is None, (b, why)
            for j in range(N):
                if (b, j) in ref["tie_alts"] and \
                        g.pend[b, j] != ref["next_pending"][b, j]:
                    out["tie_differs"] += 1
            out["exact"] += 1
            continue
        # Ratio-test near-tie: one of the oracle's branches.
        tied = accept_ties[b]
        matched = None
        whys = []
        for mask in range(1 << len(tied)):
            flip = frozenset((b, tied[k]) for k in range(len(tied))
                             if mask >> k & 1)
            if flip not in branches:
                branches[flip] = ref if not flip else rerun(flip)
            why = _branch_mismatch(g, branches[flip], b, N, tol_rel)
            if why is None:
                matched = branches[flip]
                break
            whys.append(why)
        assert matched is not None, (b, whys)
        for i in range(1, nc):
            assert matched["u_accept"][b, i] <= g.ratio[b, i], (b, i)
        if nc < n:
            assert matched["u_accept"][b, nc] >= g.ratio[b, nc], (b, nc)
        if matched is not ref:
            out["tie_differs"] += 1
    return out
