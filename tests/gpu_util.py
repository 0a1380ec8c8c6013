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
def gpu_state_from(ostate, device):
    return dict(
        pending=torch.as_tensor(ostate["pending"], dtype=torch.int32,
                                device=device).contiguous(),
        n_pending=torch.as_tensor(ostate["n_pending"], dtype=torch.int32,
                                  device=device).contiguous(),
        q_row=torch.as_tensor(ostate["q_row"], dtype=torch.int32,
                              device=device).contiguous(),
        q_stats=torch.as_tensor(np.nan_to_num(ostate["q_stats"]),
                                dtype=torch.float32, device=device)
        .contiguous())


def oracle_initial_state(st):
    return dict(pending=i64(st["pending"]), n_pending=i64(st["n_pending"]),
                q_row=i64(st["q_row"]),
                q_stats=st["q_stats"].detach().cpu().double().numpy())


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


def gpu_accept(lc, lp, seq_len, state_in, seed, step, proposal=None):
    B, K, V = lc.shape
    N = K // 2
    o = AcceptStep(B, N, K, lc.device)
    isd.accept_resample(lc, lp, seq_len, state_in, o.state_out, o.n_commit,
                        o.commit_tokens, seed, step, row_stats=o.row_stats,
                        ratio=o.ratio, status=o.status, proposal=proposal)
    return o


def compare_accept(o, ref, n_in, rows_cur_f64, tol_rel=1e-5):
    """Compare GPU accept outputs with the oracle's.

    Near-ties (``ref["ties"]``) are handled per decision: a near-tie in a
    ratio test leaves that sequence checked for validity only; a near-tie in
    a draw leaves only that drawn token checked for validity.  Everything
    else must match exactly (statistics and ratios within ``tol_rel``).
    Returns counters: decisions compared exactly, near-ties, and near-ties
    on which the GPU chose differently.
    """
    B, N = ref["next_pending"].shape
    accept_tie = {b for b, kind, _ in ref["ties"] if kind == "accept"}
    slot_tie = {(b, 0 if kind in ("bonus", "resample") else j)
                for b, kind, j in ref["ties"] if kind != "accept"}
    nc = i64(o.n_commit)
    ct = i64(o.commit_tokens)
    pend = i64(o.state_out["pending"])
    n_out = i64(o.state_out["n_pending"])
    qr = i64(o.state_out["q_row"])
    qs = o.state_out["q_stats"].cpu().double().numpy()
    rs = o.row_stats.cpu().double().numpy()
    ratio = o.ratio.cpu().double().numpy()
    out = dict(exact=0, ties=len(ref["ties"]), tie_differs=0)
    for b in range(B):
        n = int(n_in[b])
        for r in range(n + N - 1):
            m_ref, s_ref = row_stats(rows_cur_f64(b, r))
            assert rs[b, r, 0] == m_ref, (b, r)
            assert abs(rs[b, r, 1] - s_ref) <= tol_rel * s_ref, (b, r)
        if b in accept_tie:
            assert 1 <= nc[b] <= n
            if nc[b] != ref["n_commit"][b]:
                out["tie_differs"] += 1
            continue
        for i in range(1, n):
            if not np.isnan(ref["ratio"][b, i]):
                assert abs(ratio[b, i] - ref["ratio"][b, i]) <= \
                    tol_rel * ref["ratio"][b, i], (b, i)
        assert nc[b] == ref["n_commit"][b], b
        assert np.array_equal(ct[b], ref["commit_tokens"][b]), b
        assert n_out[b] == ref["next_n"][b], b
        assert np.array_equal(qr[b], ref["next_q_row"][b]), b
        for j in range(N):
            if (b, j) in slot_tie:
                assert ref["next_pending"][b, j] < 0 or pend[b, j] >= 0
                if pend[b, j] != ref["next_pending"][b, j]:
                    out["tie_differs"] += 1
                continue
            assert pend[b, j] == ref["next_pending"][b, j], (b, j)
        for j in range(1, N):
            if ref["next_q_row"][b, j] >= 0:
                assert qs[b, j, 0] == ref["next_q_stats"][b, j, 0]
                assert abs(qs[b, j, 1] - ref["next_q_stats"][b, j, 1]) <= \
                    tol_rel * ref["next_q_stats"][b, j, 1]
        out["exact"] += 1
    return out
