"""Pins for the oracle's paged strided attention (CPU only).

The oracle walks the page table page by page and appends the causal stride
rows.  These tests pin it to things other than itself: torch's
scaled_dot_product_attention (a library routine) on a dense layout
gathered by fancy indexing, closed-form special cases, page-permutation
invariance and causality.
"""

import math

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

from introspective_strided_decoding_b200 import synth
from oracle import attention


def _np(t):
    return t.detach().to(torch.float64).cpu().numpy()


def _inputs(w, seed, sharp=False, seq_len=None):
    c = synth.make_cache(w, seed, "cpu", seq_len=seq_len)
    q, k, v = synth.make_stride(w, seed, 0, "cpu", sharp=sharp)
    return dict(q=_np(q), k_new=_np(k), v_new=_np(v),
                k_cache=_np(c["k_cache"]), v_cache=_np(c["v_cache"]),
                page_table=c["page_table"].numpy(),
                seq_len=c["seq_len"].numpy())


def _run(x, scale):
    return attention.attn_strided(x["q"], x["k_new"], x["v_new"],
                                  x["k_cache"], x["v_cache"],
                                  x["page_table"], x["seq_len"], scale)


def _sdpa_reference(x, scale):
    """Dense gather by fancy indexing, then torch SDPA with a causal mask."""
    q = x["q"]
    B, K, Hq, d = q.shape
    Hkv = x["k_new"].shape[2]
    g = Hq // Hkv
    out = np.zeros_like(q)
    for b in range(B):
        L = int(x["seq_len"][b])
        t = np.arange(L)
        phys = x["page_table"][b][t // 16]
        kc = x["k_cache"][phys, :, t % 16]          # [L][Hkv][d]
        vc = x["v_cache"][phys, :, t % 16]
        keys = np.concatenate([kc, x["k_new"][b]], axis=0)   # [L+K][Hkv][d]
        vals = np.concatenate([vc, x["v_new"][b]], axis=0)
        kk = torch.from_numpy(np.repeat(keys.transpose(1, 0, 2), g, axis=0))
        vv = torch.from_numpy(np.repeat(vals.transpose(1, 0, 2), g, axis=0))
        qq = torch.from_numpy(q[b].transpose(1, 0, 2).copy())  # [Hq][K][d]
        allowed = (np.arange(L + K)[None, :] <= L + np.arange(K)[:, None])
        o = torch.nn.functional.scaled_dot_product_attention(
            qq, kk, vv, attn_mask=torch.from_numpy(allowed), scale=scale)
        out[b] = o.numpy().transpose(1, 0, 2)
    return out


CASES = [
    synth.TINY,
    synth.TINY.with_(B=3, Hq=8, Hkv=2, L_lo=0, L_hi=45, shuffle_pages=True),
    synth.TINY.with_(B=2, Hq=6, Hkv=3, d=32, N=3, L_lo=17, L_hi=33,
                     shuffle_pages=True),
]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name + str(w.B))
@pytest.mark.parametrize("sharp", [False, True])
def test_matches_library_attention(w, sharp):
    x = _inputs(w, 3, sharp=sharp)
    scale = 1.0 / math.sqrt(w.d)
    out, lse = _run(x, scale)
    ref = _sdpa_reference(x, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_lse_matches_logsumexp():
    w = CASES[1]
    x = _inputs(w, 5, sharp=True)
    scale = 1.0 / math.sqrt(w.d)
    _, lse = _run(x, scale)
    b, r, hq = 2, 1, 5
    h = hq // (w.Hq // w.Hkv)
    L = int(x["seq_len"][b])
    t = np.arange(L)
    phys = x["page_table"][b][t // 16]
    keys = np.concatenate([x["k_cache"][phys, h, t % 16],
                           x["k_new"][b, :r + 1, h]])
    s = scale * keys @ x["q"][b, r, hq]
    assert lse[b, r, hq] == pytest.approx(logsumexp(s), rel=1e-13)


def test_empty_prefix_first_row_is_v0():
    w = synth.TINY.with_(B=2, L_lo=0, L_hi=0)
    x = _inputs(w, 1, sharp=True)
    out, lse = _run(x, 0.125)
    for b in range(2):
        for hq in range(w.Hq):
            np.testing.assert_allclose(out[b, 0, hq], x["v_new"][b, 0, 0],
                                       rtol=0, atol=1e-15)
            s0 = 0.125 * x["k_new"][b, 0, 0] @ x["q"][b, 0, hq]
            assert lse[b, 0, hq] == pytest.approx(s0, rel=1e-14)


def test_equal_keys_give_mean_of_visible_values():
    w = synth.TINY.with_(B=1, L_lo=37, L_hi=37, shuffle_pages=True)
    x = _inputs(w, 2)
    x["k_cache"][:] = 0.3
    x["k_new"][:] = 0.3
    out, _ = _run(x, 0.125)
    L = 37
    t = np.arange(L)
    phys = x["page_table"][0][t // 16]
    vis = x["v_cache"][phys, 0, t % 16]
    for r in range(w.K):
        allv = np.concatenate([vis, x["v_new"][0, :r + 1, 0]])
        for hq in range(w.Hq):
            np.testing.assert_allclose(out[0, r, hq], allv.mean(axis=0),
                                       rtol=1e-12, atol=1e-13)


def test_one_hot_score_selects_that_value():
    w = synth.TINY.with_(B=1, L_lo=40, L_hi=40, shuffle_pages=True)
    x = _inputs(w, 4)
    x["k_cache"][:] = 0.0
    x["k_new"][:] = 0.0
    target = 23
    phys = x["page_table"][0][target // 16]
    x["k_cache"][phys, 0, target % 16] = 1.0
    x["q"][:] = 1.0
    out, _ = _run(x, 100.0)   # score 6400 on one key, 0 elsewhere
    for r in range(w.K):
        for hq in range(w.Hq):
            np.testing.assert_allclose(out[0, r, hq],
                                       x["v_cache"][phys, 0, target % 16],
                                       rtol=0, atol=1e-12)


def test_page_permutation_invariance():
    w = synth.TINY.with_(B=2, Hq=4, Hkv=2, L_lo=50, L_hi=70)
    x = _inputs(w, 6, sharp=True)
    out, lse = _run(x, 0.125)
    # Move every owned page to a new physical slot in a bigger pool.
    P = x["k_cache"].shape[0]
    perm = np.random.default_rng(0).permutation(2 * P)
    kc = np.zeros((2 * P,) + x["k_cache"].shape[1:])
    vc = np.zeros_like(kc)
    kc[perm[:P]] = x["k_cache"]
    vc[perm[:P]] = x["v_cache"]
    pt = np.where(x["page_table"] >= 0, perm[np.maximum(x["page_table"], 0)],
                  -1)
    y = dict(x, k_cache=kc, v_cache=vc, page_table=pt)
    out2, lse2 = _run(y, 0.125)
    assert np.array_equal(out, out2) and np.array_equal(lse, lse2)


def test_causal_inside_the_stride():
    w = synth.TINY.with_(B=1, N=3, L_lo=20, L_hi=20)
    x = _inputs(w, 8, sharp=True)
    out, _ = _run(x, 0.125)
    r = 2
    y = {k: v.copy() for k, v in x.items()}
    y["k_new"][0, r + 1:] += 5.0
    y["v_new"][0, r + 1:] -= 7.0
    y["q"][0, r + 1:] *= -1.0
    out2, _ = _run(y, 0.125)
    assert np.array_equal(out[0, :r + 1], out2[0, :r + 1])
    assert not np.allclose(out[0, r + 1:], out2[0, r + 1:])
