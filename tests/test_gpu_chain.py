"""The C=64 stationary batch over 100 consecutive steps, in lockstep with
the oracle, plus determinism and the tokens-per-forward check.

Lockstep: at every step the GPU starts from the oracle's decoding state
(pending tokens, modes, q rows and statistics, lengths, page table, free
stack top) and the same seeded logits and stride K/V.  Accepted counts,
tokens and page tables must match bit for bit (near-tie sequences are
reported and only checked for validity; the oracle's commit counts then
drive both commits so later steps stay comparable).  Attention is
compared at sampled steps on sampled (b, h) pairs against the oracle run on
the cache content the oracle itself reconstructs from the inputs.
"""

import math

import numpy as np
import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from introspective_strided_decoding_b200.driver import Decoder
from oracle import attention as oattn
from oracle import step as ostep
from oracle import tpf
from tests.gpu_util import (TOL, compare_accept, f32, f64, gpu_state_from, i64,
                            next_oracle_state, oracle_initial_state)

pytestmark = pytest.mark.gpu
DEV = "cuda"


class _View:
    """Adapter giving compare_accept the decoder's outputs."""

    def __init__(self, dec):
        self.n_commit = dec.n_commit
        self.commit_tokens = dec.commit_tokens
        self.state_out = dec.states[1 - dec.cur]
        self.row_stats = dec.row_stats
        self.ratio = dec.ratio


def _logical_prefix(cache, b, L):
    """Host copy of the committed K/V of sequence b (input data)."""
    npg = (L + 15) // 16
    phys = cache["page_table"][b, :npg].long()
    k = cache["k_cache"][phys].float().cpu().numpy()     # [npg][Hkv][16][d]
    v = cache["v_cache"][phys].float().cpu().numpy()
    k = k.transpose(0, 2, 1, 3).reshape(npg * 16, k.shape[1], k.shape[3])[:L]
    v = v.transpose(0, 2, 1, 3).reshape(npg * 16, v.shape[1], v.shape[3])[:L]
    return [k.astype(np.float64), v.astype(np.float64)]


def _oracle_attn_logical(w, kv, q, k, v, b, h):
    """Oracle attention of pair (b, h) over a logical prefix laid out in
    identity-mapped pages."""
    Kp, Vp = kv
    L = Kp.shape[0]
    npg = max(1, (L + 15) // 16)
    kc = np.zeros((npg, w.Hkv, 16, w.d))
    vc = np.zeros_like(kc)
    for t in range(L):
        kc[t // 16, :, t % 16] = Kp[t]
        vc[t // 16, :, t % 16] = Vp[t]
    pt = np.arange(npg)[None, :]
    return oattn.attn_strided(q[b:b + 1], k[b:b + 1], v[b:b + 1], kc, vc, pt,
                              np.array([L]), 1.0 / math.sqrt(w.d),
                              pairs=[(0, h)])


def test_c64_stationary_lockstep_100_steps():
    w = synth.C64
    steps = w.steps
    seed = 5
    cache = synth.make_cache(w, seed, DEV)
    st0 = synth.initial_state(w, seed, DEV)
    dec = Decoder(w, cache, st0, DEV, seed, record=True)
    ostate = oracle_initial_state(st0)
    L = i64(cache["seq_len"])
    pt = i64(cache["page_table"])
    fs = i64(cache["free_stack"])
    top = int(cache["free_top"].item())
    sampled = [0, 31, 63]
    logical = {b: _logical_prefix(cache, b, int(L[b])) for b in sampled}
    attn_steps = {0, 1, 2, 50, 99}
    lp_host = np.zeros((w.B, w.K, w.V), dtype=np.float32)
    dummy = np.zeros((cache["k_cache"].shape[0], 1, 16, 1))
    ties = compared = differs = 0
    for s in range(steps):
        L_dev = torch.as_tensor(L, dtype=torch.int32, device=DEV)
        lc = synth.step_logits(w, seed, L_dev,
                               torch.as_tensor(ostate["n_pending"],
                                               device=DEV), s, DEV)
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.logits_cur.copy_(lc)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        # Lockstep: the GPU starts from the oracle's state.
        for key, t in gpu_state_from(ostate, DEV).items():
            dec.state[key].copy_(t)
        cache["seq_len"].copy_(L_dev)
        cache["page_table"].copy_(torch.as_tensor(pt, dtype=torch.int32))
        cache["free_top"].fill_(top)
        dec.step_idx = s
        dec.attention()
        dec.accept()
        torch.cuda.synchronize()
        lc_host = f32(lc)
        def oracle(flip=(), lc_host=lc_host, lp_host=lp_host,
                   ostate=ostate, L=L, s=s):
            return ostep.accept_resample(lc_host, lp_host, ostate["pending"],
                                         ostate["n_pending"], ostate["q_row"],
                                         L, seed, s, w.N, flip=flip)
        ref = oracle()
        c = compare_accept(_View(dec), ref, ostate["n_pending"],
                           lambda b, r: lc_host[b, r].astype(np.float64),
                           oracle, ostate["pending"])
        compared += c["exact"]
        ties += c["ties"]
        differs += c["tie_differs"]
        if s in attn_steps:
            qh, kh, vh = f64(q), f64(k), f64(v)
            out = f64(dec.out)
            for b in sampled:
                for h in (0, w.Hkv - 1):
                    o_ref, _ = _oracle_attn_logical(w, logical[b], qh, kh, vh,
                                                    b, h)
                    g = w.g
                    sl = slice(h * g, (h + 1) * g)
                    err = np.abs(out[b, :, sl] - o_ref[0, :, sl]).max()
                    assert err <= TOL["bf16"], (s, b, h, err)
        # Both commits use the oracle's counts.
        nc = ref["n_commit"]
        dec.n_commit.copy_(torch.as_tensor(nc, dtype=torch.int32))
        dec.commit()
        _, _, pt, L_new, top, rst = ostep.kv_commit(
            np.zeros((w.B, w.K, 1, 1)), np.zeros((w.B, w.K, 1, 1)), dummy,
            dummy, pt, L, nc, fs, top)
        assert rst == ostep.STATUS_OK
        torch.cuda.synchronize()
        assert int(dec.status.item()) == isd.OK
        assert np.array_equal(i64(cache["page_table"]), pt), s
        assert np.array_equal(i64(cache["seq_len"]), L_new), s
        assert int(cache["free_top"].item()) == top, s
        kh_host, vh_host = f64(k), f64(v)
        for b in sampled:
            logical[b][0] = np.concatenate([logical[b][0],
                                            kh_host[b, :nc[b]]])
            logical[b][1] = np.concatenate([logical[b][1],
                                            vh_host[b, :nc[b]]])
        dec.advance()
        ostate = next_oracle_state(ref)
        L = L_new
        lp_host = lc_host
    print(f"lockstep: {compared} sequence-steps exact, {ties} near-ties, "
          f"{differs} of them decided differently")
    assert compared >= 0.98 * w.B * steps


def _free_run(w, seed, steps):
    cache = synth.make_cache(w, seed, DEV)
    st0 = synth.initial_state(w, seed, DEV)
    dec = Decoder(w, cache, st0, DEV, seed)
    counts, tested, accepted = [], 0, 0
    for s in range(steps):
        dec.logits_cur.copy_(synth.step_logits(w, seed, cache["seq_len"],
                                               dec.state["n_pending"], s,
                                               DEV))
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        n_in = dec.state["n_pending"].clone()
        dec.step()
        counts.append(dec.n_commit.clone())
        # Drafts tested: the accepted ones plus the first rejected one.
        acc = dec.n_commit - 1
        rej = (dec.n_commit < n_in).to(torch.int64)
        tested += int(acc.sum() + rej.sum())
        accepted += int(acc.sum())
    torch.cuda.synchronize()
    assert int(dec.status.item()) == isd.OK
    return torch.stack(counts), cache, tested, accepted


def test_free_running_is_deterministic():
    w = synth.C64.with_(B=16, steps=20)
    c1, cache1, _, _ = _free_run(w, 3, 20)
    c2, cache2, _, _ = _free_run(w, 3, 20)
    assert torch.equal(c1, c2)
    for key in cache1:
        assert torch.equal(cache1[key], cache2[key]), key


@pytest.mark.parametrize("B,N,target", [(64, 4, 0.9), (32, 2, 0.5),
                                        (8, 8, 0.9), (64, 8, 0.5),
                                        (1, 4, 0.9)])
def test_tokens_per_forward_matches_chain(B, N, target):
    """Measured tokens per forward against the exact finite-horizon value
    of the pages' TPF chain at the measured per-draft acceptance."""
    T = 40
    w = synth.sweep_workload(B, N, target).with_(L_lo=512, L_hi=2048,
                                                  steps=T)
    counts, _, tested, accepted = _free_run(w, 11, T)
    alpha = accepted / tested
    print(f"B={B} N={N} target={target}: acceptance {alpha:.4f}, "
          f"TPF {counts.double().mean().item():.4f}")
    assert abs(alpha - target) < 0.03 + 3 * math.sqrt(target * (1 - target)
                                                     / tested)
    per_seq = counts.sum(0).double().cpu().numpy()
    expect = tpf.expected_tokens(alpha, N, T)
    if B > 1:
        se = per_seq.std(ddof=1) / math.sqrt(B)
        assert abs(per_seq.mean() - expect) < 4.5 * se + 0.02 * expect
    else:
        assert abs(per_seq.mean() - expect) < 0.35 * expect
