"""A captured CUDA graph of the step replays exactly what the eager calls
compute (same commits, tokens, pages and cache bytes, step after step),
and free-running replays agree with the oracle at every step."""

import numpy as np
import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from introspective_strided_decoding_b200.driver import Decoder
from oracle import step as ostep
from tests.gpu_util import compare_accept, f32, i64, oracle_initial_state

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(w, seed, steps, graphs):
    cache = synth.make_cache(w, seed, DEV)
    dec = Decoder(w, cache, synth.initial_state(w, seed, DEV), DEV, seed)
    if graphs:
        dec.capture()
    hist = []
    for s in range(steps):
        dec.logits_cur.copy_(synth.step_logits(w, seed, cache["seq_len"],
                                               dec.state["n_pending"], s,
                                               DEV))
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        if graphs:
            dec.replay()
        else:
            dec.step()
        hist.append((dec.n_commit.clone(), dec.state["pending"].clone(),
                     dec.out.clone()))
    torch.cuda.synchronize()
    assert int(dec.status.item()) == isd.OK
    return hist, cache


def test_graph_replay_matches_eager():
    w = synth.C64.with_(B=16, steps=10)
    h1, c1 = _run(w, 4, 8, graphs=False)
    h2, c2 = _run(w, 4, 8, graphs=True)
    for (a1, b1, o1), (a2, b2, o2) in zip(h1, h2):
        assert torch.equal(a1, a2) and torch.equal(b1, b2)
        assert torch.equal(o1, o2)
    for key in c1:
        assert torch.equal(c1[key], c2[key]), key


class _View:
    """compare_accept's view of the step the decoder has just replayed."""

    def __init__(self, dec):
        self.n_commit = dec.n_commit
        self.commit_tokens = dec.commit_tokens
        self.state_out = dec.state           # already swapped in
        self.row_stats = dec.row_stats
        self.ratio = dec.ratio


@pytest.mark.parametrize("peaked", [False, True])
def test_graph_replay_free_running_matches_oracle(peaked):
    """Free-running CUDA-graph replays, each step checked against the
    oracle started from the state the GPU itself carried into the step:
    decisions, tokens, next state and the commit's page table, lengths and
    free-stack top.  Near-ties are checked for validity and the run then
    follows the GPU's branch."""
    w = synth.C64.with_(B=16, steps=12)
    if peaked:
        w = w.with_(peak=18.6)   # max p about 0.9 at sigma_p 3, V 151 936
    seed = 9
    cache = synth.make_cache(w, seed, DEV)
    dec = Decoder(w, cache, synth.initial_state(w, seed, DEV), DEV, seed,
                  record=True)
    dec.capture()
    lp_host = np.zeros((w.B, w.K, w.V), dtype=np.float32)
    dummy = np.zeros((cache["k_cache"].shape[0], 1, 16, 1))
    fs = i64(cache["free_stack"])
    exact = ties = 0
    for s in range(w.steps):
        st = dec.state
        ostate = oracle_initial_state(st)
        L = i64(cache["seq_len"])
        pt = i64(cache["page_table"])
        top = int(cache["free_top"].item())
        lc = synth.step_logits(w, seed, cache["seq_len"], st["n_pending"], s,
                               DEV)
        dec.logits_cur.copy_(lc)
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        dec.replay()
        torch.cuda.synchronize()
        assert int(dec.status.item()) == isd.OK
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
        exact += c["exact"]
        ties += c["ties"]
        # The commit of the GPU's own (validated) counts.
        nc = i64(dec.n_commit)
        _, _, pt_ref, L_ref, top_ref, rst = ostep.kv_commit(
            np.zeros((w.B, w.K, 1, 1)), np.zeros((w.B, w.K, 1, 1)), dummy,
            dummy, pt, L, nc, fs, top)
        assert rst == ostep.STATUS_OK
        assert np.array_equal(i64(cache["page_table"]), pt_ref), s
        assert np.array_equal(i64(cache["seq_len"]), L_ref), s
        assert int(cache["free_top"].item()) == top_ref, s
        lp_host = lc_host
    dec.release_graphs()
    print(f"graph free run: {exact} sequence-steps exact, {ties} near-ties")
    assert exact >= 0.9 * w.B * w.steps


def _snap(dec, cache):
    st = {k: v.clone() for k, v in dec.state.items()}
    return dict(st, **{k: cache[k].clone() for k in
                       ("seq_len", "page_table", "free_top", "k_cache",
                        "v_cache")})


@pytest.mark.parametrize("with_lm", [False, True])
def test_multi_step_graph_matches_single_steps(with_lm):
    """S = 4 steps per graph replay, two replays, against eight eager steps
    on the same inputs: the state, lengths, page table, free-stack top and
    cache bytes agree bit for bit after every replay."""
    S, R = 4, 2
    if with_lm:
        w = synth.Workload("multi_lm", B=8, Hq=32, Hkv=8, d=128, N=4,
                           L_lo=100, L_hi=400, V=8200, sigma_p=3.0,
                           sigma_q=0.25, D=256, steps=S * R)
    else:
        w = synth.C64.with_(name="multi_logits", B=8, steps=S * R)
    seed = 17
    lm = None
    if with_lm:
        lm = dict(weight=synth.lm_weight(seed, w.V, w.D, DEV)
                  .to(torch.bfloat16).contiguous())

    def fresh():
        cache = synth.make_cache(w, seed, DEV)
        dec = Decoder(w, cache, synth.initial_state(w, seed, DEV), DEV, seed,
                      lm=lm)
        return dec, cache

    # Eager reference, recording each step's inputs.
    dec, cache = fresh()
    inputs, snaps = [], []
    for s in range(S * R):
        st = dec.state
        if with_lm:
            first = synth.step_hidden(w, seed, cache["seq_len"],
                                      st["n_pending"], s, DEV)
            dec.hidden.copy_(first)
        else:
            first = synth.step_logits(w, seed, cache["seq_len"],
                                      st["n_pending"], s, DEV)
            dec.logits_cur.copy_(first)
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        inputs.append((first, q, k, v))
        dec.step()
        if s % S == S - 1:
            snaps.append(_snap(dec, cache))
    torch.cuda.synchronize()
    assert int(dec.status.item()) == isd.OK

    # One graph of S steps, replayed R times.
    dec2, cache2 = fresh()
    dec2.capture_multi(S)
    for r in range(R):
        for i in range(S):
            first, q, k, v = inputs[r * S + i]
            dec2.slots["first"][i].copy_(first)
            dec2.slots["q"][i].copy_(q)
            dec2.slots["k_new"][i].copy_(k)
            dec2.slots["v_new"][i].copy_(v)
        dec2.replay_multi()
        torch.cuda.synchronize()
        assert int(dec2.status.item()) == isd.OK
        got = _snap(dec2, cache2)
        for key, ref in snaps[r].items():
            assert torch.equal(got[key], ref), (r, key)
    dec2.release_graphs()
