"""A captured CUDA graph of the step replays exactly what the eager calls
compute: same commits, tokens, pages and cache bytes, step after step."""

import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from introspective_strided_decoding_b200.driver import Decoder

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
