"""isd_accept_commit returns exactly what isd_accept_resample followed by
isd_kv_commit returns: every output of the accept step, the next decoding
state, the KV cache bytes, the page tables, the lengths, the free-stack top
and the status word, step after step (its parity with the oracle follows
from that of the two calls; the free-running decoder and graph tests also
run it against the oracle)."""

import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from introspective_strided_decoding_b200.driver import Decoder

pytestmark = pytest.mark.gpu
DEV = torch.device("cuda", 0)

OUTS = ("n_commit", "commit_tokens")


def _run(w, seed, steps, fused, proposal=isd.PROPOSAL_SAMPLE, pool=None):
    cache = synth.make_cache(w, seed, DEV)
    if pool is not None:
        cache["free_top"].fill_(pool)        # too few free pages
    dec = Decoder(w, cache, synth.initial_state(w, seed, DEV), DEV, seed,
                  proposal=proposal)
    rec = []
    for s in range(steps):
        dec.logits_cur.copy_(synth.step_logits(w, seed, cache["seq_len"],
                                               dec.state["n_pending"], s, DEV))
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        dec.attention()
        if fused:
            dec.accept_commit()
        else:
            dec.accept()
            dec.commit()
        torch.cuda.synchronize()
        out = {key: getattr(dec, key).clone() for key in OUTS}
        out.update({f"state_{key}": t.clone()
                    for key, t in dec.states[1 - dec.cur].items()})
        out.update({f"cache_{key}": t.clone() for key, t in cache.items()})
        out["status"] = dec.status.clone()
        rec.append(out)
        dec.advance()
    return rec


def _assert_same(a, b):
    for s, (x, y) in enumerate(zip(a, b)):
        for key in x:
            assert torch.equal(x[key], y[key]), (s, key)


@pytest.mark.parametrize("w,proposal", [
    (synth.C64.with_(B=16, steps=6), isd.PROPOSAL_SAMPLE),
    (synth.sweep_workload(8, 8, 0.5).with_(steps=6), isd.PROPOSAL_SAMPLE),
    (synth.sweep_workload(1, 4, 0.9).with_(steps=6), isd.PROPOSAL_SAMPLE),
    (synth.C64.with_(B=8, steps=6), isd.PROPOSAL_ARGMAX),
    (synth.TINY.with_(B=3, steps=6), isd.PROPOSAL_SAMPLE),
], ids=["c64_b16", "b8_n8_p05", "b1_n4", "argmax_b8", "tiny_f32"])
def test_fused_equals_separate_calls(w, proposal):
    seed = 11
    _assert_same(_run(w, seed, w.steps, True, proposal),
                 _run(w, seed, w.steps, False, proposal))


def test_fused_equals_separate_calls_at_full_size():
    w = synth.C64.with_(steps=3)
    _assert_same(_run(w, 4, 3, True), _run(w, 4, 3, False))


def test_fused_failed_commit_writes_nothing_like_the_separate_call():
    """A pool too small for the commit: the same status, no cache byte,
    page, length or top changed, in both forms; the draws still run."""
    w = synth.C64.with_(B=8, steps=6)
    fused = _run(w, 6, 6, True, pool=0)
    _assert_same(fused, _run(w, 6, 6, False, pool=0))
    # The status word keeps the first error: some step needed a new page.
    assert int(fused[-1]["status"].item()) == isd.ERR_POOL_EXHAUSTED
    assert torch.equal(fused[-1]["cache_free_top"], fused[0]["cache_free_top"])
