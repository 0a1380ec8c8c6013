"""isd_accept_resample_static: the accept / resample step for callers that
cannot allocate device memory (a program linking the C ABI without a
device allocator of its own, or a process whose framework has already
reserved the memory pool).  Its scratch lives in a fixed buffer inside the
library instead of a caller workspace.

The test drives it through the C ABI and checks that two calls in a row
(an R-mode step, then an S-mode step that verifies real drafts, so the
buffer already holds the first call's contents) give exactly the outputs
of isd_accept_resample with a caller workspace.  The file sorts last so a
run that stops at the first failure has run every other test first.
"""

import pytest
import torch

from introspective_strided_decoding_b200 import build, isd, synth
from tests.gpu_util import AcceptStep

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _call(which, lc, lp, L, state, seed, step):
    B, K, _ = lc.shape
    o = AcceptStep(B, K // 2, K, lc.device)
    if which == "workspace":
        isd.accept_resample(lc, lp, L, state, o.state_out, o.n_commit,
                            o.commit_tokens, seed, step,
                            row_stats=o.row_stats, ratio=o.ratio,
                            status=o.status)
    else:
        isd.accept_resample_static(lc, lp, L, state, o.state_out, o.n_commit,
                                   o.commit_tokens, seed, step,
                                   row_stats=o.row_stats, ratio=o.ratio,
                                   status=o.status)
    return o


def _same(a, b):
    return torch.equal(a.nan_to_num(), b.nan_to_num())


def test_static_scratch_matches_workspace_entry_point():
    build.build()
    w = synth.Workload("no_alloc", B=16, Hq=32, Hkv=8, d=128, N=4, L_lo=100,
                       L_hi=900, V=151936, target_accept=0.7)
    seed = 9
    state = synth.initial_state(w, seed, DEV)
    L = synth.prefix_lengths(w, seed).to(DEV)
    lp = torch.zeros((w.B, w.K, w.V), dtype=w.torch_dtype, device=DEV)
    for step in range(2):
        lc = synth.step_logits(w, seed, L, state["n_pending"], step, DEV)
        ref = _call("workspace", lc, lp, L, state, seed, step)
        got = _call("static", lc, lp, L, state, seed, step)
        torch.cuda.synchronize()
        assert int(ref.status.item()) == isd.OK
        assert int(got.status.item()) == isd.OK
        assert _same(got.n_commit, ref.n_commit)
        assert _same(got.commit_tokens, ref.commit_tokens)
        for key in isd.STATE_KEYS:
            assert _same(got.state_out[key], ref.state_out[key]), key
        assert _same(got.row_stats, ref.row_stats)
        assert _same(got.ratio, ref.ratio)
        if step == 1:
            # The second step verified drafts (S mode) for most sequences.
            assert int((state["n_pending"] == w.N).sum()) > w.B // 2
        state, lp = ref.state_out, lc
        L = L + ref.n_commit
