"""GPU parity of isd_kv_commit against the oracle: page tables, lengths,
the free-stack top and the cache bytes must be bit-exact."""

import numpy as np
import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from oracle import step as ostep
from tests.gpu_util import i64

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(w, seed, spare=4):
    w = w.with_(spare_pages=spare)
    cache = synth.make_cache(w, seed, DEV)
    _, k, v = synth.make_stride(w, seed, 0, DEV, sharp=True)
    g = torch.Generator().manual_seed(seed)
    nc = torch.randint(0, w.N + 1, (w.B,), generator=g).to(torch.int32)
    return cache, k, v, nc.to(DEV)


def _host(t):
    return t.detach().cpu().float().numpy() if t.is_floating_point() \
        else i64(t)


def _run_both(w, cache, k, v, nc):
    ref = ostep.kv_commit(_host(k), _host(v), _host(cache["k_cache"]),
                          _host(cache["v_cache"]), i64(cache["page_table"]),
                          i64(cache["seq_len"]), i64(nc),
                          i64(cache["free_stack"]),
                          int(cache["free_top"].item()))
    status = torch.zeros((1,), dtype=torch.int32, device=DEV)
    ws = torch.zeros(256, dtype=torch.uint8, device=DEV)
    isd.kv_commit(k, v, cache["k_cache"], cache["v_cache"],
                  cache["page_table"], cache["seq_len"], nc,
                  cache["free_stack"], cache["free_top"], status, workspace=ws)
    torch.cuda.synchronize()
    # The workspace counter is back at zero after every call.
    assert int(ws.count_nonzero().item()) == 0
    return ref, int(status.item())


WS = [
    synth.Workload("c_bf16", B=7, Hq=32, Hkv=8, d=128, N=4, L_lo=0, L_hi=70,
                   V=16),
    synth.Workload("c_bf16_n8", B=5, Hq=64, Hkv=8, d=128, N=8, L_lo=10,
                   L_hi=50, V=16),
    synth.Workload("c_f32", B=4, Hq=4, Hkv=1, d=64, N=2, L_lo=14, L_hi=18,
                   V=16, dtype="f32"),
    synth.Workload("c_b64_long", B=64, Hq=32, Hkv=8, d=128, N=4, L_lo=100,
                   L_hi=400, V=16),
    # More sequences than CTAs (1024): two sequences per CTA.
    synth.Workload("c_b1500_f32", B=1500, Hq=4, Hkv=1, d=64, N=2, L_lo=0,
                   L_hi=40, V=16, dtype="f32"),
]


@pytest.mark.parametrize("w", WS, ids=lambda w: w.name)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_commit_bit_exact(w, seed):
    cache, k, v, nc = _case(w, seed)
    ref, st = _run_both(w, cache, k, v, nc)
    kc, vc, pt, sl, top, rst = ref
    assert rst == ostep.STATUS_OK and st == isd.OK
    assert np.array_equal(i64(cache["page_table"]), pt)
    assert np.array_equal(i64(cache["seq_len"]), sl)
    assert int(cache["free_top"].item()) == top
    assert np.array_equal(_host(cache["k_cache"]), kc)
    assert np.array_equal(_host(cache["v_cache"]), vc)


def test_pool_exhausted_changes_nothing():
    w = synth.Workload("ex", B=6, Hq=32, Hkv=8, d=128, N=4, L_lo=15, L_hi=15,
                       V=16, shuffle_pages=True)
    cache, k, v, _ = _case(w, 3, spare=0)
    nc = torch.full((w.B,), 2, dtype=torch.int32, device=DEV)
    cache["free_top"].fill_(3)             # six sequences cross a page
    before = {key: t.clone() for key, t in cache.items()}
    ref, st = _run_both(w, cache, k, v, nc)
    assert ref[5] == ostep.STATUS_POOL_EXHAUSTED
    assert st == isd.ERR_POOL_EXHAUSTED
    for key, t in before.items():
        assert torch.equal(cache[key], t), key


def test_page_table_full():
    w = synth.Workload("full", B=3, Hq=32, Hkv=8, d=128, N=4, L_lo=10,
                       L_hi=10, V=16)
    cache, k, v, _ = _case(w, 4)
    stride = cache["page_table"].shape[1]
    cache["seq_len"][1] = stride * 16 - 1
    nc = torch.full((w.B,), 2, dtype=torch.int32, device=DEV)
    before = {key: t.clone() for key, t in cache.items()}
    ref, st = _run_both(w, cache, k, v, nc)
    assert ref[5] == ostep.STATUS_PAGE_TABLE_FULL
    assert st == isd.ERR_PAGE_TABLE_FULL
    for key, t in before.items():
        assert torch.equal(cache[key], t), key


def test_bad_free_stack_id_changes_nothing():
    """A free-stack entry the commit would pop holds an id outside the pool:
    the whole commit is refused before any write (the id is validated, never
    used as an address)."""
    w = synth.Workload("badid", B=6, Hq=32, Hkv=8, d=128, N=4, L_lo=15,
                       L_hi=15, V=16)
    cache, k, v, _ = _case(w, 5, spare=4)
    nc = torch.full((w.B,), 2, dtype=torch.int32, device=DEV)
    top = int(cache["free_top"].item())
    P = cache["k_cache"].shape[0]
    cache["free_stack"][top - 3] = P + 7          # popped by sequence 2
    before = {key: t.clone() for key, t in cache.items()}
    status = torch.zeros((1,), dtype=torch.int32, device=DEV)
    isd.kv_commit(k, v, cache["k_cache"], cache["v_cache"],
                  cache["page_table"], cache["seq_len"], nc,
                  cache["free_stack"], cache["free_top"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == isd.ERR_BAD_PAGE
    for key, t in before.items():
        assert torch.equal(cache[key], t), key


def test_malformed_length_changes_nothing():
    w = synth.Workload("badlen", B=4, Hq=32, Hkv=8, d=128, N=4, L_lo=20,
                       L_hi=40, V=16)
    cache, k, v, nc = _case(w, 6)
    cache["seq_len"][3] = -5
    before = {key: t.clone() for key, t in cache.items()}
    status = torch.zeros((1,), dtype=torch.int32, device=DEV)
    isd.kv_commit(k, v, cache["k_cache"], cache["v_cache"],
                  cache["page_table"], cache["seq_len"], nc,
                  cache["free_stack"], cache["free_top"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == isd.ERR_BAD_STATE
    for key, t in before.items():
        assert torch.equal(cache[key], t), key


def test_status_keeps_the_first_error():
    """An error recorded earlier in the step survives a commit that
    succeeds (the status word is never cleared by a kernel)."""
    w = synth.Workload("keep", B=5, Hq=32, Hkv=8, d=128, N=4, L_lo=20,
                       L_hi=40, V=16)
    cache, k, v, nc = _case(w, 7)
    status = torch.full((1,), isd.ERR_BAD_STATE, dtype=torch.int32,
                        device=DEV)
    ref = ostep.kv_commit(_host(k), _host(v), _host(cache["k_cache"]),
                          _host(cache["v_cache"]), i64(cache["page_table"]),
                          i64(cache["seq_len"]), i64(nc),
                          i64(cache["free_stack"]),
                          int(cache["free_top"].item()))
    isd.kv_commit(k, v, cache["k_cache"], cache["v_cache"],
                  cache["page_table"], cache["seq_len"], nc,
                  cache["free_stack"], cache["free_top"], status)
    torch.cuda.synchronize()
    assert int(status.item()) == isd.ERR_BAD_STATE
    assert np.array_equal(i64(cache["seq_len"]), ref[3])
    assert np.array_equal(i64(cache["page_table"]), ref[2])
