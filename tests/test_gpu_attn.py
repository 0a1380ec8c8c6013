"""GPU parity of isd_attn_strided against the fp64 oracle.

Tolerance (element-wise, absolute): 2e-2 for bf16 inputs, 1e-5 for fp32.
Small cases compare every output and span several units per CTA, CTAs that
split a (b, h) (combine path) and ragged page tails; full-size workloads
compare sampled (b, h) pairs the oracle computes one by one, in the launch
configuration the benchmark uses.
"""

import math

import numpy as np
import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from tests.gpu_util import (TOL, f64, gpu_attention, i64, oracle_attention,
                            oracle_attention_pairs)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf(**kw):
    base = dict(name="small", B=3, Hq=8, Hkv=2, d=128, N=4, L_lo=0, L_hi=100,
                V=1024, dtype="bf16", sigma_q=0.3, shuffle_pages=True)
    base.update(kw)
    return synth.Workload(**base)


SMALL = [
    synth.TINY,                                              # fp32, d 64
    synth.TINY.with_(name="tiny_ragged", B=3, Hq=8, Hkv=2, L_lo=0, L_hi=70,
                     shuffle_pages=True),
    _bf(name="bf16_m32", L_lo=0, L_hi=100),
    _bf(name="bf16_m16", N=2, L_lo=15, L_hi=130),
    _bf(name="bf16_m64", B=2, Hq=16, Hkv=2, L_lo=17, L_hi=260),
    _bf(name="bf16_m128", B=2, Hq=16, Hkv=2, N=8, L_lo=1, L_hi=300),
    _bf(name="bf16_m128_g4", B=2, Hq=8, Hkv=2, N=8, L_lo=30, L_hi=40),
    _bf(name="bf16_m24", B=3, Hq=6, Hkv=2, N=4, L_lo=3, L_hi=140),
    _bf(name="bf16_m48", B=2, Hq=12, Hkv=2, N=4, L_lo=40, L_hi=150),
    _bf(name="bf16_m96", B=2, Hq=12, Hkv=2, N=8, L_lo=20, L_hi=90),
]


@pytest.mark.parametrize("w", SMALL, ids=lambda w: w.name)
@pytest.mark.parametrize("num_ctas", [0, 1, 3, 7, 300])
@pytest.mark.parametrize("sharp", [False, True])
def test_small_cases_every_output(w, num_ctas, sharp):
    cache = synth.make_cache(w, 11, DEV)
    q, k, v = synth.make_stride(w, 11, 0, DEV, sharp=sharp)
    out, lse = gpu_attention(w, cache, q, k, v, num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_attention(w, cache, q, k, v)
    tol = TOL[w.dtype]
    err = np.abs(f64(out) - ref)
    assert err.max() <= tol, (err.max(), np.unravel_index(err.argmax(),
                                                          err.shape))
    assert np.abs(f64(lse) - ref_lse).max() <= tol


@pytest.mark.parametrize("w", [SMALL[2], SMALL[4], SMALL[9], SMALL[5]],
                         ids=lambda w: w.name)
@pytest.mark.parametrize("num_ctas", [0, 3])
def test_reference_max_moves_on_later_blocks(w, num_ctas):
    """Cached keys scaled by 1 + 4i on logical page i, with unscaled queries
    and 3 to 5 blocks of 128 keys per sequence: each block raises the row
    maxima by about 7 (natural-log units), more than the 2^8 (5.5) the
    kernel tolerates against its running reference max, so on every later
    block the reference moves, O and the row sums are rescaled and the
    block's pass is redone (at 32, 64, 96 and 128 rows per KV head, with
    and without split segments)."""
    w = w.with_(L_lo=300, L_hi=600)
    cache = synth.make_cache(w, 11, DEV)
    pt = cache["page_table"].long().cpu()
    L = cache["seq_len"].long().cpu()
    kc = cache["k_cache"]
    with torch.no_grad():
        for b in range(w.B):
            for i in range((int(L[b]) + 15) // 16):
                kc[int(pt[b, i])] *= 1.0 + 4.0 * i
    q, k, v = synth.make_stride(w, 11, 0, DEV, sharp=True)
    out, lse = gpu_attention(w, cache, q, k, v, num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_attention(w, cache, q, k, v)
    tol = TOL[w.dtype]
    err = np.abs(f64(out) - ref)
    assert err.max() <= tol, (err.max(), np.unravel_index(err.argmax(),
                                                          err.shape))
    # lse grows to hundreds here: the same bound, relative to its size.
    lse_err = np.abs(f64(lse) - ref_lse) / np.maximum(1.0, np.abs(ref_lse))
    assert lse_err.max() <= tol


@pytest.mark.parametrize("L", [0, 1, 15, 16, 17, 32])
def test_edge_lengths(L):
    w = _bf(name="edge", B=2, L_lo=L, L_hi=L)
    cache = synth.make_cache(w, 5, DEV)
    q, k, v = synth.make_stride(w, 5, 0, DEV, sharp=True)
    for nc in (0, 2):
        out, lse = gpu_attention(w, cache, q, k, v, num_ctas=nc)
        ref, ref_lse = oracle_attention(w, cache, q, k, v)
        assert np.abs(f64(out) - ref).max() <= TOL["bf16"]
        assert np.abs(f64(lse) - ref_lse).max() <= TOL["bf16"]


def test_unwritten_slots_may_hold_nan():
    # Slots past L_b in a sequence's last page are never read as values.
    w = _bf(name="nan", B=3, L_lo=20, L_hi=40)
    cache = synth.make_cache(w, 6, DEV)
    pt, sl = i64(cache["page_table"]), i64(cache["seq_len"])
    for b in range(w.B):
        L = int(sl[b])
        if L % 16:
            page = int(pt[b, L // 16])
            cache["v_cache"][page, :, L % 16:] = float("nan")
            cache["k_cache"][page, :, L % 16:] = float("nan")
    q, k, v = synth.make_stride(w, 6, 0, DEV)
    out, _ = gpu_attention(w, cache, q, k, v)
    assert torch.isfinite(out).all()
    ref, _ = oracle_attention(w, cache, q, k, v)
    assert np.abs(f64(out) - ref).max() <= TOL["bf16"]


def test_bad_page_id_is_reported_not_faulted():
    w = _bf(name="badpage", B=2, L_lo=40, L_hi=40)
    cache = synth.make_cache(w, 7, DEV)
    cache["page_table"][1, 1] = 10 ** 6
    q, k, v = synth.make_stride(w, 7, 0, DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    out, _ = gpu_attention(w, cache, q, k, v, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == isd.ERR_BAD_PAGE
    # Sequence 0 is untouched by the bad entry.
    ref, _ = oracle_attention(w, cache, q, k, v, pairs=[(0, 0), (0, 1)])
    assert np.abs(f64(out)[0] - ref[0]).max() <= TOL["bf16"]


def test_paging_invariance_on_gpu():
    w = _bf(name="perm", B=2, L_lo=50, L_hi=120)
    cache = synth.make_cache(w, 8, DEV)
    q, k, v = synth.make_stride(w, 8, 0, DEV, sharp=True)
    out1, lse1 = gpu_attention(w, cache, q, k, v, num_ctas=1)
    P = cache["k_cache"].shape[0]
    perm = torch.randperm(P, generator=torch.Generator().manual_seed(0))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(P)
    c2 = dict(cache)
    c2["k_cache"] = cache["k_cache"][perm.to(DEV)].contiguous()
    c2["v_cache"] = cache["v_cache"][perm.to(DEV)].contiguous()
    pt = cache["page_table"].long()
    c2["page_table"] = torch.where(pt >= 0, inv.to(DEV)[pt.clamp(min=0)],
                                   pt).to(torch.int32).contiguous()
    out2, lse2 = gpu_attention(w, c2, q, k, v, num_ctas=1)
    assert torch.equal(out1, out2) and torch.equal(lse1, lse2)


def test_deterministic():
    w = _bf(name="det", B=4, L_lo=100, L_hi=900)
    cache = synth.make_cache(w, 9, DEV)
    q, k, v = synth.make_stride(w, 9, 0, DEV)
    a, la = gpu_attention(w, cache, q, k, v)
    b, lb = gpu_attention(w, cache, q, k, v)
    assert torch.equal(a, b) and torch.equal(la, lb)


@pytest.mark.parametrize("num_ctas", [0, 5, 1024])
def test_workspace_counters_reset_between_calls(num_ctas):
    """One workspace reused by consecutive calls on different inputs: each
    call equals a call on a fresh workspace bit for bit (nothing carries
    over between calls)."""
    w = _bf(name="reuse", B=3, L_lo=40, L_hi=700)
    cache = synth.make_cache(w, 4, DEV)
    a = None
    ws = None
    for step in range(3):
        q, k, v = synth.make_stride(w, 4, step, DEV)
        out = torch.empty_like(q)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=DEV)
        args = isd.attn_args(q, k, v, cache["k_cache"], cache["v_cache"],
                             cache["page_table"], cache["seq_len"], out, lse,
                             None, 1.0 / math.sqrt(w.d), None, num_ctas)
        if ws is None:
            ws = torch.zeros(isd.attn_workspace_bytes(args), dtype=torch.uint8,
                             device=DEV)
        isd.attn_strided(q, k, v, cache["k_cache"], cache["v_cache"],
                         cache["page_table"], cache["seq_len"], out=out,
                         lse=lse, softmax_scale=1.0 / math.sqrt(w.d),
                         workspace=ws, num_ctas=num_ctas)
        ref_out, ref_lse = gpu_attention(w, cache, q, k, v, num_ctas=num_ctas)
        torch.cuda.synchronize()
        assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse), step
        ref, _ = oracle_attention(w, cache, q, k, v)
        assert np.abs(f64(out) - ref).max() <= TOL["bf16"]


FULL = [synth.SHAPE_8B, synth.C64, synth.SHAPE_32B,
        synth.sweep_workload(8, 2, 0.9), synth.sweep_workload(8, 8, 0.5)]


@pytest.mark.parametrize("w", FULL, ids=lambda w: w.name)
def test_full_size_sampled_pairs(w):
    w = w.with_(steps=1)
    cache = synth.make_cache(w, 1, DEV)
    q, k, v = synth.make_stride(w, 1, 0, DEV)
    out, lse = gpu_attention(w, cache, q, k, v)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and torch.isfinite(lse).all()
    rng = np.random.default_rng(0)
    pairs = sorted({(int(rng.integers(w.B)), int(rng.integers(w.Hkv)))
                    for _ in range(3)} | {(w.B - 1, w.Hkv - 1)})
    ref, ref_lse = oracle_attention_pairs(w, cache, q, k, v, pairs,
                                          i64(cache["page_table"]),
                                          i64(cache["seq_len"]))
    g = w.Hq // w.Hkv
    for b, h in pairs:
        sl = slice(h * g, (h + 1) * g)
        assert np.abs(f64(out)[b, :, sl] - ref[b, :, sl]).max() <= TOL["bf16"]
        assert np.abs(f64(lse)[b, :, sl] - ref_lse[b, :, sl]).max() <= \
            TOL["bf16"]
