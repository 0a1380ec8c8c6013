"""GPU parity of isd_lm_head (tcgen05 GEMM + vocabulary statistics + gated
LoRA) and of the accept step fed by its statistics, against the fp64 oracle.

The synthetic hidden states, weights and (sparse) LoRA factors are integers
scaled by powers of two, so every contraction is exact in float32 in any
order: the tensor cores and the oracle round the same exact value, and the
logits must match bit for bit.  Sub-chunk maxima and first indices are then
exact too, and the sums of exp(l - max) agree within 1e-5 relative.  Dense
LoRA factors make the bf16 rounding of the rank-r intermediate visible;
that case is held to a bound derived from the two roundings.
"""

import numpy as np
import pytest
import torch

from introspective_strided_decoding_b200 import isd, synth
from oracle import lm_head as olm
from oracle import step as ostep
from tests.gpu_util import (compare_accept, f32, f64, gpu_accept,
                            gpu_state_from, i64, next_oracle_state,
                            oracle_initial_state)

pytestmark = pytest.mark.gpu
DEV = "cuda"
SUB = 2048


def _inputs(seed, M, D, V, s_h=12.0):
    W = synth.lm_weight(seed, V, D, DEV).to(torch.bfloat16)
    H = synth.hidden_rows(seed, torch.arange(M), torch.zeros(M, dtype=torch.int64),
                          -1, D, s_h, 0.0, DEV).to(torch.bfloat16)
    return H.contiguous(), W.contiguous()


def _oracle_logits(H, W, lora=None, chunk=16384):
    """round_bf16 of the fp64 oracle logits, computed in vocabulary chunks."""
    h = f64(H)
    V = W.shape[0]
    out = np.empty((h.shape[0], V))
    for v0 in range(0, V, chunk):
        w = f64(W[v0:v0 + chunk])
        lo = None
        if lora is not None:
            lo = dict(lora, B=lora["B"][v0:v0 + chunk])
        out[:, v0:v0 + chunk] = olm.lm_head(h, w, lo)
    return out


def _gpu(H, W, stats=True, **kw):
    M, V = H.shape[0], W.shape[0]
    logits = torch.empty((M, V), dtype=torch.bfloat16, device=DEV)
    vs = isd.new_vocab_stats(M, V, DEV) if stats else None
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    isd.lm_head(H, W, logits, vocab_stats=vs, status=status, **kw)
    torch.cuda.synchronize()
    return logits, vs, int(status.item())


def _check_stats(vs, ref_rounded, M, V, rows=None, chunks=None):
    csum, cmax, cidx = isd.vocab_stats_view(vs, M, V)
    csum, cmax, cidx = (csum.cpu().numpy(), cmax.cpu().double().numpy(),
                        cidx.cpu().numpy())
    rows = range(M) if rows is None else rows
    for m in rows:
        r_max, r_sum, r_idx = olm.vocab_stats(ref_rounded[m:m + 1], SUB)
        cs = range(r_max.shape[1]) if chunks is None else chunks
        for c in cs:
            assert cmax[m, c] == r_max[0, c], (m, c)
            assert cidx[m, c] == r_idx[0, c], (m, c)
            assert abs(csum[m, c] - r_sum[0, c]) <= 1e-5 * r_sum[0, c], (m, c)


# (M, D, V): single and double accumulators (M <= 128 / > 128), partial
# row tiles, ragged vocabulary tiles and sub-chunks, a short and a long K.
SHAPES = [(1, 64, 8), (8, 128, 264), (100, 256, 1000), (128, 512, 4104),
          (200, 256, 2056), (512, 128, 6152), (300, 4096, 2312)]


@pytest.mark.parametrize("M,D,V", SHAPES)
def test_logits_and_statistics_exact(M, D, V):
    H, W = _inputs(7, M, D, V)
    logits, vs, st = _gpu(H, W)
    assert st == isd.OK
    ref = olm.round_bf16(_oracle_logits(H, W))
    got = f64(logits)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]
    _check_stats(vs, ref, M, V)


def test_logits_without_statistics():
    H, W = _inputs(8, 64, 256, 520)
    logits, _, st = _gpu(H, W, stats=False)
    assert st == isd.OK
    assert np.array_equal(f64(logits), olm.round_bf16(_oracle_logits(H, W)))


def _lora_inputs(seed, B, K, D, V, r, sparse, n_choices):
    M = B * K
    H, W = _inputs(seed, M, D, V)
    A, Bf = synth.lora_factors(seed, r, D, V, DEV, sparse=sparse)
    g = torch.Generator().manual_seed(seed)
    n_pending = torch.as_tensor(n_choices)[
        torch.randint(0, len(n_choices), (B,), generator=g)].to(torch.int32)
    return H, W, A.to(torch.bfloat16).contiguous(), \
        Bf.to(torch.bfloat16).contiguous(), n_pending.to(DEV)


@pytest.mark.parametrize("B,K,D,V,r", [(16, 8, 512, 4104, 128),
                                       (40, 8, 256, 2312, 64),
                                       (4, 16, 128, 1032, 256)])
def test_gated_lora_sparse_is_exact(B, K, D, V, r):
    # One 1 per row of A: U = h[:, cols] exactly, so everything stays exact.
    H, W, A, Bf, n_pending = _lora_inputs(11, B, K, D, V, r, True,
                                          [1, K // 2, 0, K])
    logits, vs, st = _gpu(H, W, lora_a=A, lora_b=Bf, lora_scale=1.0,
                          n_pending=n_pending, rows_per_seq=K)
    assert st == isd.OK
    mask = olm.mask_rows(i64(n_pending), K)
    ref = olm.round_bf16(_oracle_logits(
        H, W, dict(A=f64(A), B=f64(Bf), scale=1.0, mask=mask)))
    got = f64(logits)
    assert np.array_equal(got, ref), np.argwhere(got != ref)[:5]
    # Clean rows are exactly the base model's logits (lossless R-ISD).
    base = olm.round_bf16(_oracle_logits(H, W))
    assert np.array_equal(got[~mask], base[~mask])
    assert mask.any() and (~mask).any()
    _check_stats(vs, ref, B * K, V)


def test_gated_lora_dense_within_rounding_bound():
    B, K, D, V, r, scale = 8, 8, 1024, 4104, 128, 2.0 ** -5
    H, W, A, Bf, n_pending = _lora_inputs(12, B, K, D, V, r, False, [1, 4])
    logits, _, st = _gpu(H, W, stats=False, lora_a=A, lora_b=Bf,
                         lora_scale=scale, n_pending=n_pending,
                         rows_per_seq=K)
    assert st == isd.OK
    mask = olm.mask_rows(i64(n_pending), K)
    lora = dict(A=f64(A), B=f64(Bf), scale=scale, mask=mask)
    ref = _oracle_logits(H, W, lora)
    # Bound: the rank-r intermediate is rounded to bf16 (relative 2^-9 per
    # entry), the logits once more (2^-9 of the value, 2^-8 to cover the
    # neighbour at a binade edge); the fp32 accumulation error is far below.
    u = np.abs(f64(H)[mask] @ f64(A).T) * scale
    tol = 2.0 ** -8 * np.abs(ref)
    tol[mask] += 2.0 ** -9 * (u @ np.abs(f64(Bf)).T) + 1e-6
    err = np.abs(f64(logits) - ref)
    assert (err <= tol + 1e-12).all(), float((err - tol).max())
    # The clean rows are exact.
    base = olm.round_bf16(_oracle_logits(H, W))
    assert np.array_equal(f64(logits)[~mask], base[~mask])


def test_bad_pending_count_is_reported_and_gets_no_lora():
    B, K, D, V, r = 4, 8, 128, 1032, 64
    H, W, A, Bf, n_pending = _lora_inputs(13, B, K, D, V, r, True, [1])
    n_pending[2] = K + 3
    logits, _, st = _gpu(H, W, stats=False, lora_a=A, lora_b=Bf,
                         lora_scale=1.0, n_pending=n_pending, rows_per_seq=K)
    assert st == isd.ERR_BAD_STATE
    base = olm.round_bf16(_oracle_logits(H, W))
    got = f64(logits)
    assert np.array_equal(got[2 * K:3 * K], base[2 * K:3 * K])


@pytest.mark.parametrize("B,K,D", [(64, 8, 4096), (32, 16, 5120)])
def test_full_size_sampled(B, K, D):
    """The C=64 LM head (512 rows, hidden 4096) and the 32B-shaped one (512
    rows, hidden 5120), vocabulary 151 936, with the rank-128 LoRA (sparse,
    exact); sampled rows and sub-chunks against the oracle, the rest by
    properties that hold for any correct result."""
    V, r = 151936, 128
    H, W, A, Bf, n_pending = _lora_inputs(14, B, K, D, V, r, True,
                                          [1, K // 2])
    logits, vs, st = _gpu(H, W, lora_a=A, lora_b=Bf, lora_scale=1.0,
                          n_pending=n_pending, rows_per_seq=K)
    assert st == isd.OK
    M = B * K
    mask = olm.mask_rows(i64(n_pending), K)
    rows = [0, 1, 127, 128, 255, 256, 300, 511]
    chunks = [0, 1, 37, 73, 74]
    hr = f64(H[rows])
    for c in chunks:
        v0, v1 = c * SUB, min(V, (c + 1) * SUB)
        w = f64(W[v0:v1])
        lo = dict(A=f64(A), B=f64(Bf[v0:v1]), scale=1.0, mask=mask[rows])
        ref = olm.round_bf16(olm.lm_head(hr, w, lo))
        got = f64(logits[rows, v0:v1])
        assert np.array_equal(got, ref), (c, np.argwhere(got != ref)[:5])
        csum, cmax, cidx = isd.vocab_stats_view(vs, M, V)
        rmax, rsum, ridx = olm.vocab_stats(ref, SUB)
        for i, m in enumerate(rows):
            assert float(cmax[m, c]) == rmax[i, 0]
            assert int(cidx[m, c]) == v0 + ridx[i, 0]
            assert abs(float(csum[m, c]) - rsum[i, 0]) <= 1e-5 * rsum[i, 0]
    # Every row and sub-chunk: the max is an entry of the chunk at the
    # reported index, the sum lies in [1, width].
    csum, cmax, cidx = isd.vocab_stats_view(vs, M, V)
    C = csum.shape[1]
    lo_idx = torch.arange(C, device=DEV) * SUB
    assert bool(((cidx >= lo_idx) & (cidx < torch.clamp(lo_idx + SUB, max=V))
                 ).all())
    picked = torch.gather(logits, 1, cidx.long()).float()
    assert torch.equal(picked, cmax)
    assert bool(((csum >= 1.0) & (csum <= SUB)).all())


@pytest.mark.parametrize("proposal", ["sample", "argmax"])
def test_fused_step_matches_oracle(proposal):
    """Hidden states -> isd_lm_head (logits + statistics) ->
    isd_accept_resample fed by those statistics, in lockstep with the oracle
    run on its own fp64 logits of the same hidden states.  With argmax
    proposals the drafts come straight from the statistics' first-argmax
    indices."""
    w = synth.Workload("lm_fused", B=8, Hq=32, Hkv=8, d=128, N=4, L_lo=100,
                       L_hi=900, V=151936, target_accept=0.9, D=1024)
    seed, steps = 21, 4
    W = synth.lm_weight(seed, w.V, w.D, DEV).to(torch.bfloat16).contiguous()
    st0 = synth.initial_state(w, seed, "cpu")
    ostate = oracle_initial_state(st0)
    L = synth.prefix_lengths(w, seed).numpy().astype(np.int64)
    M = w.B * w.K
    lp_dev = torch.zeros((w.B, w.K, w.V), dtype=torch.bfloat16, device=DEV)
    lp_host = np.zeros((w.B, w.K, w.V), dtype=np.float32)
    exact = rejected = accepted_all = 0
    for s in range(steps):
        H = synth.step_hidden(w, seed, torch.from_numpy(L),
                              torch.from_numpy(ostate["n_pending"]), s,
                              DEV).reshape(M, w.D).contiguous()
        lc_dev = torch.empty((w.B, w.K, w.V), dtype=torch.bfloat16,
                             device=DEV)
        vs = isd.new_vocab_stats(M, w.V, DEV)
        isd.lm_head(H, W, lc_dev.view(M, w.V), vocab_stats=vs)
        lc_host = olm.round_bf16(_oracle_logits(H, W)).astype(
            np.float32).reshape(w.B, w.K, w.V)

        def oracle(flip=(), lc_host=lc_host, lp_host=lp_host, ostate=ostate,
                   L=L, s=s):
            return ostep.accept_resample(lc_host, lp_host, ostate["pending"],
                                         ostate["n_pending"], ostate["q_row"],
                                         L, seed, s, w.N, proposal=proposal,
                                         flip=flip)
        ref = oracle()
        o = gpu_accept(lc_dev, lp_dev,
                       torch.as_tensor(L, dtype=torch.int32, device=DEV),
                       gpu_state_from(ostate, DEV), seed, s,
                       proposal=isd.PROPOSAL_ARGMAX if proposal == "argmax"
                       else isd.PROPOSAL_SAMPLE, vocab_stats=vs)
        torch.cuda.synchronize()
        assert int(o.status.item()) == isd.OK
        c = compare_accept(o, ref, ostate["n_pending"],
                           lambda b, r: lc_host[b, r].astype(np.float64),
                           oracle, ostate["pending"])
        exact += c["exact"]
        rejected += int(ref["rejected"].sum())
        accepted_all += int(((ostate["n_pending"] == w.N)
                             & ~ref["rejected"]).sum())
        ostate = next_oracle_state(ref)
        L = L + ref["n_commit"]
        lp_dev, lp_host = lc_dev, lc_host
    print(f"fused: {exact} exact, {rejected} rejected, {accepted_all} "
          "all-accepted")
    assert exact >= 0.9 * w.B * steps


@pytest.mark.parametrize("graph", [False, True])
def test_decoder_with_lm_head_and_lora_matches_oracle(graph):
    """The decoder's step with the LM head and the R-ISD LoRA (eager calls
    or CUDA-graph replays), each step checked against the oracle started
    from the state the GPU carried into it: the LoRA gate must follow that
    state's pending counts."""
    from introspective_strided_decoding_b200.driver import Decoder
    w = synth.Workload("lm_decoder", B=8, Hq=32, Hkv=8, d=128, N=4,
                       L_lo=100, L_hi=400, V=8200, sigma_p=3.0, sigma_q=0.25,
                       D=256, steps=6)
    seed, r = 31, 64
    W = synth.lm_weight(seed, w.V, w.D, DEV).to(torch.bfloat16).contiguous()
    A, Bf = synth.lora_factors(seed, r, w.D, w.V, DEV, sparse=True)
    A = A.to(torch.bfloat16).contiguous()
    Bf = Bf.to(torch.bfloat16).contiguous()
    cache = synth.make_cache(w, seed, DEV)
    dec = Decoder(w, cache, synth.initial_state(w, seed, DEV), DEV, seed,
                  record=True, lm=dict(weight=W, lora_a=A, lora_b=Bf,
                                       lora_scale=1.0))
    if graph:
        dec.capture()
    M = w.B * w.K
    lp_host = np.zeros((w.B, w.K, w.V), dtype=np.float32)
    exact = 0
    for s in range(w.steps):
        st = dec.state
        ostate = oracle_initial_state(st)
        L = i64(cache["seq_len"])
        H = synth.step_hidden(w, seed, cache["seq_len"], st["n_pending"], s,
                              DEV)
        dec.hidden.copy_(H)
        q, k, v = synth.make_stride(w, seed, s, DEV)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        if graph:
            dec.replay()
        else:
            dec.step_idx = s
            dec.step()
        torch.cuda.synchronize()
        assert int(dec.status.item()) == isd.OK
        mask = olm.mask_rows(ostate["n_pending"], w.K)
        lc_host = olm.round_bf16(_oracle_logits(
            H.reshape(M, w.D), W, dict(A=f64(A), B=f64(Bf), scale=1.0,
                                       mask=mask))
        ).astype(np.float32).reshape(w.B, w.K, w.V)
        # The logits the step made (the buffer it just used).
        assert np.array_equal(f64(dec.logits[1 - dec.cur]),
                              lc_host.astype(np.float64))

        def oracle(flip=(), lc_host=lc_host, lp_host=lp_host, ostate=ostate,
                   L=L, s=s):
            return ostep.accept_resample(lc_host, lp_host, ostate["pending"],
                                         ostate["n_pending"], ostate["q_row"],
                                         L, seed, s, w.N, flip=flip)

        class View:
            n_commit = dec.n_commit
            commit_tokens = dec.commit_tokens
            state_out = dec.state
            row_stats = dec.row_stats
            ratio = dec.ratio
        c = compare_accept(View, oracle(), ostate["n_pending"],
                           lambda b, rr: lc_host[b, rr].astype(np.float64),
                           oracle, ostate["pending"])
        exact += c["exact"]
        lp_host = lc_host
    if graph:
        dec.release_graphs()
    assert exact >= 0.9 * w.B * w.steps
