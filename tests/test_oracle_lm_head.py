"""Pins for the oracle's LM head, gated LoRA, bfloat16 rounding and
sub-chunk vocabulary statistics (CPU only)."""

import numpy as np
import pytest
import torch

from oracle import lm_head as olm
from oracle import vocab


def _brute_logits(h, w, lora=None):
    """Pure-Python triple loop (tiny sizes)."""
    M, D = len(h), len(h[0])
    V = len(w)
    out = [[0.0] * V for _ in range(M)]
    for m in range(M):
        for v in range(V):
            acc = 0.0
            for d in range(D):
                acc += float(h[m][d]) * float(w[v][d])
            out[m][v] = acc
    if lora is not None:
        A, B, scale, mask = lora["A"], lora["B"], lora["scale"], lora["mask"]
        r = len(A)
        for m in range(M):
            if not mask[m]:
                continue
            u = [sum(float(h[m][d]) * float(A[j][d]) for d in range(D))
                 for j in range(r)]
            for v in range(V):
                out[m][v] += scale * sum(u[j] * float(B[v][j])
                                         for j in range(r))
    return np.array(out)


def test_worked_example():
    # hidden rows (1, 2) and (0, -1); weight rows (3, 0), (1, 1), (-2, 5).
    h = np.array([[1.0, 2.0], [0.0, -1.0]])
    w = np.array([[3.0, 0.0], [1.0, 1.0], [-2.0, 5.0]])
    np.testing.assert_array_equal(olm.lm_head(h, w),
                                  [[3.0, 3.0, 8.0], [0.0, -1.0, -5.0]])


def test_one_hot_hidden_selects_a_weight_column():
    rng = np.random.default_rng(0)
    D, V = 16, 40
    w = rng.normal(size=(V, D))
    h = np.eye(D)[[3, 0, 15]]
    out = olm.lm_head(h, w)
    np.testing.assert_array_equal(out[0], w[:, 3])
    np.testing.assert_array_equal(out[1], w[:, 0])
    np.testing.assert_array_equal(out[2], w[:, 15])


def test_matches_brute_force_with_and_without_lora():
    rng = np.random.default_rng(1)
    M, D, V, r = 6, 5, 7, 3
    h = rng.normal(size=(M, D))
    w = rng.normal(size=(V, D))
    lora = dict(A=rng.normal(size=(r, D)), B=rng.normal(size=(V, r)),
                scale=0.75, mask=np.array([0, 1, 1, 0, 0, 1], dtype=bool))
    np.testing.assert_allclose(olm.lm_head(h, w), _brute_logits(h, w),
                               rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(olm.lm_head(h, w, lora),
                               _brute_logits(h, w, lora), rtol=1e-13,
                               atol=1e-13)


def test_lora_rank_one_closed_form_and_clean_rows_untouched():
    # A = e_i, B = column b: a MASK row gains scale * h[i] * b, a clean row
    # is exactly the base logits (the lossless property of R-ISD).
    rng = np.random.default_rng(2)
    M, D, V = 4, 8, 10
    h = rng.normal(size=(M, D))
    w = rng.normal(size=(V, D))
    b = rng.normal(size=V)
    mask = np.array([False, True, False, True])
    lora = dict(A=np.eye(D)[[5]], B=b[:, None], scale=2.0, mask=mask)
    base = olm.lm_head(h, w)
    out = olm.lm_head(h, w, lora)
    for m in range(M):
        want = base[m] + (2.0 * h[m, 5] * b if mask[m] else 0.0)
        np.testing.assert_allclose(out[m], want, rtol=1e-14, atol=1e-14)
    np.testing.assert_array_equal(out[~mask], base[~mask])


def test_mask_rows_follow_the_stride_layout():
    # K = 4: sequence 0 has one pending row (R mode), sequence 1 two (N = 2).
    got = olm.mask_rows([1, 2], 4)
    np.testing.assert_array_equal(got, [False, True, True, True,
                                        False, False, True, True])


def test_round_bf16_known_values_and_ties_to_even():
    one = 1.0
    ulp = 2.0 ** -7                      # bfloat16 spacing in [1, 2)
    cases = {
        one: one,
        one + ulp / 2: one,               # tie, even neighbour is 1.0
        one + 3 * ulp / 2: one + 2 * ulp,  # tie, even neighbour is 1 + 2 ulp
        one + ulp / 4: one,
        one + 3 * ulp / 4: one + ulp,
        -(one + 3 * ulp / 4): -(one + ulp),
        0.0: 0.0,
        2.0 ** -130: 2.0 ** -130,         # float32 subnormal, kept bits
    }
    for x, want in cases.items():
        assert olm.round_bf16(np.array([x]))[0] == want, x


def test_round_bf16_matches_torch_conversion():
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.normal(0, 4, 20000),
                        rng.normal(0, 1e-3, 2000),
                        rng.integers(-2 ** 20, 2 ** 20, 2000) * 2.0 ** -11])
    x = x.astype(np.float32).astype(np.float64)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    np.testing.assert_array_equal(olm.round_bf16(x), ref.double().numpy())


def test_vocab_stats_brute_force_and_merge_to_row_stats():
    rng = np.random.default_rng(4)
    for V, width in ((10, 4), (64, 16), (2050, 2048), (5000, 256)):
        x = rng.normal(0, 3, (3, V))
        x[1, V // 2] = x[1].max() + 1.0   # a known argmax
        x[2, 1] = x[2, 3] = x[2].max() + 2.0   # a tie: first index wins
        cmax, csum, cidx = olm.vocab_stats(x, width)
        C = (V + width - 1) // width
        assert cmax.shape == (3, C)
        for m in range(3):
            for c in range(C):
                blk = list(x[m, c * width:min(V, (c + 1) * width)])
                mx = max(blk)
                assert cmax[m, c] == mx
                assert cidx[m, c] == c * width + blk.index(mx)
                assert csum[m, c] == pytest.approx(
                    sum(np.exp(v - mx) for v in blk), rel=1e-13)
            # Merging the chunks gives the row statistics.
            mr, sr = vocab.row_stats(x[m])
            assert cmax[m].max() == mr
            merged = np.sum(csum[m] * np.exp(cmax[m] - mr))
            assert merged == pytest.approx(sr, rel=1e-13)
        assert cidx[1, (V // 2) // width] == V // 2
        assert cidx[2, 0] == 1
