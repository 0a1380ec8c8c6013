"""Pins for the tokens-per-forward reading (CPU only).

The closed form and the printed values come from the hada.io summary of
"Introspective Diffusion Language Models" ("Speedup Factor Explorer" and
"Throughput").  The schedule chain is built from the stride reading alone,
so its agreement with the closed form pins that reading.
"""

import os

import numpy as np
import pytest

from oracle import tpf

GOLDEN = os.path.join(os.path.dirname(__file__), "golden",
                      "tpf_printed_values.txt")


def _printed():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            w = line.split()
            rows.append(dict(name=w[0], N=int(w[1]), p=float(w[2]),
                             tpf=float(w[3]), tpf_tol=float(w[4]),
                             eff=float(w[5]), eff_tol=float(w[6]),
                             qs=int(w[7]), closed=(w[8] == "yes")))
    return rows


@pytest.mark.parametrize("row", _printed(), ids=lambda r: r["name"])
def test_printed_values(row):
    if row["closed"]:
        t = tpf.tpf_closed_form(row["p"], row["N"])
        assert abs(t - row["tpf"]) <= row["tpf_tol"]
        assert abs(tpf.efficiency(t, row["qs"]) - row["eff"]) <= row["eff_tol"]
        # The query size that reproduces the printed efficiency is 2N - 1.
        assert row["qs"] == 2 * row["N"] - 1
        assert abs(tpf.efficiency(t, 2 * row["N"]) - row["eff"]) > 0.1
    else:
        # Only the efficiency definition: some TPF within the printed
        # rounding of the TPF must give the printed efficiency.
        lo = np.sqrt((row["eff"] - row["eff_tol"]) * row["qs"])
        hi = np.sqrt((row["eff"] + row["eff_tol"]) * row["qs"])
        assert lo <= row["tpf"] + row["tpf_tol"]
        assert hi >= row["tpf"] - row["tpf_tol"]


def test_closed_form_exact_value():
    # (2 + 0.9 + 0.81) / (2 - 0.729) written out by hand.
    assert tpf.tpf_closed_form(0.9, 4) == pytest.approx(3.71 / 1.271,
                                                        rel=1e-14)


@pytest.mark.parametrize("N", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("p", [0.0, 0.3, 0.5, 0.7, 0.9, 0.99, 1.0])
def test_schedule_chain_realises_closed_form(N, p):
    assert tpf.tpf_markov(p, N) == pytest.approx(tpf.tpf_closed_form(p, N),
                                                 rel=1e-12, abs=1e-12)


def test_limits():
    # p = 1: every stride accepts everything, N tokens per forward.
    for N in (2, 4, 8):
        assert tpf.tpf_closed_form(1.0, N) == pytest.approx(N)
    # p = 0: S and R alternate, yielding 1 token each.
    assert tpf.tpf_closed_form(0.0, 4) == pytest.approx(1.0)


def test_finite_horizon_converges_to_stationary():
    for N, p in ((4, 0.9), (8, 0.7), (2, 0.5)):
        T = 20000
        assert tpf.expected_tokens(p, N, T) / T == pytest.approx(
            tpf.tpf_closed_form(p, N), rel=1e-3)


def test_finite_horizon_small_cases_by_hand():
    # From R: step 1 always yields 1 token and lands in S.
    assert tpf.expected_tokens(0.9, 4, 1) == pytest.approx(1.0)
    # Step 2 is an S step: 1 + p + p^2 + p^3 expected tokens.
    assert tpf.expected_tokens(0.9, 4, 2) == pytest.approx(
        1.0 + 1 + 0.9 + 0.81 + 0.729)
