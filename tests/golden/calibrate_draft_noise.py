"""Find the draft-noise sigma_q that gives a target mean acceptance.

The synthetic logits model draws verify logits sigma_p * g1 and draft
logits sigma_p * g1 + sigma_q * g2 (g1, g2 standard normal rows).  The
expected acceptance of one draft is sum_v min(p_v, q_v) for p, q the two
softmaxes.  This script bisects sigma_q so that the mean of that overlap
over calibration rows equals each target, using the oracle's fp64 softmax,
and writes draft_noise_sigma.json beside itself.

Run from the repository root:  python tests/golden/calibrate_draft_noise.py
"""

import json
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(
    os.path.abspath(__file__)))))
from oracle.vocab import probs  # noqa: E402

CASES = [(151936, 3.0, 0.9), (151936, 3.0, 0.7), (151936, 3.0, 0.5),
         (1024, 2.0, 0.9), (1024, 2.0, 0.7), (1024, 2.0, 0.5)]
ROWS = 48


def mean_overlap(V, sigma_p, sigma_q, g1, g2):
    acc = 0.0
    for i in range(g1.shape[0]):
        p = probs(sigma_p * g1[i])
        q = probs(sigma_p * g1[i] + sigma_q * g2[i])
        acc += float(np.minimum(p, q).sum())
    return acc / g1.shape[0]


def main():
    out = []
    for V, sp, target in CASES:
        rng = np.random.default_rng(20240601 + V)
        g1 = rng.standard_normal((ROWS, V))
        g2 = rng.standard_normal((ROWS, V))
        lo, hi = 0.0, 8.0
        for _ in range(36):
            mid = 0.5 * (lo + hi)
            if mean_overlap(V, sp, mid, g1, g2) > target:
                lo = mid
            else:
                hi = mid
        sq = 0.5 * (lo + hi)
        got = mean_overlap(V, sp, sq, g1, g2)
        out.append(dict(V=V, sigma_p=sp, target=target,
                        sigma_q=round(sq, 6), overlap=round(got, 6)))
        print(out[-1], flush=True)
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                        "draft_noise_sigma.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)


if __name__ == "__main__":
    main()
