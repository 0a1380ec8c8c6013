"""Philox4x32-10 counter-based generator and the ISD uniform stream.

Test infrastructure only (see ``oracle/__init__.py``).

The pages on Introspective Diffusion Language Models say nothing about the
random numbers the sampler draws.  The reading taken here: every uniform is
a pure function of (seed, sequence, step, absolute position, stream), so the
GPU and this oracle draw the same numbers without sharing state.

Philox4x32-10 is written from its published definition (J. K. Salmon,
M. A. Moraes, R. O. Dror, D. E. Shaw, "Parallel random numbers: as easy as
1, 2, 3", SC'11, section 3.2 and Table 2):

* a round maps counter (c0, c1, c2, c3) under round key (k0, k1) to
  (hi(M1*c2) ^ c1 ^ k0, lo(M1*c2), hi(M0*c0) ^ c3 ^ k1, lo(M0*c0)),
  where hi/lo are the upper/lower 32 bits of the 64-bit product;
* the multipliers are M0 = 0xD2511F53, M1 = 0xCD9E8D57;
* between rounds the key is bumped by the Weyl constants
  W0 = 0x9E3779B9 (golden ratio) and W1 = 0xBB67AE85 (sqrt(3) - 1);
* ten rounds.

Stream packing (reading of the ISD sampler, no counterpart on the pages):
key = (seed mod 2^32, seed >> 32); counter = (seq, step, pos, stream);
the uniform is u = (x0 >> 8) * 2^-24 where x0 is the first output word, so
u is one of the 2^24 values k / 2^24 and is exact in float32 and float64.
"""

import numpy as np

PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF

# Stream identifiers: which decision a uniform feeds.
STREAM_ACCEPT = 0    # ratio test of a draft
STREAM_RESAMPLE = 1  # the stride's exact token: residual or bonus sample
STREAM_BONUS = 1
STREAM_DRAFT = 2     # inverse-CDF draw of a new draft from q


def philox4x32_10(ctr, key):
    """Ten Philox4x32 rounds on one 128-bit counter (pure Python ints).

    ctr: 4 ints in [0, 2^32); key: 2 ints in [0, 2^32).  Returns 4 ints.
    """
    c0, c1, c2, c3 = (int(v) & MASK32 for v in ctr)
    k0, k1 = (int(v) & MASK32 for v in key)
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + PHILOX_W0) & MASK32
            k1 = (k1 + PHILOX_W1) & MASK32
        p0 = PHILOX_M0 * c0
        p1 = PHILOX_M1 * c2
        c0, c1, c2, c3 = (
            ((p1 >> 32) ^ c1 ^ k0) & MASK32,
            p1 & MASK32,
            ((p0 >> 32) ^ c3 ^ k1) & MASK32,
            p0 & MASK32,
        )
    return c0, c1, c2, c3


def philox4x32_10_np(c0, c1, c2, c3, k0, k1):
    """Vectorised Philox4x32-10 over numpy arrays of counters.

    All arguments broadcast; they are taken modulo 2^32.  Returns four
    uint64 arrays holding the 32-bit output words.
    """
    m = np.uint64(MASK32)
    c0 = np.asarray(c0, dtype=np.uint64) & m
    c1 = np.asarray(c1, dtype=np.uint64) & m
    c2 = np.asarray(c2, dtype=np.uint64) & m
    c3 = np.asarray(c3, dtype=np.uint64) & m
    k0 = np.asarray(k0, dtype=np.uint64) & m
    k1 = np.asarray(k1, dtype=np.uint64) & m
    for rnd in range(10):
        if rnd > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & m
            k1 = (k1 + np.uint64(PHILOX_W1)) & m
        # 32x32 -> 64-bit products fit in uint64 without wrapping.
        p0 = np.uint64(PHILOX_M0) * c0
        p1 = np.uint64(PHILOX_M1) * c2
        c0, c1, c2, c3 = (
            ((p1 >> np.uint64(32)) ^ c1 ^ k0) & m,
            p1 & m,
            ((p0 >> np.uint64(32)) ^ c3 ^ k1) & m,
            p0 & m,
        )
    return c0, c1, c2, c3


def uniform(seed, seq, step, pos, stream):
    """U(seed, seq, step, pos, stream) in [0, 1 - 2^-24], exact in float64."""
    key = (seed & MASK32, (seed >> 32) & MASK32)
    x0 = philox4x32_10((seq, step, pos, stream), key)[0]
    return float(x0 >> 8) * (2.0 ** -24)


def uniform_np(seed, seq, step, pos, stream):
    """Vectorised ``uniform`` (arrays broadcast); returns float64."""
    x0, _, _, _ = philox4x32_10_np(seq, step, pos, stream,
                                   seed & MASK32, (seed >> 32) & MASK32)
    return (x0 >> np.uint64(8)).astype(np.float64) * (2.0 ** -24)
