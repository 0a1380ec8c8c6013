"""Strided-query causal GQA attention over a paged KV cache, in fp64.

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix.  The model keeps strict causal attention with a logit
shift (hada.io summary, "Méthodologie d'I-DLM": causal attention, logit
shift, all-masked objective; "Serving compatible AR": strict causal
attention), the KV cache is paged and attention reads it through a
paged-only kernel ("Serving (SGLang)").  One forward pass of an ISD step
carries, per sequence, a stride of K query rows appended after the
committed prefix ("Introspective Strided Decoding": verify the previous
tokens and generate new ones in one forward pass).

Reading taken where the pages are silent:
* row r of the stride sits at absolute position L_b + r, where L_b is the
  committed length of sequence b;
* it attends to every committed position [0, L_b) through the page table
  and to stride rows 0..r (causal inside the stride); no window, no bias;
* Q and K arrive after any positional rotation (the caller applies it);
* grouped-query heads: query head hq reads KV head hq // g, g = Hq / Hkv;
* the softmax scale is a parameter (1/sqrt(d) in every workload).

Layouts (all float64 numpy arrays here):
  q        [B][K][Hq][d]
  k_new    [B][K][Hkv][d]   keys of the stride rows (staging)
  v_new    [B][K][Hkv][d]
  k_cache  [P][Hkv][page_size][d]
  v_cache  [P][Hkv][page_size][d]
  page_table int [B][max_pages]; logical page i of sequence b lives in
             physical page page_table[b][i]
  seq_len  int [B]
"""

import numpy as np


def gather_prefix(cache, page_table_row, length, h, page_size):
    """Walk the page table and return the first ``length`` rows of head h.

    Returns an array [length][d] in logical (position) order.
    """
    d = cache.shape[-1]
    rows = np.empty((length, d), dtype=np.float64)
    n_pages = (length + page_size - 1) // page_size
    for lp in range(n_pages):
        phys = int(page_table_row[lp])
        lo = lp * page_size
        hi = min(length, lo + page_size)
        rows[lo:hi] = cache[phys, h, 0:hi - lo]
    return rows


def attn_strided(q, k_new, v_new, k_cache, v_cache, page_table, seq_len,
                 scale, page_size=16, pairs=None):
    """Causal attention of each stride row over its committed prefix.

    For every sequence b, KV head h, stride row r and group member j
    (query head hq = h * g + j):

        keys   = prefix keys [0, L_b) of head h, then k_new[b, 0..r, h]
        s      = scale * keys @ q[b, r, hq]
        O      = sum_t softmax(s)_t * values_t
        lse    = log(sum_t exp(s_t))            (natural log)

    The softmax is taken in two passes (max, then sum of exponentials).
    ``pairs`` optionally restricts the work to a list of (b, h); outputs of
    other pairs are left as NaN.  Returns (out [B][K][Hq][d], lse [B][K][Hq]).
    """
    B, K, Hq, d = q.shape
    Hkv = k_new.shape[2]
    g = Hq // Hkv
    out = np.full((B, K, Hq, d), np.nan)
    lse = np.full((B, K, Hq), np.nan)
    if pairs is None:
        pairs = [(b, h) for b in range(B) for h in range(Hkv)]
    for b, h in pairs:
        L = int(seq_len[b])
        pk = gather_prefix(k_cache, page_table[b], L, h, page_size)
        pv = gather_prefix(v_cache, page_table[b], L, h, page_size)
        for r in range(K):
            keys = np.concatenate([pk, k_new[b, 0:r + 1, h]], axis=0)
            vals = np.concatenate([pv, v_new[b, 0:r + 1, h]], axis=0)
            for j in range(g):
                hq = h * g + j
                s = scale * (keys @ q[b, r, hq])
                m = np.max(s)
                e = np.exp(s - m)
                den = np.sum(e)
                out[b, r, hq] = (e @ vals) / den
                lse[b, r, hq] = m + np.log(den)
    return out, lse
