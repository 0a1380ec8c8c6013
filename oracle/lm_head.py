"""The LM head that produces the step's logits, with the R-ISD gated LoRA, and
per-sub-chunk vocabulary statistics (fp64).

Test infrastructure only (see ``oracle/__init__.py``).

What the pages fix: one forward pass over the stride gives every row its
distribution over the vocabulary, p at the clean rows and q at the MASK rows
("Inference & ISD" on the hada.io summary); the logits of a row are its final
hidden state times the output embedding (the model is an ordinary causal
transformer, "Méthodologie d'I-DLM").  R-ISD adds a gated LoRA of rank 128
that acts only at MASK positions, so the clean rows -- and with them p -- are
exactly the base model's and the method stays lossless ("Speedup Factor
Explorer" and the R-ISD model description on the same summary).

Readings (the pages give no formula for either):
* logits[m][v] = sum_d hidden[m][d] * weight[v][d]   (weight stored [V][D],
  one row per vocabulary entry);
* with the LoRA, a MASK row m adds
  scale * sum_j (sum_d hidden[m][d] * A[j][d]) * B[v][j]   (A [r][D],
  B [V][r]); a clean row adds nothing.  Row m of a batch of strides belongs
  to sequence m // K at stride row m % K, and it is a MASK row when
  m % K >= n_pending[m // K].

``round_bf16`` is the rounding of a value to the nearest bfloat16 (ties to
even), the storage format the logits are kept in.
"""

import numpy as np


def mask_rows(n_pending, K):
    """Boolean [B*K]: row m is a MASK row (stride row >= n_pending)."""
    n = np.asarray(n_pending, dtype=np.int64)
    r = np.arange(K)
    return (r[None, :] >= n[:, None]).reshape(-1)


def lm_head(hidden, weight, lora=None):
    """logits [M][V] = hidden [M][D] . weight [V][D]^T in float64.

    ``lora``: None, or a dict with ``A`` [r][D], ``B`` [V][r], ``scale``
    and ``mask`` (boolean [M], the rows it acts on)."""
    h = np.asarray(hidden, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    out = h @ w.T
    if lora is not None:
        a = np.asarray(lora["A"], dtype=np.float64)
        b = np.asarray(lora["B"], dtype=np.float64)
        mask = np.asarray(lora["mask"], dtype=bool)
        delta = (h[mask] @ a.T) @ b.T
        out[mask] += float(lora["scale"]) * delta
    return out


def round_bf16(x):
    """Nearest bfloat16 (ties to even) of values exactly representable in
    float32, returned as float64.  bfloat16 keeps the top 16 bits of the
    float32 encoding: add half of the dropped part's unit, plus one when
    the kept part is odd (ties to even), and truncate."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    keep_odd = (bits >> np.uint64(16)) & np.uint64(1)
    bits = (bits + np.uint64(0x7FFF) + keep_odd) >> np.uint64(16)
    out = (bits << np.uint64(16)).astype(np.uint32).view(np.float32)
    return out.astype(np.float64)


def vocab_stats(logits, width):
    """Statistics of each row's vocabulary sub-chunks of ``width`` entries
    (the last one ragged): per (row, chunk) the maximum, the sum of
    exp(l - maximum) and the first index (in the whole row) holding the
    maximum.  Returns (cmax [M][C], csum [M][C], cidx [M][C])."""
    x = np.asarray(logits, dtype=np.float64)
    M, V = x.shape
    C = (V + width - 1) // width
    cmax = np.empty((M, C))
    csum = np.empty((M, C))
    cidx = np.empty((M, C), dtype=np.int64)
    for c in range(C):
        blk = x[:, c * width:min(V, (c + 1) * width)]
        m = blk.max(axis=1)
        cmax[:, c] = m
        csum[:, c] = np.exp(blk - m[:, None]).sum(axis=1)
        cidx[:, c] = c * width + np.argmax(blk, axis=1)
    return cmax, csum, cidx
