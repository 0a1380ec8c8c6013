"""Seeded synthetic inputs for the ISD step (torch, any device).

This module holds input recipes only: shapes, value distributions, the
paged-cache layout and the logits model.  It does none of the step's
arithmetic and imports nothing else from the package, so the CUDA path
and the CPU oracle can both be fed from it.

Workload shapes stand in for the serving workloads of the I-DLM pages
(8B and 32B models converted from Qwen3: 32 query / 8 KV heads and
64 / 8, head dim 128, vocabulary 151 936).  There are no weights and no
datasets: every tensor is drawn from a seeded generator.

Logits model.  The verify logits of sequence b at absolute position t are
sigma_p * G(seed, b, t) for a keyed standard-normal row G, so a position
scores the same whenever it is verified.  A MASK row that drafts position
t at step s carries the same row plus sigma_q * G'(seed, b, t, s).  The
expected acceptance of a draft is then sum_v min(p_v, q_v); sigma_q is
chosen per target acceptance from ``DRAFT_SIGMA_Q`` (values found by the
calibration script ``tests/golden/calibrate_draft_noise.py``).

Peaked rows.  A trained model's rows put most of their mass on a few
tokens.  With ``peak`` > 0 every row of (b, t) adds ``peak`` to the logit
of one keyed token, shared by the clean row and the MASK rows of that
position, so p and q concentrate on the same token (peak = 18.6 gives that
token about 0.9 of the mass at sigma_p = 3 and V = 151 936).
"""

import math
from dataclasses import dataclass, field, replace

import torch

PAGE_SIZE = 16
_M32 = 0xFFFFFFFF
_MIX = 0x045D9F3B  # < 2^27, so 32-bit values times it stay inside int64

# sigma_q giving a target mean acceptance sum_v min(p_v, q_v), keyed by
# (vocab, sigma_p, target).  Written by tests/golden/calibrate_draft_noise.py.
DRAFT_SIGMA_Q = {
    (151936, 3.0, 0.9): 0.254096,
    (151936, 3.0, 0.7): 0.782094,
    (151936, 3.0, 0.5): 1.377923,
    (1024, 2.0, 0.9): 0.268481,
    (1024, 2.0, 0.7): 0.813761,
    (1024, 2.0, 0.5): 1.414946,
}


@dataclass(frozen=True)
class Workload:
    """One synthetic ISD workload (shapes + distributions)."""
    name: str
    B: int
    Hq: int
    Hkv: int
    d: int
    N: int
    L_lo: int
    L_hi: int
    V: int
    dtype: str = "bf16"          # "bf16" or "f32"
    sigma_p: float = 3.0
    sigma_q: float = 0.0
    target_accept: float = None
    qkv_scale: float = None      # default 1/sqrt(d)
    shuffle_pages: bool = True
    steps: int = 1
    spare_pages: int = 0         # extra free pages beyond growth over steps
    peak: float = 0.0            # logit boost of one keyed token per row
    D: int = 4096                # hidden size (LM-head inputs)
    meta: dict = field(default_factory=dict, compare=False)

    @property
    def K(self):
        return 2 * self.N

    @property
    def g(self):
        return self.Hq // self.Hkv

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32

    def with_(self, **kw):
        return replace(self, **kw)


def draft_sigma(w):
    """sigma_q of a workload: explicit, or looked up by target acceptance."""
    if w.target_accept is None:
        return w.sigma_q
    key = (w.V, float(w.sigma_p), float(w.target_accept))
    if key not in DRAFT_SIGMA_Q:
        raise KeyError(f"no calibrated sigma_q for {key}")
    return DRAFT_SIGMA_Q[key]


# The workloads of the benchmark suite.
TINY = Workload("tiny_f32", B=1, Hq=4, Hkv=1, d=64, N=2, L_lo=128, L_hi=128,
                V=1024, dtype="f32", sigma_p=2.0, sigma_q=0.3,
                qkv_scale=1.0 / 8.0, shuffle_pages=False)
SHAPE_8B = Workload("8b_b1", B=1, Hq=32, Hkv=8, d=128, N=4, L_lo=4096,
                    L_hi=4096, V=151936, sigma_p=3.0, target_accept=0.9)
C64 = Workload("c64_stationary", B=64, Hq=32, Hkv=8, d=128, N=4, L_lo=1024,
               L_hi=8192, V=151936, sigma_p=3.0, target_accept=0.9,
               steps=100)
SHAPE_32B = Workload("32b_b32", B=32, Hq=64, Hkv=8, d=128, N=8, L_lo=16384,
                     L_hi=16384, V=151936, sigma_p=3.0, target_accept=0.7,
                     D=5120)


# The C=64 step with the LM head in the path (hidden states in; D = 4096),
# and the same with the R-ISD gated LoRA of rank 128 at MASK rows.
C64_LM = C64.with_(name="c64_lm_head", meta={"lm_head": True})
C64_RLORA = C64.with_(name="c64_rlora",
                      meta={"lm_head": True, "lora_rank": 128,
                            "lora_scale": 2.0 ** -5})


def sweep_workload(B, N, target):
    return Workload(f"sweep_b{B}_n{N}_p{target}", B=B, Hq=32, Hkv=8, d=128,
                    N=N, L_lo=512, L_hi=16384, V=151936, sigma_p=3.0,
                    target_accept=target)


# ---------------------------------------------------------------------------
# keyed Gaussian rows


def _mix32(x):
    """32-bit integer finaliser on int64 tensors holding [0, 2^32)."""
    x = x ^ (x >> 16)
    x = (x * _MIX) & _M32
    x = x ^ (x >> 16)
    x = (x * _MIX) & _M32
    x = x ^ (x >> 16)
    return x


def _row_keys(seed, *parts):
    """Fold integer tensors (broadcast) and a seed into one 32-bit key."""
    k = None
    for p in parts:
        p = torch.as_tensor(p).to(torch.int64) & _M32
        k = _mix32(p) if k is None else _mix32(k ^ _mix32(p + 0x3C6EF372))
    return _mix32(k ^ (int(seed) & _M32)) ^ _mix32(
        torch.full_like(k, (int(seed) >> 32) & _M32) + 0x1B873593)


def keyed_normal(keys, V, device, chunk_rows=64):
    """Standard-normal rows [R][V] (float32), a pure function of the keys."""
    keys = keys.to(device=device, dtype=torch.int64).reshape(-1)
    R = keys.numel()
    out = torch.empty(R, V, dtype=torch.float32, device=device)
    col = torch.arange(V, device=device, dtype=torch.int64)
    for r0 in range(0, R, chunk_rows):
        k = keys[r0:r0 + chunk_rows, None]
        h = _mix32(k ^ _mix32(col[None, :] * 2 + 1))
        a = _mix32(h ^ 0x68E31DA4)
        b = _mix32(h ^ 0x5B2F4E1D)
        u1 = (a.to(torch.float64) + 0.5) * (1.0 / 4294967296.0)
        u2 = (b.to(torch.float64) + 0.5) * (1.0 / 4294967296.0)
        z = torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * math.pi * u2)
        out[r0:r0 + chunk_rows] = z.to(torch.float32)
    return out


def peak_token(seed, b, pos, V):
    """The keyed token a peaked row of (b, pos) boosts."""
    return _row_keys(seed ^ 0x2545F491, b, pos, 7) % V


def logits_rows(seed, b, pos, mask_step, V, sigma_p, sigma_q, device,
                peak=0.0):
    """Logits rows for (sequence b, absolute position pos) pairs.

    ``mask_step`` is -1 for a clean (verify) row and the step index for a
    MASK (draft) row.  ``peak`` is added to the logit of ``peak_token``.
    Returns float32 [R][V].
    """
    b = torch.as_tensor(b, device=device).reshape(-1).to(torch.int64)
    pos = torch.as_tensor(pos, device=device).reshape(-1).to(torch.int64)
    ms = torch.as_tensor(mask_step, device=device).reshape(-1).to(torch.int64)
    ms = ms.expand_as(pos) if ms.numel() == 1 else ms
    base = sigma_p * keyed_normal(_row_keys(seed, b, pos, 0), V, device)
    is_mask = ms >= 0
    if sigma_q != 0.0 and bool(is_mask.any()):
        idx = torch.nonzero(is_mask).reshape(-1)
        noise = keyed_normal(
            _row_keys(seed ^ 0x7F4A7C15, b[idx], pos[idx], ms[idx] + 1),
            V, device)
        base[idx] += sigma_q * noise
    if peak != 0.0:
        tok = peak_token(seed, b, pos, V)
        base[torch.arange(base.shape[0], device=device), tok] += peak
    return base


def step_logits(w, seed, seq_len, n_pending, step, device, dtype=None):
    """logits_cur [B][K][V] for one step given the sequences' state.

    Row r of sequence b scores position L_b + r + 1; rows r >= n_b are
    MASK rows (drafting), the others clean.
    """
    dtype = dtype or w.torch_dtype
    B, K, V = w.B, w.K, w.V
    L = torch.as_tensor(seq_len, device=device).to(torch.int64)
    n = torch.as_tensor(n_pending, device=device).to(torch.int64)
    r = torch.arange(K, device=device, dtype=torch.int64)
    bb = torch.arange(B, device=device, dtype=torch.int64)[:, None].expand(B, K)
    pos = L[:, None] + r[None, :] + 1
    ms = torch.where(r[None, :] >= n[:, None],
                     torch.full_like(pos, int(step)), torch.full_like(pos, -1))
    rows = logits_rows(seed, bb.reshape(-1), pos.reshape(-1), ms.reshape(-1),
                       V, w.sigma_p, draft_sigma(w), device, peak=w.peak)
    return rows.reshape(B, K, V).to(dtype)


# ---------------------------------------------------------------------------
# attention inputs and the paged cache


def prefix_lengths(w, seed):
    g = torch.Generator().manual_seed(int(seed) * 7919 + 17)
    if w.L_lo == w.L_hi:
        return torch.full((w.B,), w.L_lo, dtype=torch.int32)
    return torch.randint(w.L_lo, w.L_hi + 1, (w.B,), generator=g,
                         dtype=torch.int64).to(torch.int32)


def make_cache(w, seed, device, seq_len=None, max_len=None):
    """A paged KV cache holding the committed prefixes.

    Returns a dict: k_cache, v_cache [P][Hkv][16][d]; page_table int32
    [B][max_pages]; seq_len int32 [B]; free_stack int32 [P]; free_top
    int32 [1].  Physical pages are a seeded permutation when
    ``shuffle_pages`` (else in order); every slot of the pool holds seeded
    values, so unused slots are finite.
    """
    if seq_len is None:
        seq_len = prefix_lengths(w, seed)
    seq_len = torch.as_tensor(seq_len, dtype=torch.int32).cpu()
    growth = w.steps * w.N + w.K
    if max_len is None:
        max_len = int(seq_len.max()) + growth
    max_pages = (max_len + PAGE_SIZE - 1) // PAGE_SIZE
    owned = [(int(L) + PAGE_SIZE - 1) // PAGE_SIZE for L in seq_len]
    grow = sum((int(L) + growth + PAGE_SIZE - 1) // PAGE_SIZE - o
               for L, o in zip(seq_len, owned))
    P = sum(owned) + grow + w.spare_pages
    gen = torch.Generator().manual_seed(int(seed) * 104729 + 3)
    perm = (torch.randperm(P, generator=gen) if w.shuffle_pages
            else torch.arange(P))
    page_table = torch.full((w.B, max_pages), -1, dtype=torch.int32)
    at = 0
    for b, o in enumerate(owned):
        page_table[b, :o] = perm[at:at + o].to(torch.int32)
        at += o
    # The free stack pops from the top (highest index) first.
    free = perm[at:].flip(0).to(torch.int32)
    free_stack = torch.full((P,), -1, dtype=torch.int32)
    free_stack[:free.numel()] = free
    free_top = torch.tensor([free.numel()], dtype=torch.int32)
    dev_gen = torch.Generator(device=device).manual_seed(int(seed) * 31 + 1)
    scale = w.qkv_scale if w.qkv_scale is not None else 1.0 / math.sqrt(w.d)
    shape = (P, w.Hkv, PAGE_SIZE, w.d)
    k_cache = (torch.randn(shape, generator=dev_gen, device=device) * scale
               ).to(w.torch_dtype)
    v_cache = torch.randn(shape, generator=dev_gen, device=device
                          ).to(w.torch_dtype)
    return dict(k_cache=k_cache, v_cache=v_cache,
                page_table=page_table.to(device), seq_len=seq_len.to(device),
                free_stack=free_stack.to(device), free_top=free_top.to(device))


def make_stride(w, seed, step, device, sharp=False):
    """Q [B][K][Hq][d] and staged K/V [B][K][Hkv][d] of one stride.

    Q and K are N(0,1) scaled by ``qkv_scale`` (1/sqrt(d) by default), V is
    N(0,1).  ``sharp`` leaves Q and K unscaled so that attention is far
    from uniform.
    """
    g = torch.Generator(device=device).manual_seed(
        int(seed) * 1000003 + int(step) * 7 + 5)
    scale = 1.0 if sharp else (w.qkv_scale if w.qkv_scale is not None
                               else 1.0 / math.sqrt(w.d))
    q = torch.randn((w.B, w.K, w.Hq, w.d), generator=g, device=device) * scale
    k = torch.randn((w.B, w.K, w.Hkv, w.d), generator=g, device=device) * scale
    v = torch.randn((w.B, w.K, w.Hkv, w.d), generator=g, device=device)
    dt = w.torch_dtype
    return q.to(dt), k.to(dt), v.to(dt)


def initial_state(w, seed, device):
    """Step-0 state: every sequence holds one exact token (R mode)."""
    g = torch.Generator().manual_seed(int(seed) * 65537 + 11)
    pending = torch.full((w.B, w.N), -1, dtype=torch.int32)
    pending[:, 0] = torch.randint(0, w.V, (w.B,), generator=g,
                                  dtype=torch.int64).to(torch.int32)
    n_pending = torch.ones(w.B, dtype=torch.int32)
    q_row = torch.full((w.B, w.N), -1, dtype=torch.int32)
    q_stats = torch.zeros((w.B, w.N, 2), dtype=torch.float32)
    return dict(pending=pending.to(device), n_pending=n_pending.to(device),
                q_row=q_row.to(device), q_stats=q_stats.to(device))


# ---------------------------------------------------------------------------
# LM-head inputs: final hidden states, the output embedding, LoRA factors.
#
# Every tensor is an integer-valued array scaled by a power of two: hidden
# states h_int * 2^-5 with |h_int| <= 63, weights w_int * 2^-6 with
# |w_int| <= 31 (both exact in bfloat16).  Every product is then an integer
# multiple of 2^-11 and any partial sum of up to 8192 of them stays below
# 2^24 such units, so the contraction is exact in float32 in any summation
# order, and the float64 oracle and the tensor cores round the same exact
# value to bfloat16.
#
# The hidden state of (sequence b, position t) is keyed like the logits rows
# above, so a position's verify logits h W^T are the same whenever it is
# verified; a MASK row adds integer noise keyed by (b, t, step).  The scales
# follow from the logits model: logit std = sqrt(D) * std(h_int) *
# std(w_int) * 2^-11 = sigma_p, and the MASK noise gives the logits a
# Gaussian perturbation of std sigma_q (the acceptance calibration above).

H_SHIFT = 5
W_SHIFT = 6
H_LIM = 63
W_LIM = 31
W_SIGMA = 8.0


def _int_rows(keys, cols, sigma, lim, device):
    z = keyed_normal(keys, cols, device)
    return torch.clamp(torch.round(sigma * z), -lim, lim)


def lm_weight(seed, V, D, device, rows=None):
    """Output embedding rows [len(rows) or V][D] (float32, bf16-exact)."""
    v = torch.arange(V) if rows is None else torch.as_tensor(rows)
    keys = _row_keys(int(seed) ^ 0x51ED270B, v, 11)
    out = torch.empty((v.numel(), D), dtype=torch.float32, device=device)
    for r0 in range(0, v.numel(), 8192):
        out[r0:r0 + 8192] = _int_rows(keys[r0:r0 + 8192], D, W_SIGMA, W_LIM,
                                      device)
    return out * 2.0 ** -W_SHIFT


def hidden_scales(w):
    """(std of h_int, std of the MASK noise before rounding)."""
    unit = 2.0 ** (H_SHIFT + W_SHIFT) / (math.sqrt(w.D) * W_SIGMA)
    s_h = w.sigma_p * unit
    noise = draft_sigma(w) * unit
    # round(s z) has variance s^2 + 1/12 for the s used here.
    s_n = math.sqrt(max(noise * noise - 1.0 / 12.0, 0.0))
    return s_h, s_n


def hidden_rows(seed, b, pos, mask_step, D, s_h, s_n, device):
    """Hidden states for (sequence b, absolute position pos) pairs;
    ``mask_step`` -1 for a clean row, else the step index.  float32 [R][D],
    bf16-exact."""
    b = torch.as_tensor(b, device=device).reshape(-1).to(torch.int64)
    pos = torch.as_tensor(pos, device=device).reshape(-1).to(torch.int64)
    ms = torch.as_tensor(mask_step, device=device).reshape(-1).to(torch.int64)
    ms = ms.expand_as(pos) if ms.numel() == 1 else ms
    h = torch.round(s_h * keyed_normal(_row_keys(seed ^ 0x2B992DDF, b, pos, 3),
                                       D, device))
    noise = torch.round(s_n * keyed_normal(
        _row_keys(seed ^ 0x68BC21EB, b, pos, ms + 1), D, device))
    h = h + torch.where(ms[:, None] >= 0, noise, torch.zeros_like(noise))
    return torch.clamp(h, -H_LIM, H_LIM) * 2.0 ** -H_SHIFT


def step_hidden(w, seed, seq_len, n_pending, step, device):
    """Final hidden states [B][K][D] of one step's strides (bf16): row r of
    sequence b is the state at position L_b + r + 1, a MASK row when
    r >= n_b."""
    B, K = w.B, w.K
    L = torch.as_tensor(seq_len, device=device).to(torch.int64)
    n = torch.as_tensor(n_pending, device=device).to(torch.int64)
    r = torch.arange(K, device=device, dtype=torch.int64)
    bb = torch.arange(B, device=device, dtype=torch.int64)[:, None].expand(B, K)
    pos = L[:, None] + r[None, :] + 1
    ms = torch.where(r[None, :] >= n[:, None],
                     torch.full_like(pos, int(step)), torch.full_like(pos, -1))
    s_h, s_n = hidden_scales(w)
    rows = hidden_rows(seed, bb.reshape(-1), pos.reshape(-1), ms.reshape(-1),
                       w.D, s_h, s_n, device)
    return rows.reshape(B, K, w.D).to(torch.bfloat16)


def lora_factors(seed, r, D, V, device, sparse=False):
    """R-ISD LoRA factors A [r][D] and B [V][r] (float32, bf16-exact).

    Dense: integer entries of std 8 scaled by 2^-6 (A) and 2^-6 (B).
    Sparse: each row j of A holds a single 1 at a keyed column, so
    (h A^T)_j is one entry of h and stays exact in bfloat16."""
    rows = torch.arange(r)
    if sparse:
        cols = _row_keys(int(seed) ^ 0x3C6EF372, rows, 5) % D
        A = torch.zeros((r, D), dtype=torch.float32, device=device)
        A[rows.to(device), cols.to(device)] = 1.0
    else:
        A = _int_rows(_row_keys(int(seed) ^ 0x3C6EF372, rows, 6), D, W_SIGMA,
                      W_LIM, device) * 2.0 ** -W_SHIFT
    keys = _row_keys(int(seed) ^ 0x1F83D9AB, torch.arange(V), 7)
    B = _int_rows(keys, r, W_SIGMA, W_LIM, device) * 2.0 ** -W_SHIFT
    return A, B
