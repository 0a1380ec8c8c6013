"""Thin ctypes binding of libisd.so over torch tensors.

Argument marshalling only: shape / dtype / device checks, ``data_ptr()``
and the current CUDA stream go to the C ABI of ``include/isd.h``; every
step of the computation runs in the library's kernels.  There is no CPU
fallback: if the library is missing the first call raises.
"""

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libisd.so")
_lib = None

# Status codes (include/isd.h).
OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_WORKSPACE = 4
ERR_POOL_EXHAUSTED = 16
ERR_PAGE_TABLE_FULL = 17
ERR_BAD_STATE = 18
ERR_BAD_PAGE = 19

PROPOSAL_SAMPLE = 0   # drafts drawn from q
PROPOSAL_ARGMAX = 1   # drafts x = argmax q
BF16 = 0
F32 = 1
PAGE_SIZE = 16

_VP = ctypes.c_void_p
_I32 = ctypes.c_int32


class AttnArgs(ctypes.Structure):
    _fields_ = [("B", _I32), ("Hq", _I32), ("Hkv", _I32), ("d", _I32),
                ("K", _I32), ("num_pages", _I32),
                ("page_table_stride", _I32), ("dtype", _I32),
                ("softmax_scale", ctypes.c_float), ("num_ctas", _I32),
                ("q", _VP), ("k_new", _VP), ("v_new", _VP), ("k_cache", _VP),
                ("v_cache", _VP), ("page_table", _VP), ("seq_len", _VP),
                ("out", _VP), ("lse", _VP), ("status", _VP),
                ("workspace", _VP), ("workspace_bytes", ctypes.c_size_t)]


class AcceptArgs(ctypes.Structure):
    _fields_ = [("B", _I32), ("N", _I32), ("K", _I32), ("V", _I32),
                ("dtype", _I32), ("step", ctypes.c_uint32),
                ("seed", ctypes.c_uint64),
                ("logits_cur", _VP), ("logits_prev", _VP), ("seq_len", _VP),
                ("pending_in", _VP), ("n_pending_in", _VP),
                ("q_row_in", _VP), ("q_stats_in", _VP),
                ("pending_out", _VP), ("n_pending_out", _VP),
                ("q_row_out", _VP), ("q_stats_out", _VP),
                ("n_commit", _VP), ("commit_tokens", _VP),
                ("row_stats", _VP), ("ratio", _VP), ("status", _VP),
                ("workspace", _VP), ("workspace_bytes", ctypes.c_size_t),
                ("step_dev", _VP), ("proposal", _I32),
                ("vocab_stats", _VP)]


class CommitArgs(ctypes.Structure):
    _fields_ = [("B", _I32), ("K", _I32), ("Hkv", _I32), ("d", _I32),
                ("num_pages", _I32), ("page_table_stride", _I32),
                ("dtype", _I32),
                ("k_new", _VP), ("v_new", _VP), ("k_cache", _VP),
                ("v_cache", _VP), ("page_table", _VP), ("seq_len", _VP),
                ("n_commit", _VP), ("free_stack", _VP), ("free_top", _VP),
                ("status", _VP), ("workspace", _VP),
                ("workspace_bytes", ctypes.c_size_t)]


class LmHeadArgs(ctypes.Structure):
    _fields_ = [("M", _I32), ("D", _I32), ("V", _I32), ("dtype", _I32),
                ("hidden", _VP), ("weight", _VP), ("logits", _VP),
                ("vocab_stats", _VP), ("lora_rank", _I32),
                ("rows_per_seq", _I32), ("lora_a", _VP), ("lora_b", _VP),
                ("n_pending", _VP), ("lora_scale", ctypes.c_float),
                ("status", _VP), ("workspace", _VP),
                ("workspace_bytes", ctypes.c_size_t)]


# Every symbol include/isd.h declares, with (restype, argtypes).
SIGNATURES = {
    "isd_attn_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(AttnArgs)]),
    "isd_attn_strided": (ctypes.c_int, [ctypes.POINTER(AttnArgs), _VP]),
    "isd_accept_workspace_bytes": (ctypes.c_size_t,
                                   [ctypes.POINTER(AcceptArgs)]),
    "isd_accept_resample": (ctypes.c_int, [ctypes.POINTER(AcceptArgs), _VP]),
    "isd_accept_resample_static": (ctypes.c_int,
                                   [ctypes.POINTER(AcceptArgs), _VP]),
    "isd_commit_workspace_bytes": (ctypes.c_size_t,
                                   [ctypes.POINTER(CommitArgs)]),
    "isd_kv_commit": (ctypes.c_int, [ctypes.POINTER(CommitArgs), _VP]),
    "isd_accept_commit": (ctypes.c_int, [ctypes.POINTER(AcceptArgs),
                                         ctypes.POINTER(CommitArgs), _VP]),
    "isd_lm_head_workspace_bytes": (ctypes.c_size_t,
                                    [ctypes.POINTER(LmHeadArgs)]),
    "isd_vocab_stats_bytes": (ctypes.c_size_t, [_I32, _I32]),
    "isd_lm_head_launches": (ctypes.c_int, [ctypes.POINTER(LmHeadArgs)]),
    "isd_lm_head": (ctypes.c_int, [ctypes.POINTER(LmHeadArgs), _VP]),
    "isd_abi_version": (ctypes.c_int, []),
    "isd_status_string": (ctypes.c_char_p, [ctypes.c_int]),
}


class IsdError(RuntimeError):
    def __init__(self, code, what):
        self.code = code
        super().__init__(f"{what}: {status_string(code)} ({code})")


def lib_path():
    return _LIB_PATH


def lib():
    """Load libisd.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(
                f"{_LIB_PATH} is missing; build it with "
                "`python -m introspective_strided_decoding_b200.build`")
        handle = ctypes.CDLL(_LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def status_string(code):
    return lib().isd_status_string(int(code)).decode()


def abi_version():
    return lib().isd_abi_version()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t):
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _check(t, name, shape=None, dtype=None, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, "
                         f"expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _raise(rc, what):
    if rc != OK:
        raise IsdError(rc, what)


# ---------------------------------------------------------------- attention
def attn_args(q, k_new, v_new, k_cache, v_cache, page_table, seq_len, out,
              lse=None, status=None, softmax_scale=None, workspace=None,
              num_ctas=0):
    """Validate tensors and fill an AttnArgs (no launch)."""
    B, K, Hq, d = q.shape
    Hkv = k_new.shape[2]
    P = k_cache.shape[0]
    dev, dt = q.device, q.dtype
    _check(q, "q", dtype=dt)
    _check(k_new, "k_new", (B, K, Hkv, d), dt, dev)
    _check(v_new, "v_new", (B, K, Hkv, d), dt, dev)
    _check(k_cache, "k_cache", (P, Hkv, PAGE_SIZE, d), dt, dev)
    _check(v_cache, "v_cache", (P, Hkv, PAGE_SIZE, d), dt, dev)
    _check(page_table, "page_table", dtype=torch.int32, device=dev)
    _check(seq_len, "seq_len", (B,), torch.int32, dev)
    _check(out, "out", (B, K, Hq, d), dt, dev)
    if page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be [B][max_pages]")
    if lse is not None:
        _check(lse, "lse", (B, K, Hq), torch.float32, dev)
    if status is not None:
        _check(status, "status", (1,), torch.int32, dev)
    scale = float(softmax_scale) if softmax_scale is not None \
        else 1.0 / float(d) ** 0.5
    a = AttnArgs(B=B, Hq=Hq, Hkv=Hkv, d=d, K=K, num_pages=P,
                 page_table_stride=page_table.shape[1], dtype=_dtype_code(q),
                 softmax_scale=scale, num_ctas=int(num_ctas),
                 q=_ptr(q), k_new=_ptr(k_new), v_new=_ptr(v_new),
                 k_cache=_ptr(k_cache), v_cache=_ptr(v_cache),
                 page_table=_ptr(page_table), seq_len=_ptr(seq_len),
                 out=_ptr(out), lse=_ptr(lse), status=_ptr(status),
                 workspace=_ptr(workspace),
                 workspace_bytes=0 if workspace is None else
                 workspace.numel() * workspace.element_size())
    return a


def attn_workspace_bytes(args):
    return int(lib().isd_attn_workspace_bytes(ctypes.byref(args)))


def attn_strided(q, k_new, v_new, k_cache, v_cache, page_table, seq_len,
                 out=None, lse=None, status=None, softmax_scale=None,
                 workspace=None, num_ctas=0, stream=None):
    """isd_attn_strided on torch tensors; returns ``out``."""
    if out is None:
        out = torch.empty_like(q)
    a = attn_args(q, k_new, v_new, k_cache, v_cache, page_table, seq_len, out,
                  lse, status, softmax_scale, workspace, num_ctas)
    if workspace is None:
        need = attn_workspace_bytes(a)
        workspace = torch.empty(max(need, 16), dtype=torch.uint8,
                                device=q.device)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel()
    _raise(lib().isd_attn_strided(ctypes.byref(a), _stream(stream)),
           "isd_attn_strided")
    return out


# ------------------------------------------------------------------ accept
STATE_KEYS = ("pending", "n_pending", "q_row", "q_stats")


def new_state(B, N, device):
    return dict(pending=torch.full((B, N), -1, dtype=torch.int32,
                                   device=device),
                n_pending=torch.ones(B, dtype=torch.int32, device=device),
                q_row=torch.full((B, N), -1, dtype=torch.int32,
                                 device=device),
                q_stats=torch.zeros((B, N, 2), dtype=torch.float32,
                                    device=device))


def accept_args(logits_cur, logits_prev, seq_len, state_in, state_out,
                n_commit, commit_tokens, seed, step, workspace=None,
                row_stats=None, ratio=None, status=None, step_dev=None,
                proposal=None, vocab_stats=None):
    B, K, V = logits_cur.shape
    N = K // 2
    dev, dt = logits_cur.device, logits_cur.dtype
    _check(logits_cur, "logits_cur", dtype=dt)
    _check(logits_prev, "logits_prev", (B, K, V), dt, dev)
    _check(seq_len, "seq_len", (B,), torch.int32, dev)
    for st, tag in ((state_in, "in"), (state_out, "out")):
        _check(st["pending"], f"pending_{tag}", (B, N), torch.int32, dev)
        _check(st["n_pending"], f"n_pending_{tag}", (B,), torch.int32, dev)
        _check(st["q_row"], f"q_row_{tag}", (B, N), torch.int32, dev)
        _check(st["q_stats"], f"q_stats_{tag}", (B, N, 2), torch.float32, dev)
    _check(n_commit, "n_commit", (B,), torch.int32, dev)
    _check(commit_tokens, "commit_tokens", (B, N), torch.int32, dev)
    if row_stats is not None:
        _check(row_stats, "row_stats", (B, K, 2), torch.float32, dev)
    if ratio is not None:
        _check(ratio, "ratio", (B, N), torch.float32, dev)
    if status is not None:
        _check(status, "status", (1,), torch.int32, dev)
    if step_dev is not None:
        _check(step_dev, "step_dev", (1,), torch.int32, dev)
    if vocab_stats is not None:
        _check(vocab_stats, "vocab_stats", (vocab_stats_bytes(B * K, V),),
               torch.uint8, dev)
    return AcceptArgs(
        B=B, N=N, K=K, V=V, dtype=_dtype_code(logits_cur),
        step=int(step) & 0xFFFFFFFF, seed=int(seed) & 0xFFFFFFFFFFFFFFFF,
        logits_cur=_ptr(logits_cur), logits_prev=_ptr(logits_prev),
        seq_len=_ptr(seq_len), pending_in=_ptr(state_in["pending"]),
        n_pending_in=_ptr(state_in["n_pending"]),
        q_row_in=_ptr(state_in["q_row"]), q_stats_in=_ptr(state_in["q_stats"]),
        pending_out=_ptr(state_out["pending"]),
        n_pending_out=_ptr(state_out["n_pending"]),
        q_row_out=_ptr(state_out["q_row"]),
        q_stats_out=_ptr(state_out["q_stats"]),
        n_commit=_ptr(n_commit), commit_tokens=_ptr(commit_tokens),
        row_stats=_ptr(row_stats), ratio=_ptr(ratio), status=_ptr(status),
        workspace=_ptr(workspace),
        workspace_bytes=0 if workspace is None else
        workspace.numel() * workspace.element_size(),
        step_dev=_ptr(step_dev),
        proposal=PROPOSAL_SAMPLE if proposal is None else int(proposal),
        vocab_stats=_ptr(vocab_stats))


def accept_workspace_bytes(args):
    return int(lib().isd_accept_workspace_bytes(ctypes.byref(args)))


def accept_resample(logits_cur, logits_prev, seq_len, state_in, state_out,
                    n_commit, commit_tokens, seed, step, workspace=None,
                    row_stats=None, ratio=None, status=None, stream=None,
                    proposal=None, vocab_stats=None):
    """isd_accept_resample on torch tensors (state dicts from new_state).
    ``proposal``: PROPOSAL_SAMPLE (default) or PROPOSAL_ARGMAX;
    ``vocab_stats``: the statistics buffer ``lm_head`` wrote for
    ``logits_cur`` (optional)."""
    a = accept_args(logits_cur, logits_prev, seq_len, state_in, state_out,
                    n_commit, commit_tokens, seed, step, workspace, row_stats,
                    ratio, status, proposal=proposal, vocab_stats=vocab_stats)
    if workspace is None:
        workspace = torch.empty(accept_workspace_bytes(a), dtype=torch.uint8,
                                device=logits_cur.device)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel()
    _raise(lib().isd_accept_resample(ctypes.byref(a), _stream(stream)),
           "isd_accept_resample")


ACCEPT_STATIC_SCRATCH = 16 << 20


def accept_resample_static(logits_cur, logits_prev, seq_len, state_in,
                           state_out, n_commit, commit_tokens, seed, step,
                           row_stats=None, ratio=None, status=None,
                           stream=None, proposal=None):
    """isd_accept_resample_static: the accept step without a caller
    workspace, for callers that cannot allocate device memory (its scratch
    is a fixed buffer inside the library; see include/isd.h)."""
    a = accept_args(logits_cur, logits_prev, seq_len, state_in, state_out,
                    n_commit, commit_tokens, seed, step, None, row_stats,
                    ratio, status, proposal=proposal)
    _raise(lib().isd_accept_resample_static(ctypes.byref(a),
                                            _stream(stream)),
           "isd_accept_resample_static")


# ------------------------------------------------------------------ commit
def commit_args(k_new, v_new, k_cache, v_cache, page_table, seq_len, n_commit,
                free_stack, free_top, status, workspace=None):
    B, K, Hkv, d = k_new.shape
    P = k_cache.shape[0]
    dev, dt = k_new.device, k_new.dtype
    _check(k_new, "k_new", dtype=dt)
    _check(v_new, "v_new", (B, K, Hkv, d), dt, dev)
    _check(k_cache, "k_cache", (P, Hkv, PAGE_SIZE, d), dt, dev)
    _check(v_cache, "v_cache", (P, Hkv, PAGE_SIZE, d), dt, dev)
    _check(page_table, "page_table", dtype=torch.int32, device=dev)
    _check(seq_len, "seq_len", (B,), torch.int32, dev)
    _check(n_commit, "n_commit", (B,), torch.int32, dev)
    _check(free_stack, "free_stack", (P,), torch.int32, dev)
    _check(free_top, "free_top", (1,), torch.int32, dev)
    _check(status, "status", (1,), torch.int32, dev)
    return CommitArgs(
        B=B, K=K, Hkv=Hkv, d=d, num_pages=P,
        page_table_stride=page_table.shape[1], dtype=_dtype_code(k_new),
        k_new=_ptr(k_new), v_new=_ptr(v_new), k_cache=_ptr(k_cache),
        v_cache=_ptr(v_cache), page_table=_ptr(page_table),
        seq_len=_ptr(seq_len), n_commit=_ptr(n_commit),
        free_stack=_ptr(free_stack), free_top=_ptr(free_top),
        status=_ptr(status), workspace=_ptr(workspace),
        workspace_bytes=0 if workspace is None else
        workspace.numel() * workspace.element_size())


def commit_workspace_bytes(args):
    return int(lib().isd_commit_workspace_bytes(ctypes.byref(args)))


def kv_commit(k_new, v_new, k_cache, v_cache, page_table, seq_len, n_commit,
              free_stack, free_top, status, workspace=None, stream=None):
    """isd_kv_commit on torch tensors (updates the cache state in place)."""
    a = commit_args(k_new, v_new, k_cache, v_cache, page_table, seq_len,
                    n_commit, free_stack, free_top, status, workspace)
    if workspace is None:
        # The commit workspace is a counter that must start at zero.
        workspace = torch.zeros(commit_workspace_bytes(a), dtype=torch.uint8,
                                device=k_new.device)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel()
    _raise(lib().isd_kv_commit(ctypes.byref(a), _stream(stream)),
           "isd_kv_commit")


def accept_commit(acc_args, com_args, stream=None):
    """isd_accept_commit on prepared argument structs (from accept_args and
    commit_args, each with its workspace set): the accept step, then the
    commit of its decisions with the draws running beside it."""
    _raise(lib().isd_accept_commit(ctypes.byref(acc_args),
                                   ctypes.byref(com_args), _stream(stream)),
           "isd_accept_commit")


# ----------------------------------------------------------------- LM head
def vocab_stats_bytes(M, V):
    return int(lib().isd_vocab_stats_bytes(int(M), int(V)))


def new_vocab_stats(M, V, device):
    """A buffer for the sub-chunk statistics of M rows of V entries."""
    return torch.empty(vocab_stats_bytes(M, V), dtype=torch.uint8,
                       device=device)


def vocab_stats_view(buf, M, V):
    """(csum f64 [M][C], cmax f32 [M][C], cidx int32 [M][C]) views of a
    statistics buffer (its layout in include/isd.h)."""
    C = (V + 2047) // 2048
    n = M * C
    csum = buf[:n * 8].view(torch.float64).view(M, C)
    cmax = buf[n * 8:n * 12].view(torch.float32).view(M, C)
    cidx = buf[n * 12:n * 16].view(torch.int32).view(M, C)
    return csum, cmax, cidx


def lm_head_args(hidden, weight, logits, vocab_stats=None, lora_a=None,
                 lora_b=None, lora_scale=1.0, n_pending=None, rows_per_seq=0,
                 status=None, workspace=None):
    M, D = hidden.shape
    V = weight.shape[0]
    dev = hidden.device
    _check(hidden, "hidden", (M, D), torch.bfloat16, dev)
    _check(weight, "weight", (V, D), torch.bfloat16, dev)
    _check(logits, "logits", (M, V), torch.bfloat16, dev)
    r = 0
    if lora_a is not None:
        r = lora_a.shape[0]
        _check(lora_a, "lora_a", (r, D), torch.bfloat16, dev)
        _check(lora_b, "lora_b", (V, r), torch.bfloat16, dev)
        _check(n_pending, "n_pending", (M // max(rows_per_seq, 1),),
               torch.int32, dev)
    if vocab_stats is not None:
        _check(vocab_stats, "vocab_stats", (vocab_stats_bytes(M, V),),
               torch.uint8, dev)
    if status is not None:
        _check(status, "status", (1,), torch.int32, dev)
    return LmHeadArgs(
        M=M, D=D, V=V, dtype=BF16, hidden=_ptr(hidden), weight=_ptr(weight),
        logits=_ptr(logits), vocab_stats=_ptr(vocab_stats), lora_rank=r,
        rows_per_seq=int(rows_per_seq), lora_a=_ptr(lora_a),
        lora_b=_ptr(lora_b), n_pending=_ptr(n_pending),
        lora_scale=float(lora_scale), status=_ptr(status),
        workspace=_ptr(workspace),
        workspace_bytes=0 if workspace is None else
        workspace.numel() * workspace.element_size())


def lm_head_workspace_bytes(args):
    return int(lib().isd_lm_head_workspace_bytes(ctypes.byref(args)))


def lm_head_launches(args):
    """Kernels isd_lm_head launches for ``args`` on the current device."""
    return int(lib().isd_lm_head_launches(ctypes.byref(args)))


def lm_head(hidden, weight, logits, vocab_stats=None, lora_a=None,
            lora_b=None, lora_scale=1.0, n_pending=None, rows_per_seq=0,
            status=None, workspace=None, stream=None):
    """isd_lm_head on torch tensors: logits = hidden . weight^T (+ the gated
    LoRA at MASK rows), optionally with the vocabulary statistics."""
    a = lm_head_args(hidden, weight, logits, vocab_stats, lora_a, lora_b,
                     lora_scale, n_pending, rows_per_seq, status, workspace)
    if workspace is None:
        workspace = torch.empty(lm_head_workspace_bytes(a), dtype=torch.uint8,
                                device=hidden.device)
        a.workspace = _ptr(workspace)
        a.workspace_bytes = workspace.numel()
    _raise(lib().isd_lm_head(ctypes.byref(a), _stream(stream)), "isd_lm_head")
