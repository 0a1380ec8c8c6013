"""The C ABI: libisd.so builds, loads and exports every symbol include/isd.h
declares; host-side validation rejects bad arguments before any launch.
These run without a GPU (no call here reaches a kernel or the device)."""

import ctypes
import os
import re
import subprocess

import pytest

from introspective_strided_decoding_b200 import build, isd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "isd.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return isd.lib()


def header_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w \*]*?\b(isd_\w+)\s*\(", text,
                                 flags=re.M)))


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("isd_attn_strided", "isd_accept_resample", "isd_kv_commit",
                 "isd_attn_workspace_bytes", "isd_accept_workspace_bytes",
                 "isd_commit_workspace_bytes", "isd_abi_version",
                 "isd_status_string"):
        assert name in fns
    assert set(fns) == set(isd.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", isd.lib_path()],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (isd_\w+)", out))
    for name in header_functions():
        assert name in exported
        assert getattr(lib, name) is not None


def test_abi_version_and_status_strings(lib):
    assert isd.abi_version() == 4
    assert isd.status_string(isd.ERR_POOL_EXHAUSTED) == "KV page pool exhausted"
    assert isd.status_string(12345) == "unknown status"


def _attn_args(**kw):
    base = dict(B=1, Hq=32, Hkv=8, d=128, K=8, num_pages=10,
                page_table_stride=4, dtype=isd.BF16, softmax_scale=0.088,
                num_ctas=0)
    base.update(kw)
    return isd.AttnArgs(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(B=0), isd.ERR_INVALID_ARG),
    (dict(Hq=30), isd.ERR_INVALID_ARG),            # Hq % Hkv != 0
    (dict(softmax_scale=0.0), isd.ERR_INVALID_ARG),
    (dict(num_ctas=-1), isd.ERR_INVALID_ARG),
    (dict(num_ctas=1025), isd.ERR_INVALID_ARG),     # at most 1024 CTAs
    (dict(d=96), isd.ERR_UNSUPPORTED),              # bf16 path: d 128
    (dict(d=64), isd.ERR_UNSUPPORTED),
    (dict(K=16, Hq=96, Hkv=8), isd.ERR_UNSUPPORTED),  # K*g = 192 rows
    (dict(K=32, Hq=8), isd.ERR_UNSUPPORTED),        # K above a page
    (dict(dtype=7), isd.ERR_INVALID_ARG),
    (dict(dtype=isd.F32, d=48), isd.ERR_UNSUPPORTED),
    (dict(), isd.ERR_INVALID_ARG),                  # null tensors
])
def test_attn_host_validation(lib, kw, code):
    a = _attn_args(**kw)
    assert lib.isd_attn_strided(ctypes.byref(a), None) == code


def test_attn_workspace_query_rejects_bad_shapes(lib):
    assert lib.isd_attn_workspace_bytes(ctypes.byref(_attn_args(d=96))) == 0
    assert lib.isd_attn_workspace_bytes(None) == 0


@pytest.mark.parametrize("kw,code", [
    (dict(N=1, K=2), isd.ERR_INVALID_ARG),
    (dict(K=9), isd.ERR_INVALID_ARG),               # K must be 2N
    (dict(N=17, K=34), isd.ERR_UNSUPPORTED),
    (dict(V=0), isd.ERR_INVALID_ARG),
    (dict(proposal=2), isd.ERR_INVALID_ARG),        # sample (0) or argmax (1)
    (dict(), isd.ERR_INVALID_ARG),                  # null tensors
])
def test_accept_host_validation(lib, kw, code):
    base = dict(B=4, N=4, K=8, V=1024, dtype=isd.BF16, step=0, seed=0)
    base.update(kw)
    a = isd.AcceptArgs(**base)
    assert lib.isd_accept_resample(ctypes.byref(a), None) == code


def test_accept_rejects_in_place_state(lib):
    fake = ctypes.c_void_p(0x10000)
    a = isd.AcceptArgs(B=1, N=2, K=4, V=64, dtype=isd.F32, logits_cur=fake,
                       logits_prev=fake, seq_len=fake, pending_in=fake,
                       n_pending_in=fake, q_row_in=fake, q_stats_in=fake,
                       pending_out=fake, n_pending_out=ctypes.c_void_p(0x20000),
                       q_row_out=ctypes.c_void_p(0x30000),
                       q_stats_out=ctypes.c_void_p(0x40000), n_commit=fake,
                       commit_tokens=fake)
    assert lib.isd_accept_resample(ctypes.byref(a), None) == isd.ERR_INVALID_ARG


def test_commit_host_validation(lib):
    a = isd.CommitArgs(B=2, K=8, Hkv=8, d=128, num_pages=4,
                       page_table_stride=2, dtype=isd.BF16)
    assert lib.isd_kv_commit(ctypes.byref(a), None) == isd.ERR_INVALID_ARG
    a.d = 4                                          # 8-byte rows
    assert lib.isd_kv_commit(ctypes.byref(a), None) == isd.ERR_UNSUPPORTED
    a.d = 128
    a.B = 32769                                      # above 1024 CTAs x 32
    assert lib.isd_kv_commit(ctypes.byref(a), None) == isd.ERR_UNSUPPORTED
    assert lib.isd_commit_workspace_bytes(ctypes.byref(a)) == 0


def _fake_accept_args(**kw):
    """Accept arguments whose pointers are distinct, aligned and never
    dereferenced (every call below is refused on the host)."""
    ptr = iter(range(0x100000, 0x100000 + 0x10000 * 40, 0x10000))
    fields = dict(logits_cur=None, logits_prev=None, seq_len=None,
                  pending_in=None, n_pending_in=None, q_row_in=None,
                  q_stats_in=None, pending_out=None, n_pending_out=None,
                  q_row_out=None, q_stats_out=None, n_commit=None,
                  commit_tokens=None)
    for k in fields:
        fields[k] = ctypes.c_void_p(next(ptr))
    fields.update(kw)
    return isd.AcceptArgs(**fields)


def test_static_scratch_rejects_problems_above_its_limit(lib):
    """The allocation-free accept entry point refuses, before any CUDA call,
    a problem whose scratch would exceed its fixed buffer."""
    a = _fake_accept_args(B=8192, N=16, K=32, V=151936, dtype=isd.BF16)
    assert lib.isd_accept_workspace_bytes(ctypes.byref(a)) > \
        isd.ACCEPT_STATIC_SCRATCH
    assert lib.isd_accept_resample_static(ctypes.byref(a), None) == \
        isd.ERR_WORKSPACE


def test_static_scratch_checks_arguments_like_the_workspace_call(lib):
    """Both accept entry points report the same error for the same bad
    arguments, argument errors before the size limit."""
    cases = [
        dict(B=8192, N=16, K=32, V=151936, dtype=isd.BF16,
             logits_cur=None),                       # null and oversized
        dict(B=4, N=1, K=2, V=64, dtype=isd.BF16),   # N < 2
        dict(B=4, N=4, K=8, V=64, dtype=isd.BF16, proposal=5),
    ]
    for kw in cases:
        a = _fake_accept_args(**kw)
        want = lib.isd_accept_resample(ctypes.byref(a), None)
        assert want == isd.ERR_INVALID_ARG
        assert lib.isd_accept_resample_static(ctypes.byref(a), None) == want
    a = _fake_accept_args(B=8192, N=16, K=32, V=151936, dtype=isd.BF16)
    a.q_stats_out = a.q_stats_in                     # in-place state
    assert lib.isd_accept_resample_static(ctypes.byref(a), None) == \
        isd.ERR_INVALID_ARG


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(isd, "_lib", None)
    monkeypatch.setattr(isd, "_LIB_PATH", str(tmp_path / "libisd.so"))
    with pytest.raises(RuntimeError, match="missing"):
        isd.lib()


# ----------------------------------------------------------------- LM head
_FAKE = 1 << 20          # a 16-byte aligned fake device address (never used)


def _lm_args(**kw):
    base = dict(M=512, D=4096, V=151936, dtype=isd.BF16, hidden=_FAKE,
                weight=_FAKE * 2, logits=_FAKE * 3, lora_rank=0,
                rows_per_seq=8, lora_scale=1.0)
    base.update(kw)
    return isd.LmHeadArgs(**base)


@pytest.mark.parametrize("kw,code", [
    (dict(M=0), isd.ERR_INVALID_ARG),
    (dict(D=0), isd.ERR_INVALID_ARG),
    (dict(lora_rank=-64), isd.ERR_INVALID_ARG),
    (dict(dtype=isd.F32), isd.ERR_UNSUPPORTED),      # bf16 tensor cores only
    (dict(D=4000), isd.ERR_UNSUPPORTED),             # D a multiple of 64
    (dict(V=151937), isd.ERR_UNSUPPORTED),           # V a multiple of 8
    (dict(lora_rank=96), isd.ERR_UNSUPPORTED),       # rank a multiple of 64
    (dict(lora_rank=320), isd.ERR_UNSUPPORTED),      # rank at most 256
    (dict(lora_rank=128, rows_per_seq=0), isd.ERR_INVALID_ARG),
    (dict(lora_rank=128, rows_per_seq=7), isd.ERR_INVALID_ARG),  # M % K
    (dict(hidden=None), isd.ERR_INVALID_ARG),
    (dict(lora_rank=128), isd.ERR_INVALID_ARG),      # LoRA pointers missing
    (dict(hidden=_FAKE + 8), isd.ERR_INVALID_ARG),   # not 16-byte aligned
    (dict(logits=_FAKE), isd.ERR_INVALID_ARG),       # logits alias hidden
    (dict(), isd.ERR_WORKSPACE),                     # no workspace
])
def test_lm_head_host_validation(lib, kw, code):
    a = _lm_args(**kw)
    assert lib.isd_lm_head(ctypes.byref(a), None) == code


def test_lm_head_workspace_and_stats_sizes(lib):
    a = _lm_args()
    plain = lib.isd_lm_head_workspace_bytes(ctypes.byref(a))
    a.vocab_stats = _FAKE * 5
    with_stats = lib.isd_lm_head_workspace_bytes(ctypes.byref(a))
    # per-record figures (records of 128 entries on CTA pairs): max (4 B),
    # sum (8 B), first index (4 B) per row
    assert with_stats - plain >= 2 * 594 * 512 * 16
    a.lora_rank, a.lora_a, a.lora_b, a.n_pending = 128, _FAKE, _FAKE, _FAKE
    with_lora = lib.isd_lm_head_workspace_bytes(ctypes.byref(a))
    assert with_lora - with_stats >= 512 * 128 * 2   # the bf16 U rows
    # csum f64, cmax f32, cidx i32 for each of M rows x ceil(V / 2048)
    assert lib.isd_vocab_stats_bytes(512, 151936) >= 512 * 75 * 16
    assert lib.isd_vocab_stats_bytes(0, 10) == 0
    assert lib.isd_lm_head_workspace_bytes(ctypes.byref(_lm_args(M=0))) == 0


def test_lm_head_launch_count(lib):
    # Below 64 rows there is never a split-K tail, so the count does not
    # depend on the device: the GEMM, the statistics merge, the LoRA
    # down-projection and its sum.
    a = _lm_args(M=32)
    assert lib.isd_lm_head_launches(ctypes.byref(a)) == 1
    a.vocab_stats = _FAKE * 5
    assert lib.isd_lm_head_launches(ctypes.byref(a)) == 2
    a.lora_rank, a.lora_a, a.lora_b, a.n_pending = 128, _FAKE, _FAKE, _FAKE
    assert lib.isd_lm_head_launches(ctypes.byref(a)) == 4
    assert lib.isd_lm_head_launches(ctypes.byref(_lm_args(M=0))) == 0


def _fake_pair():
    """Accept and commit arguments for the fused call, each consistent on
    its own (fake aligned pointers, workspaces large enough) and describing
    the same sequences; nothing here is ever launched."""
    ws = ctypes.c_void_p(0x8000000)
    a = _fake_accept_args(B=4, N=4, K=8, V=1024, dtype=isd.BF16, workspace=ws,
                          workspace_bytes=1 << 24)
    ptr = iter(range(0x4000000, 0x4000000 + 0x10000 * 16, 0x10000))
    f = {k: ctypes.c_void_p(next(ptr)) for k in (
        "k_new", "v_new", "k_cache", "v_cache", "page_table", "free_stack",
        "free_top", "status", "workspace")}
    c = isd.CommitArgs(B=4, K=8, Hkv=8, d=128, num_pages=64,
                       page_table_stride=8, dtype=isd.BF16,
                       seq_len=a.seq_len, n_commit=a.n_commit,
                       workspace_bytes=256, **f)
    return a, c


def test_accept_commit_host_validation(lib):
    """The fused call applies both calls' checks and refuses a commit that
    does not consume this accept step's decisions."""
    def call(a, c):
        return lib.isd_accept_commit(ctypes.byref(a), ctypes.byref(c), None)

    a, c = _fake_pair()
    c.n_commit = ctypes.c_void_p(0x7000000)        # another n_commit
    assert call(a, c) == isd.ERR_INVALID_ARG
    a, c = _fake_pair()
    c.seq_len = ctypes.c_void_p(0x7000000)         # another seq_len
    assert call(a, c) == isd.ERR_INVALID_ARG
    a, c = _fake_pair()
    c.B = 3
    assert call(a, c) == isd.ERR_INVALID_ARG
    a, c = _fake_pair()
    c.K = 16
    assert call(a, c) == isd.ERR_INVALID_ARG
    # Each half's own errors, with the codes of the separate calls.
    a, c = _fake_pair()
    a.logits_cur = None
    assert call(a, c) == lib.isd_accept_resample(ctypes.byref(a), None) == \
        isd.ERR_INVALID_ARG
    a, c = _fake_pair()
    a.workspace = None
    assert call(a, c) == isd.ERR_WORKSPACE
    a, c = _fake_pair()
    c.workspace = None
    assert call(a, c) == lib.isd_kv_commit(ctypes.byref(c), None) == \
        isd.ERR_WORKSPACE
    a, c = _fake_pair()
    c.d = 4                                          # 8-byte rows
    assert call(a, c) == isd.ERR_UNSUPPORTED
    # The commit's counter inside the accept's workspace.
    a, c = _fake_pair()
    c.workspace = ctypes.c_void_p(a.workspace + 256)
    assert call(a, c) == isd.ERR_INVALID_ARG
