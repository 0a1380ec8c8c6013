"""Stationary-batch ISD decode loop on one GPU.

The pages' serving engine keeps batch membership fixed across steps
("stationary-batch decode loop", hada.io summary, "Serving (SGLang)").
``Decoder`` owns the per-step device buffers (logits ping-pong, decoding
state ping-pong, attention output, workspaces) and runs one step as the
three C-ABI calls on one stream:

    isd_attn_strided -> (caller's LM head fills logits) -> isd_accept_resample
    -> isd_kv_commit

With an LM head (``lm``: the output embedding and, for R-ISD, the gated
LoRA factors) the step starts from the rows' final hidden states instead
of logits:

    isd_attn_strided -> isd_lm_head (logits + vocabulary statistics)
    -> isd_accept_resample (fed by those statistics) -> isd_kv_commit

The argument structs are built once, so a step costs three or four ctypes
calls on the host.  All memory is allocated here, through torch, never by
the library.
"""

import ctypes
import math

import torch

from . import isd


class Decoder:
    def __init__(self, w, cache, state0, device, seed, num_ctas=0,
                 with_lse=False, record=False, proposal=None, lm=None):
        self.w = w
        self.cache = cache
        self.device = torch.device(device)
        self.seed = int(seed)
        B, K, N, V, Hq, d = w.B, w.K, w.N, w.V, w.Hq, w.d
        dt = w.torch_dtype
        dev = self.device
        self.q = torch.zeros((B, K, Hq, d), dtype=dt, device=dev)
        self.k_new = torch.zeros((B, K, w.Hkv, d), dtype=dt, device=dev)
        self.v_new = torch.zeros((B, K, w.Hkv, d), dtype=dt, device=dev)
        self.out = torch.empty((B, K, Hq, d), dtype=dt, device=dev)
        self.lse = torch.empty((B, K, Hq), dtype=torch.float32, device=dev) \
            if with_lse else None
        self.logits = [torch.zeros((B, K, V), dtype=dt, device=dev)
                       for _ in range(2)]
        self.states = [isd.new_state(B, N, dev), isd.new_state(B, N, dev)]
        for key in isd.STATE_KEYS:
            self.states[0][key].copy_(state0[key])
        self.n_commit = torch.zeros(B, dtype=torch.int32, device=dev)
        self.commit_tokens = torch.zeros((B, N), dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        # Optional per-step diagnostics (row statistics, draft ratios).
        self.row_stats = torch.full((B, K, 2), float("nan"),
                                    dtype=torch.float32, device=dev) \
            if record else None
        self.ratio = torch.full((B, N), float("nan"), dtype=torch.float32,
                                device=dev) if record else None
        self.cur = 0
        self.step_idx = 0
        scale = 1.0 / math.sqrt(d)
        self._attn = isd.attn_args(
            self.q, self.k_new, self.v_new, cache["k_cache"],
            cache["v_cache"], cache["page_table"], cache["seq_len"], self.out,
            self.lse, self.status, scale, None, num_ctas)
        self.ws_attn = torch.empty(max(isd.attn_workspace_bytes(self._attn),
                                       16), dtype=torch.uint8, device=dev)
        self._attn.workspace = ctypes.c_void_p(self.ws_attn.data_ptr())
        self._attn.workspace_bytes = self.ws_attn.numel()
        self.lm = lm
        self.vocab_stats = None
        self._lm = []
        if lm is not None:
            # Hidden states [B][K][D] in, logits and statistics out.
            M, D = B * K, lm["weight"].shape[1]
            self.hidden = torch.zeros((B, K, D), dtype=torch.bfloat16,
                                      device=dev)
            self.vocab_stats = isd.new_vocab_stats(M, V, dev)
            for c in range(2):
                a = isd.lm_head_args(
                    self.hidden.view(M, D), lm["weight"],
                    self.logits[c].view(M, V), self.vocab_stats,
                    lm.get("lora_a"), lm.get("lora_b"),
                    lm.get("lora_scale", 1.0),
                    self.states[c]["n_pending"] if lm.get("lora_a")
                    is not None else None, K, self.status)
                self._lm.append(a)
            self.ws_lm = torch.empty(max(isd.lm_head_workspace_bytes(
                self._lm[0]), 16), dtype=torch.uint8, device=dev)
            for a in self._lm:
                a.workspace = ctypes.c_void_p(self.ws_lm.data_ptr())
                a.workspace_bytes = self.ws_lm.numel()
        self._acc = []
        for c in range(2):
            a = isd.accept_args(self.logits[c], self.logits[1 - c],
                                cache["seq_len"], self.states[c],
                                self.states[1 - c], self.n_commit,
                                self.commit_tokens, self.seed, 0,
                                row_stats=self.row_stats, ratio=self.ratio,
                                status=self.status, proposal=proposal,
                                vocab_stats=self.vocab_stats)
            self._acc.append(a)
        self.ws_acc = torch.empty(isd.accept_workspace_bytes(self._acc[0]),
                                  dtype=torch.uint8, device=dev)
        for a in self._acc:
            a.workspace = ctypes.c_void_p(self.ws_acc.data_ptr())
            a.workspace_bytes = self.ws_acc.numel()
        self._com = isd.commit_args(
            self.k_new, self.v_new, cache["k_cache"], cache["v_cache"],
            cache["page_table"], cache["seq_len"], self.n_commit,
            cache["free_stack"], cache["free_top"], self.status)
        self.ws_com = torch.zeros(isd.commit_workspace_bytes(self._com),
                                  dtype=torch.uint8, device=dev)
        self._com.workspace = ctypes.c_void_p(self.ws_com.data_ptr())
        self._com.workspace_bytes = self.ws_com.numel()
        self._lib = isd.lib()

    # The buffers the caller fills before a step.
    @property
    def logits_cur(self):
        return self.logits[self.cur]

    @property
    def state(self):
        """Decoding state the next step reads; after a step, the state that
        step wrote (the ping-pong pair has already been swapped)."""
        return self.states[self.cur]

    def attention(self, stream=None):
        rc = self._lib.isd_attn_strided(ctypes.byref(self._attn),
                                        isd._stream(stream))
        if rc != isd.OK:
            raise isd.IsdError(rc, "isd_attn_strided")

    def lm_head(self, stream=None):
        rc = self._lib.isd_lm_head(ctypes.byref(self._lm[self.cur]),
                                   isd._stream(stream))
        if rc != isd.OK:
            raise isd.IsdError(rc, "isd_lm_head")

    def accept(self, stream=None):
        a = self._acc[self.cur]
        a.step = self.step_idx & 0xFFFFFFFF  # unused once step_dev is set
        rc = self._lib.isd_accept_resample(ctypes.byref(a),
                                           isd._stream(stream))
        if rc != isd.OK:
            raise isd.IsdError(rc, "isd_accept_resample")

    def commit(self, stream=None):
        rc = self._lib.isd_kv_commit(ctypes.byref(self._com),
                                     isd._stream(stream))
        if rc != isd.OK:
            raise isd.IsdError(rc, "isd_kv_commit")

    def accept_commit(self, stream=None):
        """The accept step and the commit in one call (isd_accept_commit):
        the commit runs beside the draws."""
        a = self._acc[self.cur]
        a.step = self.step_idx & 0xFFFFFFFF  # unused once step_dev is set
        rc = self._lib.isd_accept_commit(ctypes.byref(a),
                                         ctypes.byref(self._com),
                                         isd._stream(stream))
        if rc != isd.OK:
            raise isd.IsdError(rc, "isd_accept_commit")

    def advance(self):
        self.cur ^= 1
        self.step_idx += 1

    def step(self, stream=None, events=None):
        """Attention, (the LM head,) accept/resample and commit.  Without
        ``events`` the last two are one isd_accept_commit call; with
        ``events`` (CUDA events, for a per-phase split) they are separate
        calls and the events are recorded around the calls: before
        attention, before the LM head or accept, (with 5 events: before
        accept,) before the commit, after it."""
        s = stream if stream is not None else torch.cuda.current_stream()
        if events:
            events[0].record(s)
        self.attention(s)
        if events:
            events[1].record(s)
        if self.lm is not None:
            self.lm_head(s)
            if events and len(events) == 5:
                events[2].record(s)
        if events:
            self.accept(s)
            events[-2].record(s)
            self.commit(s)
            events[-1].record(s)
        else:
            self.accept_commit(s)
        if getattr(self, "step_dev", None) is not None:
            # Once graphs are captured the accept call reads the step index
            # from the device counter; eager steps advance it too.
            with torch.cuda.stream(s):
                self.step_dev.add_(1)
        self.advance()

    # ------------------------------------------------------ CUDA graphs
    def _step_counter(self):
        """The device step counter the captured graphs read (one tensor for
        every graph of this decoder, set to the current step index)."""
        if getattr(self, "step_dev", None) is None:
            self.step_dev = torch.full((1,), self.step_idx, dtype=torch.int32,
                                       device=self.device)
        else:
            self.step_dev.fill_(self.step_idx)

    def capture(self, stream=None):
        """Capture the step into two CUDA graphs, one per ping-pong parity
        (the pages' serving stack replays a captured decode step; "Serving
        (SGLang)" credits CUDA-graph capture with the largest gain).  The
        accept call then reads the step index from a device counter that
        the graph itself advances, so the same graph serves every step."""
        dev = self.device
        self._step_counter()
        for a in self._acc:
            a.step_dev = ctypes.c_void_p(self.step_dev.data_ptr())
        cur0 = self.cur
        s = stream if stream is not None else torch.cuda.Stream(dev)
        self.graphs = []
        for parity in (0, 1):
            self.cur = parity
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                self.attention()
                if self.lm is not None:
                    self.lm_head()
                self.accept_commit()
                self.step_dev.add_(1)
            self.graphs.append(g)
        self.cur = cur0

    def replay(self):
        """One step from the captured graph of the current parity."""
        self.graphs[self.cur].replay()
        self.advance()

    # ------------------------------------------- multi-step CUDA graph
    def capture_multi(self, steps, stream=None):
        """Capture ``steps`` consecutive steps (an even number, so the
        ping-pong parity comes back) into one CUDA graph: one replay runs
        them all, launching nothing from the host in between.  Step i reads
        its inputs from slot i of ``self.slots`` (hidden states with an LM
        head, else logits; the stride's Q and staged K/V) and the step
        index from the device counter.  With logits as inputs, slot i is
        the step's logits_cur and the stored q rows of step i come from slot
        i - 1; slot -1 (the previous replay's last step) is ``carry``, which
        the graph refreshes from slot S - 1 at its end."""
        if steps < 2 or steps % 2:
            raise ValueError("steps must be even and >= 2")
        S, w, dev = steps, self.w, self.device
        self._step_counter()
        first = self.hidden if self.lm is not None else self.logits_cur
        self.slots = dict(
            first=torch.zeros((S,) + tuple(first.shape), dtype=first.dtype,
                              device=dev),
            q=torch.zeros((S,) + tuple(self.q.shape), dtype=self.q.dtype,
                          device=dev),
            k_new=torch.zeros((S,) + tuple(self.k_new.shape),
                              dtype=self.k_new.dtype, device=dev),
            v_new=torch.zeros((S,) + tuple(self.v_new.shape),
                              dtype=self.v_new.dtype, device=dev))
        if self.lm is None:
            self.carry = self.logits[1 - self.cur].clone()

        def clone_args(a, **ptrs):
            c = type(a).from_buffer_copy(a)
            for k, t in ptrs.items():
                setattr(c, k, ctypes.c_void_p(t.data_ptr()))
            return c

        attn, lm, acc, com = [], [], [], []
        for i in range(S):
            par = (self.cur + i) % 2
            sq, sk, sv = (self.slots["q"][i], self.slots["k_new"][i],
                          self.slots["v_new"][i])
            attn.append(clone_args(self._attn, q=sq, k_new=sk, v_new=sv))
            com.append(clone_args(self._com, k_new=sk, v_new=sv))
            if self.lm is not None:
                lm.append(clone_args(self._lm[par],
                                     hidden=self.slots["first"][i]))
                a = clone_args(self._acc[par])
            else:
                prev = self.carry if i == 0 else self.slots["first"][i - 1]
                a = clone_args(self._acc[par],
                               logits_cur=self.slots["first"][i],
                               logits_prev=prev)
            a.step_dev = ctypes.c_void_p(self.step_dev.data_ptr())
            acc.append(a)
        self._multi_args = (attn, lm, acc, com)   # kept alive with the graph
        s = stream if stream is not None else torch.cuda.Stream(dev)
        g = torch.cuda.CUDAGraph()
        lib = self._lib
        with torch.cuda.graph(g, stream=s):
            cs = torch.cuda.current_stream()
            for i in range(S):
                for rc, what in (
                        (lib.isd_attn_strided(ctypes.byref(attn[i]),
                                              isd._stream(cs)),
                         "isd_attn_strided"),
                        (lib.isd_lm_head(ctypes.byref(lm[i]), isd._stream(cs))
                         if lm else isd.OK, "isd_lm_head"),
                        (lib.isd_accept_commit(ctypes.byref(acc[i]),
                                               ctypes.byref(com[i]),
                                               isd._stream(cs)),
                         "isd_accept_commit")):
                    if rc != isd.OK:
                        raise isd.IsdError(rc, what)
                self.step_dev.add_(1)
            if self.lm is None:
                self.carry.copy_(self.slots["first"][S - 1])
        self.multi_graph = g
        self.multi_steps = S

    def replay_multi(self):
        """The captured ``steps`` steps in one graph replay."""
        self.multi_graph.replay()
        self.step_idx += self.multi_steps

    def set_step(self, cur, step_idx):
        """Rewind (or move) the decoder to ping-pong parity ``cur`` and
        step index ``step_idx``, the device step counter included."""
        self.cur = int(cur)
        self.step_idx = int(step_idx)
        if getattr(self, "graphs", None):
            self.step_dev.fill_(self.step_idx)

    def release_graphs(self):
        """Drop the captured graphs (before the buffers they use)."""
        self.graphs = []
        self.multi_graph = None

    @property
    def launches_per_step(self):
        """This library's kernel launches per step: attention (bf16: the
        tcgen05 kernel and the split-segment combine; fp32: one kernel),
        the LM head's kernels when it is part of the step (as the library
        counts them), the accept kernels (statistics, decide, draw; with an
        LM head the statistics come from it) and the commit."""
        attn = 2 if self.w.dtype == "bf16" else 1
        if self.lm is None:
            return attn + 3 + 1
        return attn + isd.lm_head_launches(self._lm[0]) + 2 + 1
