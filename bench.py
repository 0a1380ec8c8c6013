"""Benchmark of one ISD step (attention + accept/resample + KV commit).

Default workload: the C=64 stationary batch (64 sequences, 32 query / 8 KV
heads, head dim 128, prefixes uniform in [1024, 8192] on a shuffled paged
cache, N=4 so K=8 query rows, vocabulary 151 936, draft noise tuned for mean
acceptance 0.9), run for consecutive steps with KV commit and rollback.
Inputs are seeded synthetic tensors; the logits of each step (the LM head's
output, not part of the timed path) are generated between steps, and L2 is
flushed before every timed step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl isd|reference]
                  [--workload c64_stationary|8b_b1|32b_b32|sweep|
                              c64_lm_head|c64_rlora|all]
                  [--eager]

Prints one JSON line (rank 0) per workload (the default: one).  ``value`` is
accepted (committed) tokens per second over all ranks: every step runs as
one replay of the captured CUDA graph of the library calls (the serving
path: isd_attn_strided, then isd_accept_commit, the accept step with the KV
commit running beside its draws), device-timed with CUDA events around it,
max over ranks.  ``--eager`` times the same calls launched one by one
instead.  The per-phase split in ``detail`` comes from further eager steps
with the accept and commit as separate calls (isd_accept_resample,
isd_kv_commit), events between them.  With N > 1
every rank runs its own replica (the path shards by sequence; no
collective on the data path).

``c64_lm_head`` and ``c64_rlora`` put the LM head in the timed step: each
step starts from the rows' final hidden states (D = 4096), isd_lm_head makes
the logits and their vocabulary statistics on the tensor cores (with the
R-ISD gated LoRA of rank 128 at MASK rows for ``c64_rlora``), and the accept
step takes those statistics; their roofline is the LM head's, against the
bf16 tensor peak.
"""

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("ISD accepted tokens/s at B=64,N=4; achieved HBM GB/s as fraction "
          "of B200 peak")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
SWEEP = [(B, N, p) for B in (1, 8, 32, 64) for N in (2, 4, 8)
         for p in (0.5, 0.9)]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="isd", choices=["isd", "reference"])
    ap.add_argument("--workload", default="c64_stationary",
                    choices=["c64_stationary", "8b_b1", "32b_b32", "sweep",
                             "c64_lm_head", "c64_rlora", "all"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=None,
                    help="override the workload's sequences per GPU (only "
                         "for profiling captures of a smaller case)")
    ap.add_argument("--vocab", type=int, default=None,
                    help="override the vocabulary size, keeping the draft "
                         "noise of the workload's own vocabulary (only for "
                         "profiling captures of a smaller case)")
    ap.add_argument("--proposal", default="sample", choices=["sample", "argmax"],
                    help="drafts drawn from q (default) or x = argmax q")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of graph replays")
    ap.add_argument("--phase-steps", type=int, default=5,
                    help="eager steps timed per phase for the split")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-steps", type=int, default=4)
    ap.add_argument("--cpu-sample-seqs", type=int, default=0,
                    help="oracle worker processes (0: one per host core, "
                         "at most one per sequence)")
    return ap.parse_args()


# DRAM traffic of the attention kernel per algorithmic byte, from one ncu
# capture of the C=64 workload at B = 16 (dram__bytes_read.sum +
# dram__bytes_write.sum over the launch's algorithmic bytes; see
# profiles/attn_tc_kernel_c64_b16_full.md).  Traffic tracks the algorithmic
# bytes, so a full launch's traffic is this ratio times its bytes.  Valid
# only for the kernel source the capture was taken on.
TRAFFIC_PER_ALGO_BYTE = (331.50 + 8.13) / 332.37
TRAFFIC_KERNEL_SHA256 = (
    "1997e7da6e61d1637e2e96214c47b461c6763b0094e2599cac508beac74df4fb")


def attention_traffic(bytes_per_launch):
    path = os.path.join(ROOT, "introspective_strided_decoding_b200", "csrc",
                        "attn_tc.cu")
    try:
        with open(path, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except OSError:
        return None
    if TRAFFIC_PER_ALGO_BYTE is None or sha != TRAFFIC_KERNEL_SHA256:
        return None
    return TRAFFIC_PER_ALGO_BYTE * bytes_per_launch


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s: the burst figure (the LM head is timed as one
    call inside the step)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def tpf_closed_form(p, N):
    """The pages' memory-bound tokens-per-forward formula (hada.io summary,
    "Speedup Factor Explorer"), for reporting beside the measured TPF."""
    num = 2.0 + sum(p ** k for k in range(1, N - 1))
    return num / (2.0 - p ** (N - 1))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clocks/throttle sampling during the timed region."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,"
         "clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.file = None

    def start(self):
        try:
            self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv",
                                                    delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.file, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.file.flush()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines()]
        os.unlink(self.file.name)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
            except ValueError:
                continue
            for name, val in zip(names, r[5:9]):
                if val.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------ distributed
def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local) if args.impl == "isd" else None
        torch.distributed.init_process_group(
            "nccl" if args.impl == "isd" else "gloo",
            timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def allreduce(x, op, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=op)
    return float(t.item())


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def rank_seed(seed, rank):
    """Each replica decodes its own seeded batch."""
    return seed + 1000 * rank


def job_figures(total_ms, tokens, e2e_ms, e2e_tokens, world, device):
    """Whole-job figures over the replicas: the slowest rank's device time,
    every rank's committed tokens (max and sum all-reductions; no-ops on
    one rank)."""
    mx = torch.distributed.ReduceOp.MAX if world > 1 else None
    sm = torch.distributed.ReduceOp.SUM if world > 1 else None
    total_ms_max = allreduce(total_ms, mx, world, device)
    tokens_all = allreduce(tokens, sm, world, device)
    e2e_ms_max = allreduce(e2e_ms, mx, world, device)
    e2e_tokens_all = allreduce(e2e_tokens, sm, world, device)
    return {"total_ms_max": total_ms_max, "tokens": tokens_all,
            "value": tokens_all / (total_ms_max / 1e3),
            "e2e_ms_max": e2e_ms_max, "e2e_tokens": e2e_tokens_all,
            "e2e_value": e2e_tokens_all / (e2e_ms_max / 1e3)}


# --------------------------------------------------------- oracle sample
def _oracle_one_sequence(job):
    """One worker of the CPU baseline: the fp64 oracle's full step
    (attention over every KV head, accept/resample, commit) for one
    sequence of the workload, ``skip + steps`` consecutive steps from the
    start state, the first ``skip`` untimed.  Returns (tokens, seconds)."""
    w, seed, b, steps, skip, proposal = job
    try:
        from threadpoolctl import threadpool_limits
        threadpool_limits(limits=1)
    except Exception:
        pass
    torch.set_num_threads(1)
    from introspective_strided_decoding_b200 import synth
    from oracle import attention as oattn
    from oracle import step as ostep
    # Sequence b of the workload: its own prefix length, pages and state.
    L_all = synth.prefix_lengths(w, seed)
    ws = w.with_(B=1, L_lo=int(L_all[b]), L_hi=int(L_all[b]))
    cache = synth.make_cache(ws, seed + 7919 * b, "cpu")
    st = synth.initial_state(ws, seed + 7919 * b, "cpu")
    kc = cache["k_cache"].float().numpy()
    vc = cache["v_cache"].float().numpy()
    pt = cache["page_table"].long().numpy()
    fs = cache["free_stack"].long().numpy()
    top = int(cache["free_top"].item())
    L = cache["seq_len"].long().numpy()
    pend = st["pending"].long().numpy()
    n = st["n_pending"].long().numpy()
    qrow = st["q_row"].long().numpy()
    prev = np.zeros((1, ws.K, ws.V), dtype=np.float32)
    tokens, secs = 0, 0.0
    for s in range(skip + steps):
        lc = synth.step_logits(ws, seed + b, torch.from_numpy(L),
                               torch.from_numpy(n), s, "cpu").float().numpy()
        q, k, v = (t.float().numpy() for t in
                   synth.make_stride(ws, seed + b, s, "cpu"))
        t0 = time.perf_counter()
        oattn.attn_strided(q.astype(np.float64), k.astype(np.float64),
                           v.astype(np.float64), kc, vc, pt, L,
                           1.0 / np.sqrt(ws.d))
        o = ostep.accept_resample(lc, prev, pend, n, qrow, L, seed, s, ws.N,
                                  proposal=proposal)
        kc, vc, pt, L2, top, _ = ostep.kv_commit(k, v, kc, vc, pt, L,
                                                 o["n_commit"], fs, top)
        if s >= skip:
            secs += time.perf_counter() - t0
            tokens += int(o["n_commit"].sum())
        L = L2
        pend, n, qrow, prev = (o["next_pending"], o["next_n"],
                               o["next_q_row"], lc)
    return tokens, secs


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(w, seed, steps, skip=1, proposal="sample", seqs=0):
    """Time the fp64 oracle on the host cores, on a bounded sample of the
    workload: one sequence per core (the first min(cores, B) sequences),
    ``steps`` timed steps each after ``skip`` untimed ones, one process per
    sequence in a spawn pool (the CUDA context of this process is not
    forked).  Throughput = tokens decided / the slowest worker's compute
    time (the workers run concurrently).  Returns (tokens/s, cores,
    description)."""
    import multiprocessing as mp
    cores = host_cores()
    nseq = min(cores, w.B, seqs if seqs > 0 else cores)
    jobs = [(w, seed, b, steps, skip, proposal) for b in range(nseq)]
    ctx = mp.get_context("spawn")
    with ctx.Pool(nseq) as pool:
        res = pool.map(_oracle_one_sequence, jobs)
    tokens = sum(r[0] for r in res)
    secs = max(r[1] for r in res)
    desc = (f"fp64 numpy oracle, {nseq} of the {w.B} sequences (one per "
            f"host core, spawn pool, 1 BLAS thread each), steps "
            f"{skip}..{skip + steps - 1} of each chain: attention over every "
            f"KV head, accept/resample, commit; tokens / slowest worker's "
            f"compute time")
    return tokens / secs, nseq, desc


# --------------------------------------------------------------- isd arm
def workload_list(args):
    from introspective_strided_decoding_b200 import synth
    named = {"c64_stationary": synth.C64, "8b_b1": synth.SHAPE_8B,
             "32b_b32": synth.SHAPE_32B}
    lm = {"c64_lm_head": synth.C64_LM, "c64_rlora": synth.C64_RLORA}
    if args.workload in named:
        return [named[args.workload]]
    if args.workload in lm:
        return [lm[args.workload]]
    sweep = [synth.sweep_workload(B, N, p) for B, N, p in SWEEP]
    if args.workload == "sweep":
        return sweep
    return list(named.values()) + sweep + list(lm.values())


MULTI_STEPS = 8


def multi_step_timing(dec, cache, prepare, run_step, flush, stream, dev):
    """Device time per step of one CUDA graph holding MULTI_STEPS steps
    (inputs from per-step slots, step index from the device counter), after
    an L2 flush; the steps' own inputs (weights, KV cache) exceed L2.  The
    inputs are those of the next MULTI_STEPS single-step replays, recorded
    and rewound; the multi-step replay must reproduce their lengths."""
    S = MULTI_STEPS
    snap = {k: v.clone() for k, v in cache.items()}
    snap_state = {k: v.clone() for k, v in dec.state.items()}
    snap_logits = [x.clone() for x in dec.logits]
    cur, idx = dec.cur, dec.step_idx
    rec = []
    for _ in range(S):
        prepare(dec.step_idx)
        rec.append(tuple(t.clone() for t in (dec.hidden, dec.q, dec.k_new,
                                             dec.v_new)))
        run_step()
    L_single = cache["seq_len"].clone()
    torch.cuda.synchronize(dev)

    def rewind():
        for k, v in snap.items():
            cache[k].copy_(v)
        for k, v in snap_state.items():
            dec.states[cur][k].copy_(v)
        for x, y in zip(dec.logits, snap_logits):
            x.copy_(y)
        dec.set_step(cur, idx)

    rewind()
    dec.capture_multi(S)
    times = []
    for rep in range(3):
        rewind()
        dec.step_dev.fill_(idx)
        for i, (h, q, k, v) in enumerate(rec):
            dec.slots["first"][i].copy_(h)
            dec.slots["q"][i].copy_(q)
            dec.slots["k_new"][i].copy_(k)
            dec.slots["v_new"][i].copy_(v)
        flush.fill_(rep & 0xFF)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        torch.cuda._sleep(100_000)
        e0.record(stream)
        dec.replay_multi()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        times.append(e0.elapsed_time(e1))
        if not torch.equal(cache["seq_len"], L_single):
            raise RuntimeError("multi-step graph diverged from single steps")
    rewind()
    ms = statistics.median(times)
    return {"steps_per_graph": S, "ms_per_step": ms / S,
            "replays": len(times), "l2": "flushed before each replay"}


def run_workload(w, args, world, rank, local, steps, warmup, with_cpu):
    from introspective_strided_decoding_b200 import build, isd, synth
    from introspective_strided_decoding_b200.driver import Decoder
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    phase_steps = max(1, args.phase_steps)
    n_e2e = max(1, args.e2e_steps)
    w = w.with_(steps=steps + warmup + phase_steps + 2 * n_e2e + 2)
    if args.batch is not None and args.batch != w.B:
        w = w.with_(B=args.batch, name=f"{w.name}_b{args.batch}")
    if args.vocab is not None and args.vocab != w.V:
        w = w.with_(V=args.vocab, target_accept=None,
                    sigma_q=synth.draft_sigma(w),
                    name=f"{w.name}_v{args.vocab}")
    seed = rank_seed(args.seed, rank)
    cache = synth.make_cache(w, seed, dev)
    st0 = synth.initial_state(w, seed, dev)
    with_lm = bool(w.meta.get("lm_head"))
    lm = None
    lm_flops = 0.0
    if with_lm:
        M, r = w.B * w.K, int(w.meta.get("lora_rank", 0))
        lm = dict(weight=synth.lm_weight(seed, w.V, w.D, dev)
                  .to(torch.bfloat16))
        lm_flops = 2.0 * M * w.D * w.V
        if r:
            a, b = synth.lora_factors(seed, r, w.D, w.V, dev)
            lm.update(lora_a=a.to(torch.bfloat16).contiguous(),
                      lora_b=b.to(torch.bfloat16).contiguous(),
                      lora_scale=float(w.meta["lora_scale"]))
            lm_flops += 2.0 * M * w.D * r + 2.0 * M * r * w.V
    dec = Decoder(w, cache, st0, dev, seed,
                  proposal=isd.PROPOSAL_ARGMAX if args.proposal == "argmax"
                  else isd.PROPOSAL_SAMPLE, lm=lm)
    stream = torch.cuda.current_stream(dev)
    use_graph = not args.eager
    if use_graph:
        dec.capture()
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    hbm_peak, peak_kind = peaks()
    es = 2 if w.dtype == "bf16" else 4
    kv_row = w.Hkv * w.d * es * 2           # K and V of one token
    qo_bytes = 2 * w.B * w.K * w.Hq * w.d * es + 2 * w.B * w.K * w.Hkv * w.d * es
    row_bytes = w.V * es

    def prepare(step):
        L = cache["seq_len"]
        n = dec.state["n_pending"]
        if with_lm:
            dec.hidden.copy_(synth.step_hidden(w, seed, L, n, step, dev))
        else:
            dec.logits_cur.copy_(synth.step_logits(w, seed, L, n, step, dev))
        q, k, v = synth.make_stride(w, seed, step, dev)
        dec.q.copy_(q)
        dec.k_new.copy_(k)
        dec.v_new.copy_(v)
        L_host = L.long().cpu()
        n_host = n.long().cpu()
        kv = int(L_host.sum()) * kv_row
        used_rows = int((n_host + w.N - 1).sum())
        flush.fill_(step & 0xFF)            # evict L2 (256 MB > 126 MB)
        return kv, used_rows

    def run_step(events=None):
        if use_graph:
            if events:
                events[0].record(stream)
            dec.replay()
            if events:
                events[-1].record(stream)
        else:
            dec.step(stream, events)

    for _ in range(warmup):
        prepare(dec.step_idx)
        run_step()
    torch.cuda.synchronize(dev)

    # ------------------------------------------------------- timed steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
          for _ in range(steps)]
    tok_dev = torch.zeros(1, dtype=torch.int64, device=dev)
    tested_dev = torch.zeros(1, dtype=torch.int64, device=dev)
    accepted_dev = torch.zeros(1, dtype=torch.int64, device=dev)
    kv_bytes, logit_rows = [], []
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    for s in range(steps):
        kv, rows = prepare(dec.step_idx)
        kv_bytes.append(kv)
        logit_rows.append(rows)
        n_in = dec.state["n_pending"].clone()
        # A short device-side sleep ahead of the first event: the host
        # queues the whole step while it runs, so the timed window holds
        # the step's kernels and not the host's launch latency.
        torch.cuda._sleep(100_000)
        run_step(ev[s])
        tok_dev += dec.n_commit.sum()
        # Drafts tested: the accepted ones plus the first rejected one.
        acc = (dec.n_commit - 1).clamp(min=0)
        accepted_dev += acc.sum()
        tested_dev += acc.sum() + (dec.n_commit < n_in).sum()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    t_step = [e[0].elapsed_time(e[-1]) for e in ev]
    total_ms = sum(t_step)
    tokens = int(tok_dev.item())
    tested, accepted = int(tested_dev.item()), int(accepted_dev.item())
    status = int(dec.status.item())
    if status != isd.OK:
        raise RuntimeError(f"device status {isd.status_string(status)}")
    step_bytes = [kv + qo_bytes + r * row_bytes for kv, r in
                  zip(kv_bytes, logit_rows)]
    step_gbs = sum(step_bytes) / (total_ms / 1e3) / 1e9
    if with_lm:
        step_gbs = None      # the logits are made in the step, not read

    # --------------------------------------- per-phase split (eager calls)
    nev = 5 if with_lm else 4
    pev = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)]
           for _ in range(phase_steps)]
    p_kv, p_rows = [], []
    for s in range(phase_steps):
        kv, rows = prepare(dec.step_idx)
        p_kv.append(kv)
        p_rows.append(rows)
        torch.cuda._sleep(100_000)
        dec.step(stream, pev[s])
    torch.cuda.synchronize(dev)
    t_attn = [e[0].elapsed_time(e[1]) for e in pev]
    t_lm = [e[1].elapsed_time(e[2]) for e in pev] if with_lm else []
    t_acc = [e[-3].elapsed_time(e[-2]) for e in pev]
    t_com = [e[-2].elapsed_time(e[-1]) for e in pev]
    attn_bytes = [kv + qo_bytes for kv in p_kv]
    achieved = sum(attn_bytes) / (sum(t_attn) / 1e3) / 1e9
    acc_bytes = sum(r * row_bytes for r in p_rows)
    aa_gbs = (sum(attn_bytes) + acc_bytes) / \
        ((sum(t_attn) + sum(t_acc)) / 1e3) / 1e9
    lm_ms = sum(t_lm) / phase_steps if with_lm else None
    if with_lm:
        aa_gbs = None

    # ---------------------------------------------------------------- e2e
    # Host-resident inputs (pinned), H2D copy + the step through the public
    # API + D2H of the step's result, all inside the timed region.  Each
    # step's inputs depend on the state the previous steps left, so they
    # are generated by running the steps once, kept on the host, and every
    # piece of state is rewound for the timed replay.
    snap = {k: v.clone() for k, v in cache.items()}
    snap_state = {k: v.clone() for k, v in dec.state.items()}
    snap_prev = dec.logits[1 - dec.cur].clone()
    snap_cur, snap_idx = dec.cur, dec.step_idx
    host_in = []
    for s in range(n_e2e):
        prepare(dec.step_idx)
        first = dec.hidden if with_lm else dec.logits_cur
        host_in.append(tuple(t.to("cpu").pin_memory() for t in
                             (first, dec.q, dec.k_new, dec.v_new)))
        run_step()
    torch.cuda.synchronize(dev)
    for k, v in snap.items():
        cache[k].copy_(v)
    for k, v in snap_state.items():
        dec.states[snap_cur][k].copy_(v)
    dec.logits[1 - snap_cur].copy_(snap_prev)
    dec.set_step(snap_cur, snap_idx)
    del snap, snap_prev
    res_host = torch.empty((w.B * (1 + w.N),), dtype=torch.int32).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host_in[0])
    d2h = res_host.numel() * 4
    flush.fill_(1)
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_tokens = 0
    e0.record(stream)
    for s in range(n_e2e):
        lg, q, k, v = host_in[s]
        (dec.hidden if with_lm else dec.logits_cur).copy_(lg,
                                                          non_blocking=True)
        dec.q.copy_(q, non_blocking=True)
        dec.k_new.copy_(k, non_blocking=True)
        dec.v_new.copy_(v, non_blocking=True)
        run_step()
        res_host[:w.B].copy_(dec.n_commit, non_blocking=True)
        res_host[w.B:].copy_(dec.state["pending"].reshape(-1),
                             non_blocking=True)
        stream.synchronize()
        e2e_tokens += int(res_host[:w.B].sum())
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    if int(dec.status.item()) != isd.OK:
        raise RuntimeError("device status after the e2e steps: "
                           f"{isd.status_string(int(dec.status.item()))}")
    multi = multi_step_timing(dec, cache, prepare, run_step, flush, stream,
                              dev) if with_lm and use_graph else None
    dec.release_graphs()
    job = job_figures(total_ms, tokens, e2e_ms, e2e_tokens, world, dev)
    total_ms_max, value = job["total_ms_max"], job["value"]
    e2e = {"value": job["e2e_value"], "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": n_e2e}
    alpha = accepted / max(tested, 1)
    tpf = tokens / (w.B * steps)
    calls = ("attention+LM head+accept/commit" if with_lm
             else "attention+accept/commit")
    inputs = "hidden-state" if with_lm else "logits"
    attn_roof = {
        "kernel": "attn_tc_kernel (+combine)", "bound": "hbm",
        "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
        "frac": achieved / hbm_peak, "peak_kind": peak_kind,
        "traffic": attention_traffic(sum(attn_bytes) / len(attn_bytes)),
        "bytes_per_launch": sum(attn_bytes) / len(attn_bytes)}
    if with_lm:
        tpk, tkind = tensor_peak()
        lm_tf = lm_flops / (lm_ms / 1e3) / 1e12
        roof = {"kernel": "lm_pair_kernel (+LoRA down, merge)",
                "bound": "tensor", "achieved": lm_tf, "peak": tpk,
                "unit": "TFLOP/s", "frac": lm_tf / tpk, "peak_kind": tkind,
                "traffic": None, "flops_per_launch": lm_flops}
    else:
        roof = attn_roof
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": total_ms_max / steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {
            "workload": w.name, "B": w.B, "N": w.N, "K": w.K, "Hq": w.Hq,
            "Hkv": w.Hkv, "d": w.d, "V": w.V, "page_size": 16,
            "prefix": [w.L_lo, w.L_hi], "pages": "shuffled",
            "target_accept": w.target_accept, "proposal": args.proposal,
            "l2": "flushed (256 MB write) before every timed step",
            "timing": ("CUDA events around one CUDA-graph replay of "
                       f"{calls} per step" if use_graph else
                       f"CUDA events around the eager {calls} calls per "
                       "step") +
                      f"; {inputs}/Q/K/V generation between steps untimed",
            "parallelism": f"replicas x{world}"},
        "roofline": roof,
        "e2e": e2e,
        "gpu_launches": dec.launches_per_step * steps,
        "clocks": clk,
        "detail": {
            "graph": use_graph,
            "attention_ms": sum(t_attn) / phase_steps,
            "accept_ms": sum(t_acc) / phase_steps,
            "commit_ms": sum(t_com) / phase_steps,
            "phase_split": f"eager calls, {phase_steps} further steps, "
                           "accept and commit as separate calls",
            "steps_per_s": steps / (total_ms / 1e3),
            "step_gbs": step_gbs,
            "step_frac": None if step_gbs is None else step_gbs / hbm_peak,
            "attn_accept_gbs": aa_gbs,
            "attn_accept_frac": None if aa_gbs is None else aa_gbs / hbm_peak,
            "tpf": tpf, "accept_rate": alpha,
            "tpf_closed_form_at_rate": tpf_closed_form(alpha, w.N),
            "tokens": tokens},
    }
    if with_lm:
        line["detail"].update(
            lm_head_ms=lm_ms, attention_roofline=attn_roof, multi_step=multi,
            lora_rank=int(w.meta.get("lora_rank", 0)), D=w.D)
        line["config"]["D"] = w.D
        line["config"]["lora_rank"] = int(w.meta.get("lora_rank", 0))
    if rank == 0 and with_cpu and not with_lm:
        v, cores, desc = oracle_sample(w, args.seed, args.cpu_sample_steps,
                                       proposal=args.proposal,
                                       seqs=args.cpu_sample_seqs)
        line["cpu_baseline"] = {"value": v, "unit": "tokens/s",
                                "cores": cores, "kind": "oracle",
                                "sample": desc}
    del dec, cache, flush
    torch.cuda.empty_cache()
    return line


def run_isd(args, world, rank, local):
    wl = workload_list(args)
    for i, w in enumerate(wl):
        many = len(wl) > 1
        steps = min(args.steps, 20) if many and w.name.startswith("sweep") \
            else args.steps
        warmup = max(3, min(args.warmup, 5)) if many else args.warmup
        line = run_workload(w, args, world, rank, local, steps, warmup,
                            with_cpu=(i == 0 and not args.no_cpu_baseline))
        if rank == 0:
            print(json.dumps(line), flush=True)


# --------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores, on the same config."""
    if rank != 0:
        return
    w = workload_list(args)[0]
    steps = max(1, args.steps)
    value, cores, desc = oracle_sample(w, args.seed, steps,
                                       skip=max(0, args.warmup),
                                       proposal=args.proposal,
                                       seqs=args.cpu_sample_seqs)
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "K": w.K,
                   "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "V": w.V,
                   "page_size": 16, "prefix": [w.L_lo, w.L_hi],
                   "pages": "shuffled", "target_accept": w.target_accept,
                   "proposal": args.proposal,
                   "l2": "host memory (no device cache)",
                   "parallelism": f"one process per host core, rank 0 of "
                                  f"{world}"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_isd(args, world, rank, local)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
