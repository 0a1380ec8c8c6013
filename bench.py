"""Benchmark of one ISD step (attention + accept/resample + KV commit).

Workload: the C=64 stationary batch (64 sequences, 32 query / 8 KV heads,
head dim 128, prefixes uniform in [1024, 8192] on a shuffled paged cache,
N=4 so K=8 query rows, vocabulary 151 936, draft noise tuned for mean
acceptance 0.9), run for consecutive steps with KV commit and rollback.
Inputs are seeded synthetic tensors; the logits of each step (the LM head's
output, not part of the timed path) are generated between steps, and L2 is
flushed before every timed step.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl isd|reference]

Prints one JSON line (rank 0).  ``value`` is accepted (committed) tokens
per second over all ranks, device-timed with CUDA events around the three
library calls of every step, max over ranks.  With N > 1 every rank runs
its own 64-sequence replica (the path shards by sequence; no collective on
the data path).
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="isd", choices=["isd", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--batch", type=int, default=64,
                    help="sequences per GPU (64 = the benchmark workload; "
                         "smaller only for profiling captures)")
    ap.add_argument("--proposal", default="sample", choices=["sample", "argmax"],
                    help="drafts drawn from q (default) or x = argmax q")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seqs", type=int, default=4)
    ap.add_argument("--cpu-sample-steps", type=int, default=8)
    return ap.parse_args()


# DRAM traffic of the attention kernel per algorithmic byte, from one ncu
# capture of this workload at B = 16 (dram__bytes_read.sum +
# dram__bytes_write.sum over the launch's algorithmic bytes; see
# profiles/attn_tc_kernel_c64_b16_full.md).  Traffic tracks the algorithmic
# bytes, so a full launch's traffic is this ratio times its bytes.  Valid only
# for the kernel source the capture was taken on.
TRAFFIC_PER_ALGO_BYTE = 340.05 / 332.02
TRAFFIC_KERNEL_SHA256 = (
    "71a076003bf7b68d3f9c2c4d7b2713ea6921847880a94e1e7c662821352cd6d0")


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
def oracle_sample(w, seed, n_seqs, steps=1, skip=0):
    """Time the fp64 oracle on a bounded sample of the workload: the first
    ``n_seqs`` sequences, full step (attention for all their KV heads,
    accept/resample, commit), ``skip + steps`` consecutive steps from the
    start state, the first ``skip`` untimed.  Returns (tokens decided,
    seconds, sample description) over the timed steps."""
    from oracle import attention as oattn
    from oracle import step as ostep
    from introspective_strided_decoding_b200 import synth
    try:
        from threadpoolctl import threadpool_limits
        limiter = threadpool_limits(limits=1)
    except Exception:
        limiter = None
    ws = w.with_(B=n_seqs)
    cache = synth.make_cache(ws, seed, "cpu")
    st = synth.initial_state(ws, seed, "cpu")
    kc = cache["k_cache"].float().numpy()
    vc = cache["v_cache"].float().numpy()
    pt = cache["page_table"].long().numpy()
    fs = cache["free_stack"].long().numpy()
    top = int(cache["free_top"].item())
    L = cache["seq_len"].long().numpy()
    pend = st["pending"].long().numpy()
    n = st["n_pending"].long().numpy()
    qrow = st["q_row"].long().numpy()
    prev = np.zeros((ws.B, ws.K, ws.V), dtype=np.float32)
    tokens, secs = 0, 0.0
    for s in range(skip + steps):
        lc = synth.step_logits(ws, seed, torch.from_numpy(L),
                               torch.from_numpy(n), s, "cpu").float().numpy()
        q, k, v = (t.float().numpy() for t in synth.make_stride(ws, seed, s,
                                                                "cpu"))
        t0 = time.perf_counter()
        oattn.attn_strided(q.astype(np.float64), k.astype(np.float64),
                           v.astype(np.float64), kc, vc, pt, L,
                           1.0 / np.sqrt(ws.d))
        o = ostep.accept_resample(lc, prev, pend, n, qrow, L, seed, s, ws.N)
        kc, vc, pt, L2, top, _ = ostep.kv_commit(k, v, kc, vc, pt, L,
                                                 o["n_commit"], fs, top)
        if s >= skip:
            secs += time.perf_counter() - t0
            tokens += int(o["n_commit"].sum())
        L = L2
        pend, n, qrow, prev = (o["next_pending"], o["next_n"],
                               o["next_q_row"], lc)
    if limiter is not None:
        limiter.restore_original_limits()
    desc = (f"fp64 numpy oracle, first {n_seqs} of {w.B} sequences, steps "
            f"{skip}..{skip + steps - 1} of the chain: attention (all KV "
            f"heads), accept/resample, commit; 1 BLAS thread")
    return tokens, secs, desc


# --------------------------------------------------------------- isd arm
def run_isd(args, world, rank, local):
    from introspective_strided_decoding_b200 import build, isd, synth
    from introspective_strided_decoding_b200.driver import Decoder
    build.build()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = synth.C64.with_(steps=args.steps + args.warmup + args.e2e_steps + 2)
    if args.batch != w.B:
        w = w.with_(B=args.batch, name=f"{w.name}_b{args.batch}")
    seed = rank_seed(args.seed, rank)
    cache = synth.make_cache(w, seed, dev)
    st0 = synth.initial_state(w, seed, dev)
    dec = Decoder(w, cache, st0, dev, seed,
                  proposal=isd.PROPOSAL_ARGMAX if args.proposal == "argmax"
                  else isd.PROPOSAL_SAMPLE)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    hbm_peak, peak_kind = peaks()
    es = 2  # bf16
    kv_row = w.Hkv * w.d * es * 2           # K and V of one token
    qo_bytes = 2 * w.B * w.K * w.Hq * w.d * es + 2 * w.B * w.K * w.Hkv * w.d * es
    row_bytes = w.V * es

    def prepare(step):
        L = cache["seq_len"]
        n = dec.state["n_pending"]
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

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
          for _ in range(args.steps)]
    tok_dev = torch.zeros(1, dtype=torch.int64, device=dev)
    tested = accepted = 0
    for s in range(args.warmup):
        prepare(dec.step_idx)
        dec.step(stream)
    torch.cuda.synchronize(dev)
    kv_bytes, logit_rows = [], []
    clocks = ClockSampler(local)
    barrier(world)
    torch.cuda.synchronize(dev)
    clocks.start()
    for s in range(args.steps):
        kv, rows = prepare(dec.step_idx)
        kv_bytes.append(kv)
        logit_rows.append(rows)
        n_in = dec.state["n_pending"].clone()
        # A short device-side sleep ahead of the first event: the host
        # queues the whole step while it runs, so the timed window holds
        # the step's kernels and not the host's launch latency.
        torch.cuda._sleep(100_000)
        dec.step(stream, ev[s])
        tok_dev += dec.n_commit.sum()
        # Drafts tested: the accepted ones plus the first rejected one.
        acc = (dec.n_commit - 1).clamp(min=0)
        tested += int(acc.sum() + (dec.n_commit < n_in).sum())
        accepted += int(acc.sum())
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    barrier(world)
    t_attn = [e[0].elapsed_time(e[1]) for e in ev]
    t_acc = [e[1].elapsed_time(e[2]) for e in ev]
    t_com = [e[2].elapsed_time(e[3]) for e in ev]
    t_step = [e[0].elapsed_time(e[3]) for e in ev]
    total_ms = sum(t_step)
    tokens = int(tok_dev.item())
    status = int(dec.status.item())
    if status != isd.OK:
        raise RuntimeError(f"device status {isd.status_string(status)}")

    attn_bytes = [kv + qo_bytes for kv in kv_bytes]
    achieved = sum(attn_bytes) / (sum(t_attn) / 1e3) / 1e9
    step_bytes = [kv + qo_bytes + r * row_bytes for kv, r in
                  zip(kv_bytes, logit_rows)]
    step_gbs = sum(step_bytes) / (total_ms / 1e3) / 1e9

    # ---------------------------------------------------------------- e2e
    # Host-resident inputs (pinned), H2D copy + the three calls + D2H of
    # the step's result, all inside the timed region.
    n_e2e = max(1, args.e2e_steps)
    # Each step's inputs depend on the state the previous steps left, so
    # generate them by running the steps once, keep host copies, then
    # rewind every piece of state for the timed replay.
    snap = {k: v.clone() for k, v in cache.items()}
    snap_state = {k: v.clone() for k, v in dec.state.items()}
    snap_prev = dec.logits[1 - dec.cur].clone()
    snap_cur, snap_idx = dec.cur, dec.step_idx
    host_in = []
    for s in range(n_e2e):
        prepare(dec.step_idx)
        host_in.append(tuple(t.to("cpu").pin_memory() for t in
                             (dec.logits_cur, dec.q, dec.k_new, dec.v_new)))
        dec.step(stream)
    torch.cuda.synchronize(dev)
    for k, v in snap.items():
        cache[k].copy_(v)
    dec.cur, dec.step_idx = snap_cur, snap_idx
    for k, v in snap_state.items():
        dec.state[k].copy_(v)
    dec.logits[1 - dec.cur].copy_(snap_prev)
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
        dec.logits_cur.copy_(lg, non_blocking=True)
        dec.q.copy_(q, non_blocking=True)
        dec.k_new.copy_(k, non_blocking=True)
        dec.v_new.copy_(v, non_blocking=True)
        dec.step(stream)
        res_host[:w.B].copy_(dec.n_commit, non_blocking=True)
        res_host[w.B:].copy_(dec.next_state["pending"].reshape(-1),
                             non_blocking=True)
        stream.synchronize()
        e2e_tokens += int(res_host[:w.B].sum())
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1)
    job = job_figures(total_ms, tokens, e2e_ms, e2e_tokens, world, dev)
    total_ms_max, value = job["total_ms_max"], job["value"]
    e2e = {"value": job["e2e_value"], "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "steps": n_e2e}

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": total_ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; no weights or datasets)",
        "config": {
            "workload": w.name, "B": w.B, "N": w.N, "K": w.K, "Hq": w.Hq,
            "Hkv": w.Hkv, "d": w.d, "V": w.V, "page_size": 16,
            "prefix": [w.L_lo, w.L_hi], "pages": "shuffled",
            "target_accept": w.target_accept, "proposal": args.proposal,
            "l2": "flushed (256 MB write) before every timed step",
            "timing": "CUDA events around attention+accept+commit per step; "
                      "logits/Q/K/V generation between steps untimed",
            "parallelism": f"replicas x{world}"},
        "roofline": {
            "kernel": "attn_tc_kernel (+combine)", "bound": "hbm",
            "achieved": achieved, "peak": hbm_peak, "unit": "GB/s",
            "frac": achieved / hbm_peak, "peak_kind": peak_kind,
            "traffic": attention_traffic(sum(attn_bytes) / len(attn_bytes)),
            "bytes_per_launch": sum(attn_bytes) / len(attn_bytes)},
        "e2e": e2e,
        "gpu_launches": Decoder.LAUNCHES_PER_STEP * args.steps,
        "clocks": clk,
        "detail": {
            "attention_ms": sum(t_attn) / args.steps,
            "accept_ms": sum(t_acc) / args.steps,
            "commit_ms": sum(t_com) / args.steps,
            "steps_per_s": args.steps / (total_ms / 1e3),
            "step_gbs": step_gbs, "step_frac": step_gbs / hbm_peak,
            "tpf": tokens / (w.B * args.steps),
            "accept_rate": accepted / max(tested, 1),
            "tokens": tokens},
    }
    if rank == 0 and not args.no_cpu_baseline:
        tok, secs, desc = oracle_sample(w, args.seed, args.cpu_sample_seqs,
                                        steps=args.cpu_sample_steps, skip=2)
        line["cpu_baseline"] = {"value": tok / secs, "unit": "tokens/s",
                                "cores": 1, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)


# --------------------------------------------------------- reference arm
def run_reference(args, world, rank):
    """The oracle, as it stands, on the host cores, on the same config."""
    if rank != 0:
        return
    from introspective_strided_decoding_b200 import synth
    w = synth.C64
    tokens, secs, desc = oracle_sample(w, args.seed, args.cpu_sample_seqs,
                                       steps=args.steps, skip=args.warmup)
    value = tokens / secs
    line = {
        "impl": "reference", "metric": METRIC, "value": value,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic (seeded; no weights or datasets)",
        "config": {"workload": w.name, "B": w.B, "N": w.N, "K": w.K,
                   "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "V": w.V,
                   "prefix": [w.L_lo, w.L_hi], "pages": "shuffled",
                   "target_accept": w.target_accept},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1,
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
