"""The N > 1 path of bench.py on CPU: two gloo ranks.

A multi-GPU run is N independent replicas (one seeded batch per rank, no
collective on the data path); the ranks meet only to reduce the whole-job
figures (slowest rank's time, all ranks' tokens).  The reference arm under
two ranks prints one line from rank 0 and exits 0 everywhere.
"""

import datetime
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.abspath(os.path.join(os.path.dirname(__file__), ".."))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group(
        "gloo", rank=rank, world_size=world,
        timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # Rank r: 10 + r ms, 100 (r + 1) tokens; e2e 20 + 2r ms, 50 tokens.
        job = bench.job_figures(10.0 + rank, 100 * (rank + 1), 20.0 + 2 * rank,
                                50, world, "cpu")
        bench.barrier(world)
        q.put((rank, job, bench.rank_seed(7, rank)))
    finally:
        torch.distributed.destroy_process_group()


def test_two_rank_job_figures():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(2):
        rank, job, seed = q.get(timeout=120)
        got[rank] = (job, seed)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in (0, 1):
        job, _ = got[rank]
        assert job["total_ms_max"] == 11.0          # slowest rank
        assert job["tokens"] == 300                 # every rank's tokens
        assert job["value"] == pytest.approx(300 / 11e-3)
        assert job["e2e_ms_max"] == 22.0
        assert job["e2e_value"] == pytest.approx(100 / 22e-3)
    assert got[0][1] != got[1][1]                   # distinct replica data


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           "--nproc-per-node", "2", "--master-addr", "127.0.0.1",
           "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1",
           "--warmup", "0", "--cpu-sample-seqs", "2"]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600,
                       cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
