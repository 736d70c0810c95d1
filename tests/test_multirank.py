"""The N > 1 path on CPU: two ranks over the gloo backend exercise the
benchmark's cross-rank plumbing (rendezvous, max-over-ranks timing, the
whole-job value of weak-scaling replicas), and a two-rank torchrun of the
reference arm prints exactly one line, from rank 0.  The attention path has no
data-path collective (heads are independent problems), so these are the only
cross-rank steps."""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_info()
    bench.init_dist(w, backend="gloo")
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * r, w)   # rank 1 is the slow one
        value = bench.job_value(2.0e12, ms, w)
        out.put((r, ms, value))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_is_the_max_and_value_counts_every_rank():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(out.get(timeout=10) for _ in range(world))
    for r, ms, value in got:
        assert ms == 15.0
        assert value == pytest.approx(2.0e12 * 2 / 15e-3 / 1e12)


def test_reference_arm_two_ranks_prints_one_line_from_rank_zero():
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), "bench.py", "--gpus", "2",
           "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, OMP_NUM_THREADS="2"))
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["scaling"] == "weak"
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"
