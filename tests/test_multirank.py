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
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["scaling"] == "strong"  # heads sharded
    assert d["value"] > 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_head_range_partitions_the_heads():
    import bench
    for H in range(1, 49):
        for world in range(1, min(H, 8) + 1):
            got = [bench.head_range(H, world, r) for r in range(world)]
            assert got[0][0] == 0 and got[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(got, got[1:]))
            sizes = [hi - lo for lo, hi in got]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    with pytest.raises(ValueError):
        bench.head_range(2, 3, 0)


def _oracle_heads(w, lo, hi):
    """The oracle's whole path on heads [lo, hi) of workload w: block scores,
    top-p selection, masked attention and the correction O + alpha_h R."""
    import dataclasses
    import numpy as np
    from block_sparse_attention_logits_b200.synthetic import make_qkv, random_bf16
    from oracle import attention as oatt, correction as ocor, scoring as osco, topp as otop
    ws = dataclasses.replace(w, H=hi - lo)
    t = make_qkv(w.B, hi - lo, w.grid, w.D, w.fp, h0=lo)
    qn, kn, vn = (t[n].float().numpy() for n in "qkv")
    _, _, P = osco.score_blocks(qn, kn, w.blk)
    _, idx, cnt = otop.select_topp_mask(P, np.full(hi - lo, w.p[0], np.float32))
    O, LSE = oatt.masked_attention(qn, kn, vn, idx, cnt, w.blk)
    R = random_bf16((w.B, w.H, w.L, w.D), 5).float().numpy()[:, lo:hi]
    O = ocor.apply_correction(O, R, np.asarray(w.alpha()[lo:hi]))
    assert ws.H == hi - lo
    return O, LSE, idx, cnt


def _shard_worker(rank, world, port, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import dataclasses
    import bench
    from block_sparse_attention_logits_b200 import configs
    w = dataclasses.replace(configs.TINY, H=5)
    bench.init_dist(world, backend="gloo")
    try:
        lo, hi = bench.head_range(w.H, world, rank)
        shard = _oracle_heads(w, lo, hi)
        gathered = [None] * world
        dist.all_gather_object(gathered, (lo, hi, shard))
        if rank == 0:
            out.put(gathered)
    finally:
        dist.destroy_process_group()


def test_head_shards_concatenate_to_the_one_rank_result():
    """Two gloo ranks each run the oracle's path on their head shard (rank r
    takes heads [r*H/N, (r+1)*H/N) of a 5-head workload, inputs drawn for
    exactly those heads); the gathered shards equal the one-rank result bit
    for bit, so the partitioning needs no data exchange."""
    import dataclasses
    import numpy as np
    from block_sparse_attention_logits_b200 import configs
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    procs = [ctx.Process(target=_shard_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    gathered = out.get(timeout=300)
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    w = dataclasses.replace(configs.TINY, H=5)
    full = _oracle_heads(w, 0, w.H)
    assert [g[:2] for g in gathered] == [(0, 3), (3, 5)]
    for k in range(4):
        cat = np.concatenate([g[2][k] for g in gathered], axis=1)
        assert np.array_equal(cat, full[k], equal_nan=True)
