#!/usr/bin/env python
"""Benchmark of the top-p block-sparse attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME]

One step = one pass of the whole hot path over one batch of the Wan2.1-14B
720P workload (B=1, H=40, D=128, 21x45x80 latent tokens, blk 128, Hilbert
order, top-p tuned to ~90% block sparsity) with inputs resident in HBM:
  gather Q, K, V into Hilbert order -> block means + block softmax -> top-p
  selection -> block-sparse attention with the fused O + alpha*R epilogue ->
  scatter O back to grid order.
value = kept-block TFLOP per step summed over ranks / device-timed step time
(max over ranks).  Under torchrun the workload's heads are split over the
ranks (rank r takes heads [r*H/N, (r+1)*H/N); heads are independent problems,
so there is no collective on the data path): strong scaling.  --shard
replicas runs one full copy of the workload per rank instead (weak scaling).

--impl reference times the CPU oracle (the plain float64 statement of the
same computation) on a bounded sample of the same workload, on the host
cores; under torchrun only rank 0 runs it.
Prints one JSON line on rank 0.
"""

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_sparse_attention_logits_b200 import configs  # noqa: E402
from block_sparse_attention_logits_b200.synthetic import make_qkv, random_bf16  # noqa: E402

METRIC = "block-sparse attn ms/call & TFLOP/s on kept blocks vs bf16 TC peak at 90% sparsity"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# launches of this library per step: pooling (with the Q/K gather into curve
# order), block softmax, selection, attention (O in grid order); the
# reordered-copies form adds the V gather
LAUNCHES_PER_STEP = 4
E2E_MAX_CHUNKS = 8     # head chunks of the pipelined end-to-end step


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan2.1-14b-720p", choices=sorted(configs.ALL))
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="oracle sample budget")
    ap.add_argument("--top-p", type=float, default=0.0,
                    help="top-p threshold for every head (default: the workload's first value)")
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first N heads of the workload (small profiling captures)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-refresh", action="store_true",
                    help="skip the dense-refresh, mask-reuse, elementwise and sweep timings")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--gather", action="store_true",
                    help="Hilbert workloads: the attention gathers its tiles from the grid-order tensors "
                         "(no reordered copies; 4-row TMA gathers, slower) instead of reading reordered copies")
    ap.add_argument("--shard", choices=["heads", "replicas"], default="heads",
                    help="N > 1: split the workload's heads over the ranks (strong scaling, the default) or run "
                         "one full replica per rank (weak scaling)")
    return ap.parse_args()


# ---------------------------------------------------------------- plumbing

def dist_info():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend="nccl"):
    """One process group per job (rendezvous from MASTER_ADDR/PORT); a short
    timeout so that ranks waiting on a dead peer end with an error."""
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300))


def max_over_ranks(ms, world, dev=None):
    """The job's time is its slowest rank's."""
    if world <= 1:
        return float(ms)
    t = torch.tensor([float(ms)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_value(flops_per_rank, ms_per_step, world):
    """Whole-job throughput in TFLOP/s: every rank runs the workload (weak scaling)."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def sum_over_ranks(x, world, dev=None):
    """Work done by the whole job (each rank's own count, summed)."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def head_range(H, world, rank):
    """Heads [lo, hi) of `rank` when the H heads of one workload are split over
    `world` ranks as evenly as possible (the first H % world ranks take one
    more).  Heads are independent problems, so no rank needs another's data."""
    if H < world:
        raise ValueError(f"cannot split {H} heads over {world} ranks")
    base, extra = divmod(H, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def attention_kernel(blk):
    """Source file and kernel name of the attention kernel a block size runs."""
    if blk == 128:
        return "attention_tile.cu", "sparse_attn_tile_kernel<128>"
    return "attention.cu", "sparse_attn_kernel<128,64>"


def source_hash(fname):
    p = os.path.join(ROOT, "block_sparse_attention_logits_b200", "csrc", fname)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def profiled_traffic(workload, blk):
    """DRAM bytes per attention launch from the committed ncu summary, only if
    it was taken on the current source of the kernel that runs."""
    p = os.path.join(ROOT, "profiles", "attention_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(workload)
    fname, _ = attention_kernel(blk)
    if not d or d.get("kernel_source") != fname or d.get("kernel_source_sha256_16") != source_hash(fname):
        return None
    return d.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.path = None
        try:
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            self.sel = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.sel = str(device_index)

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.sel, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.25)
        self.proc.terminate()
        self.proc.wait()
        rows = [r.split(", ") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


def kept_flops(mask, L, blk, D):
    """4*D*sum over kept (i, j) of rows_i * cols_j, real tokens only."""
    nb = mask.shape[-1]
    sizes = torch.full((nb,), float(blk), dtype=torch.float64, device=mask.device)
    sizes[-1] = L - (nb - 1) * blk
    per_row = (mask.double() * sizes).sum(-1)  # kept key tokens per query block
    return float(4.0 * D * (per_row * sizes).sum().item())


# ---------------------------------------------------------- oracle sample

def oracle_sample(w, p, seconds, max_blocks=None):
    """Time the oracle on head 0 of the workload: Hilbert order, block scores,
    top-p selection, then masked attention of as many query blocks as fit in
    `seconds` (at least 4).  Returns (kept_flops, seconds, n_blocks, detail)."""
    from oracle import attention as oatt
    from oracle import hilbert as ohil
    from oracle import scoring as osco
    from oracle import topp as otop

    t = make_qkv(1, 1, w.grid, w.D, w.fp)
    q, k, v = (t[n].float().numpy() for n in ("q", "k", "v"))
    t0 = time.perf_counter()
    if w.hilbert:
        perm, _ = ohil.hilbert_perm(*w.grid)
        q, k, v = (ohil.permute_rows(x, perm) for x in (q, k, v))
    _, _, P = osco.score_blocks(q, k, w.blk)
    _, idx, cnt = otop.select_topp_mask_fast(P, np.array([p], np.float32))
    t_score = time.perf_counter() - t0
    rng = np.random.default_rng(0)
    order = rng.permutation(w.NB)
    sizes = np.full(w.NB, w.blk)
    sizes[-1] = w.L - (w.NB - 1) * w.blk
    flops, done, t_att = 0.0, 0, 0.0
    for i in order:
        if (t_att >= seconds and done >= 4) or (max_blocks and done >= max_blocks):
            break
        t1 = time.perf_counter()
        kb = idx[0, 0, i, :cnt[0, 0, i]]
        oatt.masked_attention_block(q, k, v, kb, w.blk, 0, 0, int(i))
        t_att += time.perf_counter() - t1
        flops += 4.0 * w.D * sizes[i] * sizes[kb].sum()
        done += 1
    # charge the scoring of the head in proportion to the blocks sampled
    total = t_att + t_score * done / w.NB
    return flops, total, done, f"head 0, {done} of {w.NB} query blocks (float64 numpy), scoring charged pro rata"


# ------------------------------------------------------------------- ours

def interval_timings(idx, cnt, L, blk, D, barrier, q=0.95, qkv=None):
    """The interval (skip-list) form of a step's kept lists: per-row runs and
    their histogram, the width for merge percentage q, encode and decode
    (decode writes kept lists only); with qkv (the attention's inputs, blk
    128) also the attention walking the merged pairs against the attention
    over the lists they decode to; times in ms per call, sizes in bytes."""
    from block_sparse_attention_logits_b200 import api
    B, H, nb = cnt.shape
    dev = cnt.device
    st = torch.zeros(1, dtype=torch.int32, device=dev)
    n_runs = torch.empty_like(cnt)
    hist = torch.zeros(api.max_intervals(nb) + 1, dtype=torch.int32, device=dev)
    api.interval_runs(idx, cnt, L, blk, D, n_runs=n_runs, hist=hist, status=st)
    Wq = api.interval_width_for_merge(hist, q)
    Wmax = api.interval_width_for_merge(hist, 1.0)
    iv = torch.empty((B, H, nb, Wq, 2), dtype=torch.int32, device=dev)
    n_int, nr2 = torch.empty_like(cnt), torch.empty_like(cnt)
    kidx, kcnt = torch.empty_like(idx), torch.empty_like(cnt)
    scratch = torch.zeros_like(hist)
    calls = [("runs", lambda: api.interval_runs(idx, cnt, L, blk, D, n_runs=nr2, hist=scratch, status=st)),
             ("encode", lambda: api.kept_to_intervals(idx, cnt, Wq, L, blk, D, iv, n_int, nr2, st)),
             ("decode", lambda: api.intervals_to_kept(iv, n_int, L, blk, D, kept_idx=kidx, kept_cnt=kcnt,
                                                      want_mask=False, status=st))]
    if qkv is not None and blk == 128:
        qa, ka, va = qkv
        oa, la = torch.empty_like(qa), torch.empty(qa.shape[:3], dtype=torch.float32, device=dev)
        calls += [("attention_walking_intervals",
                   lambda: api.sparse_attn_fwd_intervals(qa, ka, va, blk, iv, n_int, o=oa, lse=la, status=st)),
                  ("attention_on_decoded_lists",
                   lambda: api.sparse_attn_fwd(qa, ka, va, blk, kidx, kcnt, o=oa, lse=la, status=st))]
    ms = {}
    for name, fn in calls:
        fn()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(10):
            fn()
        a1.record()
        barrier()
        ms[name] = round(a0.elapsed_time(a1) / 10, 4)
    rows = B * H * nb
    before = cnt.double().sum().item()
    extra = {}
    if "attention_walking_intervals" in ms:
        extra = {"attention_walking_intervals_ms": ms["attention_walking_intervals"],
                 "attention_on_decoded_lists_ms": ms["attention_on_decoded_lists"]}
    return {"runs_ms": ms["runs"], "encode_ms": ms["encode"], "decode_ms": ms["decode"], **extra,
            "merge_q": q, "width_at_q": Wq, "width_max": Wmax, "max_possible": api.max_intervals(nb),
            "runs_per_row_mean": round(n_runs.double().mean().item(), 2),
            "rows_merged_frac": round((n_runs > Wq).double().mean().item(), 4),
            "blocks_added_by_merge_frac": round((kcnt.double().sum().item() - before) / max(before, 1.0), 5),
            "list_bytes": rows * nb * 4 + rows * 4, "interval_bytes_at_q": rows * Wq * 8 + rows * 4,
            "interval_bytes_max": rows * Wmax * 8 + rows * 4, "status": int(st.item())}


def tail_timings(q, k, v, mask, idx, cnt, blk, barrier):
    """The coarse tail of the omitted blocks on a step's inputs: statistics
    (block moments and pooled covariance), the tail, the refinement at a
    refresh (with the exact tail over the complement lists) and the
    reconstruction; ms per call."""
    from block_sparse_attention_logits_b200 import api
    L = q.shape[2]
    st = torch.zeros(1, dtype=torch.int32, device=q.device)
    o_S, l_S = api.sparse_attn_fwd(q, k, v, blk, idx, cnt, status=st)
    ci, cc = api.complement_lists(mask, L, blk)
    o_T, l_T = api.sparse_attn_fwd(q, k, v, blk, ci, cc, status=st)
    _, _, _, _, ws = api.tail_stats(k, v, blk, status=st)
    lbar, obar = api.coarse_tail(q, mask, blk, ws, status=st)
    d_l, d_o = api.tail_refinement(l_T, o_T, lbar, obar)
    calls = (("stats", lambda: api.tail_stats(k, v, blk, ws=ws, status=st)),
             ("coarse_tail", lambda: api.coarse_tail(q, mask, blk, ws, status=st)),
             ("refinement", lambda: api.tail_refinement(l_T, o_T, lbar, obar)),
             ("reconstruct", lambda: api.tail_reconstruct(l_S, o_S, lbar, obar, d_l, d_o)))
    ms = {}
    for name, fn in calls:
        fn()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(5):
            fn()
        a1.record()
        barrier()
        ms[name + "_ms"] = round(a0.elapsed_time(a1) / 5, 4)
    ms["status"] = int(st.item())
    return ms


def fp8_timings(q, k, v, idx, cnt, blk, flops, barrier, hbm_gbs):
    """FP8 Q.K^T attention on a step's inputs: E4M3 quantization of Q and K
    per token block (HBM-bound: 2 bytes read and 1 written per element), then
    the block-sparse attention over the same kept lists with S = Q.K^T from
    the codes; ms per call and kept TFLOP/s."""
    from block_sparse_attention_logits_b200 import api
    st = torch.zeros(1, dtype=torch.int32, device=q.device)
    q8, qs = api.quantize_fp8(q, blk)
    k8, ks = api.quantize_fp8(k, blk)
    o, lse = api.sparse_attn_fwd_fp8(q8, qs, k8, ks, v, blk, idx, cnt, status=st)
    calls = (("quantize_qk", lambda: (api.quantize_fp8(q, blk, q8, qs), api.quantize_fp8(k, blk, k8, ks))),
             ("attention", lambda: api.sparse_attn_fwd_fp8(q8, qs, k8, ks, v, blk, idx, cnt, o=o, lse=lse,
                                                           status=st)))
    ms = {}
    for name, fn in calls:
        fn()
        barrier()
        a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a0.record()
        for _ in range(5):
            fn()
        a1.record()
        barrier()
        ms[name] = a0.elapsed_time(a1) / 5
    qk_bytes = 2 * q.numel() * 3
    return {"quantize_qk_ms": round(ms["quantize_qk"], 4),
            "quantize_GB/s": round(qk_bytes / (ms["quantize_qk"] * 1e-3) / 1e9, 1),
            "quantize_frac_of_hbm": round(qk_bytes / (ms["quantize_qk"] * 1e-3) / 1e9 / hbm_gbs, 3),
            "attention_ms": round(ms["attention"], 4),
            "kept_tflops": round(flops / (ms["attention"] * 1e-3) / 1e12, 2),
            "scaling": "E4M3 per (batch, head, 128-token block), scale = amax / 448; P and V bf16",
            "status": int(st.item())}


def run_ours(args, w, world, rank, local):
    from block_sparse_attention_logits_b200 import api, _lib
    from block_sparse_attention_logits_b200 import build as bsa_build
    from block_sparse_attention_logits_b200.step import alloc_buffers, run_step

    init_dist(world)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    bsa_build.build()
    _lib.load()

    # this rank's heads: all of them (N = 1, or replicas), or its head shard
    h_lo, h_hi = head_range(w.H, world, rank) if args.shard == "heads" else (0, w.H)
    B, H, L, D, blk = w.B, h_hi - h_lo, w.L, w.D, w.blk
    p = float(w.p[0])
    pin = torch.cuda.is_available()
    host = {n: torch.empty((B, H, L, D), dtype=torch.bfloat16, pin_memory=pin) for n in ("q", "k", "v")}
    make_qkv(B, H, w.grid, D, w.fp, out=host, h0=h_lo)
    q, k, v = (host[n].to(dev) for n in ("q", "k", "v"))
    # cached refinement: in grid order when the attention gathers its tiles,
    # in curve order when it reads reordered copies
    R_h = random_bf16((B, H, L, D), 99 + h_lo, scale=0.05).to(dev)
    alpha = torch.tensor(w.alpha()[h_lo:h_hi], dtype=torch.float32, device=dev)
    strong = args.shard == "heads" and world > 1

    perm = api.reorder_tokens(*w.grid, device=dev)[0] if w.hilbert else None
    gather = w.hilbert and args.gather
    nb = api.n_blocks(L, blk)
    bufs = alloc_buffers(B, H, L, D, blk, dev, copies=not gather)
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    side = torch.cuda.Stream(dev)  # the V gather beside block softmax and selection

    def path(b, qi, ki, vi, Ri, ai, events=None, side_stream=None):
        """One pass of the hot path on buffers `b` (the full set or one head
        chunk): scoring in Hilbert order, selection, sparse attention with the
        fused correction, output in grid order."""
        return run_step(b, qi, ki, vi, blk, p, perm, Ri, ai, status, events, gather=gather, side=side_stream)

    def step(qi, ki, vi, events=None):
        return path(bufs, qi, ki, vi, R_h, alpha, events, side)

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    # warm-up
    for _ in range(max(args.warmup, 3)):
        step(q, k, v)
    torch.cuda.synchronize()
    if status.item() != 0:
        raise RuntimeError(f"attention kernel reported status {status.item()}")
    flops = kept_flops(bufs["mask"], L, blk, D)
    sparsity = 1.0 - bufs["cnt"].double().sum().item() / (B * H * nb * nb)

    # timed region: K steps, events per stage
    K = args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(K)]
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    start.record()
    for i in range(K):
        step(q, k, v, evs[i])
    stop.record()
    barrier()
    clk = clocks.stop()
    elapsed_ms = start.elapsed_time(stop)
    attn_ms = [evs[i][1].elapsed_time(evs[i][2]) for i in range(K)]
    sel_ms = [evs[i][0].elapsed_time(evs[i][1]) for i in range(K)]
    elapsed_ms = max_over_ranks(elapsed_ms, world, dev)
    ms_step = elapsed_ms / K
    job_flops = sum_over_ranks(flops, world, dev)  # every rank's kept work (replicas: world x one workload)
    value = job_flops / (ms_step * 1e-3) / 1e12

    # e2e: host buffers in, result out, through the same API calls.  Heads are
    # independent, so the step runs over head chunks on three streams: the
    # copy-in of chunk c+1 and the copy-out of chunk c-1 overlap the compute of
    # chunk c (PCIe carries 3.1 GB per step; the compute takes ~14 ms).
    e2e = None
    if not args.no_e2e:
        o_host = torch.empty((B, H, L, D), dtype=torch.bfloat16, pin_memory=pin)
        lse_host = torch.empty((B, H, L), dtype=torch.float32, pin_memory=pin)
        qd, kd, vd = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        n_chunks = max(d for d in range(1, E2E_MAX_CHUNKS + 1) if H % d == 0) if B == 1 else 1
        if (L * (H // n_chunks)) % 4:  # keep every float32 [L] slice 16-byte aligned
            n_chunks = 1
        hc = H // n_chunks
        s_in, s_cmp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(n_chunks)]
        ev_cmp = [torch.cuda.Event() for _ in range(n_chunks)]
        chunk_bufs = []
        for c in range(n_chunks):
            hs = slice(c * hc, (c + 1) * hc)
            # token-row buffers are head slices (16-byte aligned offsets); the
            # per-block score and list buffers get their own allocations (an
            # [NB, NB] slice of an odd NB is not 16-byte aligned)
            chunk_bufs.append({n: (None if t is None else t[:, hs] if n in ("qh", "kh", "vh", "oh", "o", "lse") else
                                   torch.empty_like(t[:, hs])) for n, t in bufs.items()})

        def chunk_step(c, qi, ki, vi):
            hs = slice(c * hc, (c + 1) * hc)
            return path(chunk_bufs[c], qi, ki, vi, R_h[:, hs], alpha[hs])

        def e2e_step():
            cur = torch.cuda.current_stream(dev)
            for s_ in (s_in, s_cmp, s_out):
                s_.wait_stream(cur)
            for c in range(n_chunks):
                hs = slice(c * hc, (c + 1) * hc)
                with torch.cuda.stream(s_in):
                    qd[:, hs].copy_(host["q"][:, hs], non_blocking=True)
                    kd[:, hs].copy_(host["k"][:, hs], non_blocking=True)
                    vd[:, hs].copy_(host["v"][:, hs], non_blocking=True)
                    ev_in[c].record(s_in)
                with torch.cuda.stream(s_cmp):
                    s_cmp.wait_event(ev_in[c])
                    o, lse = chunk_step(c, qd[:, hs], kd[:, hs], vd[:, hs])
                    ev_cmp[c].record(s_cmp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_cmp[c])
                    o_host[:, hs].copy_(o, non_blocking=True)
                    lse_host[:, hs].copy_(lse, non_blocking=True)
            for s_ in (s_in, s_cmp, s_out):
                cur.wait_stream(s_)

        for _ in range(2):
            e2e_step()
        Ke = max(3, min(K, 20))
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record()
        for _ in range(Ke):
            e2e_step()
        e2.record()
        barrier()
        e_ms = max_over_ranks(s2.elapsed_time(e2), world, dev)
        # the pipelined step must give the one-stream step's result
        o_ref, _ = step(q, k, v)
        torch.cuda.synchronize()
        if not torch.equal(o_ref.cpu(), o_host):
            raise RuntimeError("pipelined end-to-end step disagrees with the one-stream step")
        e2e = {"value": round(job_flops / (e_ms / Ke * 1e-3) / 1e12, 3), "unit": "TFLOP/s",
               "ms_per_step": round(e_ms / Ke, 3), "steps": Ke,
               "pipeline": f"{n_chunks} head chunks on 3 streams (copy-in, compute, copy-out)",
               "h2d_bytes_per_step": 3 * B * H * L * D * 2, "d2h_bytes_per_step": B * H * L * D * 2 + B * H * L * 4}

    # the calls below run on the curve-order tensors: with gathered tiles the
    # step made no copies, so make them here, outside every timed region
    if gather and not args.no_refresh:
        bufs["qh"], bufs["kh"], bufs["vh"] = (api.permute_tokens(x, perm) for x in (q, k, v))

    # dense refresh on the same inputs and kept lists: the single-pass call
    # against the two-pass path (dense call, sparse call, refinement)
    refresh = None
    if not args.no_refresh and blk == 128:
        qs, ks, vs = (bufs["qh"], bufs["kh"], bufs["vh"]) if w.hilbert else (q, k, v)
        rb = dict(o_dense=torch.empty_like(q), o_sparse=torch.empty_like(q), R=torch.empty_like(q),
                  lse_dense=torch.empty((B, H, L), dtype=torch.float32, device=dev),
                  lse_sparse=torch.empty((B, H, L), dtype=torch.float32, device=dev),
                  kept_mass=torch.empty((B, H, L), dtype=torch.float32, device=dev))

        def fused():
            api.sparse_attn_refresh(qs, ks, vs, blk, bufs["idx"], bufs["cnt"], out=rb, status=status)

        def two_pass():
            api.sparse_attn_fwd(qs, ks, vs, blk, o=rb["o_dense"], lse=rb["lse_dense"], status=status)
            api.sparse_attn_fwd(qs, ks, vs, blk, bufs["idx"], bufs["cnt"], o=rb["o_sparse"], lse=rb["lse_sparse"],
                                status=status)
            api.refresh_refinement(rb["o_dense"], rb["o_sparse"], out=rb["R"])

        times = {}
        for name, fn in (("fused", fused), ("two_pass", two_pass)):
            fn()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            for _ in range(3):
                fn()
            a1.record()
            barrier()
            times[name] = a0.elapsed_time(a1) / 3
        dense_tflop = 4.0 * B * H * L * L * D / 1e12
        refresh = {"fused_ms": round(times["fused"], 3), "two_pass_ms": round(times["two_pass"], 3),
                   "dense_tflop": round(dense_tflop, 2),
                   "fused_dense_equiv_tflops": round(dense_tflop / (times["fused"] * 1e-3), 1),
                   "calls": "fused: bsa_sparse_attn_refresh; two-pass: dense + sparse bsa_sparse_attn_fwd + "
                            "bsa_refresh_refinement"}

    # mask reuse on the same inputs: drift of the block means against a
    # reference step, and scoring / selection restricted to the current mask
    reuse = None
    if not args.no_refresh:
        qp_ref = bufs["qp"] * 1.01
        kp_ref = bufs["kp"].clone()
        cand = bufs["mask"].clone()
        rprobs, rmask = torch.empty_like(bufs["probs"]), torch.empty_like(bufs["mask"])
        ridx, rcnt = torch.empty_like(bufs["idx"]), torch.empty_like(bufs["cnt"])
        qs_, ks_ = (bufs["qh"], bufs["kh"]) if w.hilbert else (q, k)

        def drift():
            api.block_drift(qp_ref, kp_ref, bufs["qp"], bufs["kp"], L, blk)

        def restricted():
            api.score_blocks(qs_, ks_, blk, bufs["qp"], bufs["kp"], rprobs, candidates=cand)
            api.select_topp_mask(rprobs, p, L, blk, D, rmask, ridx, rcnt, candidates=cand)

        rt = {}
        for name, fn in (("drift", drift), ("restricted_score_select", restricted)):
            fn()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            for _ in range(5):
                fn()
            a1.record()
            barrier()
            rt[name] = round(a0.elapsed_time(a1) / 5, 4)
        reuse = {"drift_ms": rt["drift"], "restricted_score_select_ms": rt["restricted_score_select"],
                 "candidates": "the step's own mask",
                 "kept_fraction_of_candidates": round(rcnt.double().sum().item() / max(cand.double().sum().item(), 1),
                                                      4)}

    # the interval (skip-list) form of the step's kept lists; a failure here
    # is reported in its own object and does not lose the step's line
    intervals = None
    if not args.no_refresh:
        try:
            qkv_ = (bufs["qh"], bufs["kh"], bufs["vh"]) if w.hilbert else (q, k, v)
            intervals = interval_timings(bufs["idx"], bufs["cnt"], L, blk, D, barrier, qkv=qkv_)
        except Exception as e:  # noqa: BLE001
            intervals = {"error": f"{type(e).__name__}: {e}"}

    # the coarse tail of the omitted blocks (D = 128, 128-token blocks)
    tail = None
    if not args.no_refresh and D == 128 and blk == 128:
        try:
            qs_, ks_, vs_ = (bufs["qh"], bufs["kh"], bufs["vh"]) if w.hilbert else (q, k, v)
            tail = tail_timings(qs_, ks_, vs_, bufs["mask"], bufs["idx"], bufs["cnt"], blk, barrier)
        except Exception as e:  # noqa: BLE001
            tail = {"error": f"{type(e).__name__}: {e}"}

    # FP8 Q.K^T attention over the step's kept lists (D = 128, 128-token blocks)
    fp8 = None
    if not args.no_refresh and D == 128 and blk == 128:
        try:
            qs_, ks_, vs_ = (bufs["qh"], bufs["kh"], bufs["vh"]) if w.hilbert else (q, k, v)
            fp8 = fp8_timings(qs_, ks_, vs_, bufs["idx"], bufs["cnt"], blk, flops, barrier,
                              load_peaks()[0]["hbm_gbs"])
        except Exception as e:  # noqa: BLE001
            fp8 = {"error": f"{type(e).__name__}: {e}"}

    # the elementwise calls (refinement at a refresh, standalone correction):
    # HBM-bound, three [B,H,L,D] bf16 streams each
    elementwise = None
    sweep = None
    if not args.no_refresh and blk == 128:
        peaks_e, _ = load_peaks()
        oa, ob_, oc = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        ew = {}
        for name, fn in (("refresh_refinement", lambda: api.refresh_refinement(bufs["oh"], q, out=oa)),
                         ("apply_correction", lambda: api.apply_correction(bufs["oh"], R_h, alpha, out=ob_))):
            fn()
            barrier()
            a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a0.record()
            for _ in range(10):
                fn()
            a1.record()
            barrier()
            ms = a0.elapsed_time(a1) / 10
            gbs = 3 * B * H * L * D * 2 / (ms * 1e-3) / 1e9
            ew[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_hbm": round(gbs / peaks_e["hbm_gbs"], 3)}
        elementwise = ew
        del oa, ob_, oc

        # the mask-reuse sweep on this shape: Q and K drift by N(0, w.drift or
        # 0.05) per step (drawn on the device, outside the timed region); the
        # mask is recomputed every 3rd step, a dense refresh renews R every 5th
        # step, the other steps run sparse attention with the fused alpha*R
        if w.hilbert:
            gen = torch.Generator(device=dev)
            gen.manual_seed(2024)
            qd_, kd_ = q.clone(), k.clone()
            sigma = w.drift if w.drift > 0 else 0.05
            Rs = torch.zeros_like(q)
            sb = dict(o_dense=torch.empty_like(q), o_sparse=torch.empty_like(q), R=Rs,
                      lse_dense=torch.empty((B, H, L), dtype=torch.float32, device=dev),
                      lse_sparse=torch.empty((B, H, L), dtype=torch.float32, device=dev))
            Rg = torch.zeros_like(q)  # the refinement in grid order, for the gathering attention
            steps_ms, kinds = [], []
            for st_ in range(10):
                if st_ > 0:
                    for x in (qd_, kd_):
                        x.copy_((x.float() + sigma * torch.randn(x.shape, generator=gen, device=dev)).to(x.dtype))
                barrier()
                a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a0.record()
                b_ = bufs
                refresh_step = st_ % 5 == 0
                # the refresh runs on reordered copies; sparse steps gather their tiles
                copies = refresh_step or not gather
                if st_ % 3 == 0:
                    api.score_blocks_gather(qd_, kd_, perm, blk, b_["qh"] if copies else None,
                                            b_["kh"] if copies else None, b_["qp"], b_["kp"], b_["probs"],
                                            copies=copies)
                    api.select_topp_mask(b_["probs"], p, L, blk, D, b_["mask"], b_["idx"], b_["cnt"])
                elif copies:
                    api.permute_tokens(qd_, perm, out=b_["qh"])
                    api.permute_tokens(kd_, perm, out=b_["kh"])
                if copies:
                    api.permute_tokens(v, perm, out=b_["vh"])
                if refresh_step:
                    api.sparse_attn_refresh(b_["qh"], b_["kh"], b_["vh"], blk, b_["idx"], b_["cnt"], want_mass=False,
                                            out=sb, status=status)
                    api.permute_tokens(sb["o_dense"], perm, inverse=True, out=b_["o"])
                    if gather:
                        api.permute_tokens(Rs, perm, inverse=True, out=Rg)
                    kinds.append("refresh")
                else:
                    if gather:
                        api.sparse_attn_fwd(qd_, kd_, v, blk, b_["idx"], b_["cnt"], Rg, alpha, b_["o"], b_["lse"],
                                            status=status, in_rows=perm)
                    else:
                        api.sparse_attn_fwd(b_["qh"], b_["kh"], b_["vh"], blk, b_["idx"], b_["cnt"], Rs, alpha,
                                            b_["o"], b_["lse"], status=status, out_rows=perm)
                    kinds.append("sparse+mask" if st_ % 3 == 0 else "sparse, mask reused")
                a1.record()
                barrier()
                steps_ms.append(round(a0.elapsed_time(a1), 3))
            sweep = {"steps_ms": steps_ms, "kinds": kinds, "total_ms": round(float(np.sum(steps_ms)), 3),
                     "schedule": f"mask every 3rd step, dense refresh every 5th, Q/K drift N(0, {sigma}) per step"}

    if status.item() != 0:
        raise RuntimeError(f"attention kernel reported status {status.item()}")

    peaks, peak_src = load_peaks()
    attn_avg_ms = float(np.mean(attn_ms))
    achieved = flops / (attn_avg_ms * 1e-3) / 1e12
    traffic = profiled_traffic(w.name, w.blk)
    # the attention launch is timed alone (CUDA events around each call), so
    # its peak is the measured burst bf16 figure; the sustained one is context
    roofline = {"bound": "tensor", "achieved": round(achieved, 2),
                "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(achieved / peaks["bf16_tflops"], 4),
                "traffic": traffic, "kernel": attention_kernel(w.blk)[1],
                "peak_kind": f"{peak_src} burst bf16 (cuBLAS 8192^3)",
                "peak_sustained": peaks["bf16_tflops_sustained"],
                "frac_of_sustained": round(achieved / peaks["bf16_tflops_sustained"], 4)}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        f, s, n, what = oracle_sample(w, p, args.cpu_seconds)
        cpu = {"value": round(f / s / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
               "sample": what, "seconds": round(s, 2)}

    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
        "scaling": "strong" if strong else "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "B": B, "H": w.H, "L": L, "D": D, "blk": blk, "grid": list(w.grid),
                   "hilbert": w.hilbert,
                   "reorder": ("attention tiles gathered from the grid-order tensors" if gather else
                               "reordered copies of Q, K, V" if w.hilbert else "none"),
                   "top_p": p, "block_sparsity": round(sparsity, 4),
                   "fused_correction": True, "kept_tflop_per_step": round(job_flops / 1e12, 4),
                   "l2": f"inputs larger than L2 (Q/K/V {3 * B * H * L * D * 2 / 1e9:.2f} GB per step per GPU), "
                         "no flush",
                   "parallelism": (f"heads sharded over {world} GPUs: rank r takes heads [r*H/N, (r+1)*H/N) "
                                   f"(rank 0: {H}), no collective" if strong
                                   else f"independent replicas x{world} (no collective)")},
        "attn": {"ms_per_call": round(attn_avg_ms, 4), "ms_p10": round(float(np.percentile(attn_ms, 10)), 4),
                 "ms_p90": round(float(np.percentile(attn_ms, 90)), 4), "kept_tflops": round(achieved, 2),
                 "dense_equiv_tflops": round(4.0 * B * H * L * L * D / (attn_avg_ms * 1e-3) / 1e12, 2)},
        "stages_ms": {"gather_score_and_select": round(float(np.mean(sel_ms)), 4), "attention": round(attn_avg_ms, 4),
                      "rest": round(ms_step - attn_avg_ms - float(np.mean(sel_ms)), 4)},
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "refresh": refresh, "reuse": reuse,
        "elementwise": elementwise, "sweep": sweep, "intervals": intervals, "tail": tail, "fp8": fp8,
        "gpu_launches": (LAUNCHES_PER_STEP + (1 if w.hilbert and not gather else 0)) * K,
        "clocks": clk,
    }
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# -------------------------------------------------------------- reference

def run_reference(args, w, world, rank):
    if rank != 0:
        return
    p = float(w.p[0])
    blocks = 12  # query blocks of head 0 per step
    times, flops = [], []
    for i in range(max(args.warmup, 3) + args.steps):
        f, s, n, what = oracle_sample(w, p, seconds=1e9, max_blocks=blocks)
        if i >= max(args.warmup, 3):
            times.append(s)
            flops.append(f)
    sec = float(np.sum(times))
    value = float(np.sum(flops)) / sec / 1e12
    cores = blas_threads()
    out = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(sec / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "strong" if (world > 1 and args.shard == "heads") else "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "D": w.D, "blk": w.blk,
                   "grid": list(w.grid), "hilbert": w.hilbert, "top_p": p,
                   "parallelism": "CPU oracle on rank 0"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": f"per step: {what}"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    args = parse_args()
    world, rank, local = dist_info()
    if world != args.gpus and world > 1:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    w = configs.ALL[args.workload]
    if args.heads:
        import dataclasses
        w = dataclasses.replace(w, H=min(args.heads, w.H))
    if args.top_p:
        import dataclasses
        w = dataclasses.replace(w, p=(float(args.top_p),))
    if args.impl == "reference":
        run_reference(args, w, world, rank)
    else:
        run_ours(args, w, world, rank, local)


if __name__ == "__main__":
    main()
