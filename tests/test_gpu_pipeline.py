"""GPU parity of the exact call sequence the benchmark times, against the
oracle's own chain.

The GPU side is `step.run_step`, the function bench.py times, in both of its
forms (reordered copies, or tiles gathered by the attention): Hilbert order,
pooling that gathers Q and K into curve order, the V gather, top-p selection
on the GPU's own block scores, and sparse attention with the fused
O + alpha*R epilogue writing O and LSE back to grid order.  The oracle side
runs its own chain from the same seeded inputs (oracle.hilbert,
oracle.scoring, oracle.topp, oracle.attention, oracle.correction); no GPU
result is fed to it.

Rows where the GPU's selection (made from its float32 scores) equals the
oracle's are compared with the oracle's output.  Where the two selections
differ (float32 scores that differ in the last bits can tip a top-p cut),
the GPU's kept list is first checked to be a valid top-p selection of the
GPU's scores, and the row's output is then compared with the oracle's
attention over that list.  So every compared row is checked against an
oracle value.

Two launch configurations:
  * the 480P shape with 2 heads, every element of O and LSE, with and
    without the Hilbert path: 512 work items, at least 3 per CTA on 148
    SMs, which runs the persistent kernel's item queue wrap, its O double
    buffer across items, the statistics buffer parity and the K/V ring phases
    carried across items;
  * the 720P workload (the benchmark's), 4 heads, on sampled query blocks
    plus every row whose selection differs in the sampled heads.
"""

import dataclasses
import math

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api, configs
from block_sparse_attention_logits_b200.step import alloc_buffers, run_step
from block_sparse_attention_logits_b200.synthetic import make_qkv, random_bf16
from oracle import attention as oatt
from oracle import correction as ocor
from oracle import hilbert as ohil
from oracle import scoring as osco
from oracle import topp as otop

from .gpu_helpers import assert_attention_close, assert_probs_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _valid_topp(P_row, p, kept):
    """A selection is valid top-p for its scores: its fixed-point mass reaches
    the target, dropping its smallest member falls below it, and no dropped
    block outranks a kept one in the (P desc, index asc) order."""
    row = otop.clamp_probs(P_row)
    u = np.floor(row.astype(np.float64) * 2.0 ** otop.FIXED_POINT_BITS)
    T = math.ceil(float(np.float32(p)) * u.sum())
    if np.float32(p) == 1:
        return kept.size == row.size
    if kept.size == 0 or u[kept].sum() < T:
        return False
    worst = min(kept, key=lambda j: (row[j], -j))
    if kept.size > 1 and u[kept].sum() - u[worst] >= T:
        return False
    dropped = np.setdiff1d(np.arange(row.size), kept)
    return not dropped.size or max((row[j], -j) for j in dropped) < (row[worst], -worst)


def _run_bench_step(w, q, k, v, R, alpha, p, gather):
    """The benchmark's step on the device; returns host copies of what it wrote."""
    perm = api.reorder_tokens(*w.grid, device=DEV)[0] if w.hilbert else None
    bufs = alloc_buffers(w.B, w.H, w.L, w.D, w.blk, DEV, copies=not gather)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    side = torch.cuda.Stream()  # the V gather beside softmax and selection, as the benchmark runs it
    o, lse = run_step(bufs, q.to(DEV), k.to(DEV), v.to(DEV), w.blk, p, perm, R.to(DEV), alpha.to(DEV), status,
                      gather=gather, side=side)
    torch.cuda.synchronize()
    assert status.item() == 0, f"status {status.item()}"
    out = {n: to_np(bufs[n]) for n in ("probs", "mask", "idx", "cnt")}
    out["o"], out["lse"] = to_np(o), to_np(lse)
    out["perm"] = None if perm is None else to_np(perm)
    return out


def _check(w, p, units_of=None, gather=False):
    """Run both chains and compare.  units_of(H, NB, differ) -> query blocks
    to compare (None: every block).  gather: the step's gathering form (R in
    grid order) instead of the reordered copies (R in curve order)."""
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    q, k, v = t["q"], t["k"], t["v"]
    R = random_bf16(q.shape, 77, scale=0.05)  # refinement
    alpha = torch.tensor(w.alpha(), dtype=torch.float32)
    g = _run_bench_step(w, q, k, v, R, alpha, p, gather)

    # oracle chain from the same seeded inputs
    qn, kn, vn = (x.float().numpy() for x in (q, k, v))
    perm_o = None
    if w.hilbert:
        perm_o, _ = ohil.hilbert_perm(*w.grid)
        assert np.array_equal(g["perm"], perm_o), "Hilbert order differs"
        qn, kn, vn = (ohil.permute_rows(x, perm_o) for x in (qn, kn, vn))
    Po = np.empty_like(g["probs"])
    for h in range(w.H):
        _, _, Po[:, h:h + 1] = osco.score_blocks(qn[:, h:h + 1], kn[:, h:h + 1], w.blk)
    assert_probs_close(g["probs"], Po, f"{w.name} block scores")
    pvec = np.full(w.H, p, np.float32)
    mask_o, idx_o, cnt_o = otop.select_topp_mask_fast(Po, pvec)

    # rows where the GPU's selection from its own scores differs: valid top-p
    differ = np.argwhere(~np.all(g["mask"] == mask_o, axis=-1))
    assert len(differ) <= max(2, 0.005 * w.B * w.H * w.NB), f"{len(differ)} rows select differently"
    idx_use, cnt_use = idx_o.copy(), cnt_o.copy()
    for (b, h, i) in differ:
        kept = g["idx"][b, h, i, :g["cnt"][b, h, i]]
        assert np.array_equal(kept, np.flatnonzero(g["mask"][b, h, i])), "kept list and mask disagree"
        assert _valid_topp(g["probs"][b, h, i], pvec[h], kept), f"row {(b, h, i)} is not a valid top-p selection"
        idx_use[b, h, i, :kept.size] = kept
        cnt_use[b, h, i] = kept.size
    # kept lists agree with the oracle's wherever the masks do
    same = np.ones(cnt_o.shape, bool)
    same[tuple(differ.T)] = False
    assert np.array_equal(g["cnt"][same], cnt_o[same])
    for (b, h, i) in np.argwhere(same)[:: max(1, same.sum() // 500)]:
        assert np.array_equal(g["idx"][b, h, i, :cnt_o[b, h, i]], idx_o[b, h, i, :cnt_o[b, h, i]])

    units = None if units_of is None else units_of(w.H, w.NB, differ)
    O, LSE = oatt.masked_attention(qn, kn, vn, idx_use, cnt_use, w.blk, units=units)
    Rn = R.float().numpy()
    if w.hilbert and gather:  # R in grid order: the row each query token reads
        Rn = ohil.permute_rows(Rn, perm_o)
    O = ocor.apply_correction(O, Rn, alpha.numpy())
    if w.hilbert:  # back to grid order, as the epilogue writes it
        O = ohil.permute_rows(O, perm_o, inverse=True)
        LSE = ohil.permute_rows(LSE[..., None], perm_o, inverse=True)[..., 0]
    emax, emean, lrel = assert_attention_close(g["o"], g["lse"], O, LSE, f"{w.name} bench step")
    return len(differ), emax, emean, lrel


@pytest.mark.parametrize("mode", ["grid-order", "hilbert-copies", "hilbert-gather"])
def test_bench_step_every_element_480p_2heads(mode):
    """Every element of O and LSE, 512 work items (>= 3 per CTA)."""
    w = dataclasses.replace(configs.WAN13B_480P, H=2, hilbert=mode != "grid-order")
    assert w.B * w.H * w.NB >= 3 * 148
    _check(w, 0.9, gather=mode == "hilbert-gather")


@pytest.mark.parametrize("gather", [False, True], ids=["copies", "gather"])
def test_bench_step_720p_sampled(gather):
    """The benchmark's workload and calls, 4 heads: sampled query blocks
    (first and last of every head, 10 more per head) plus every row whose
    selection differs."""
    w = dataclasses.replace(configs.WAN14B_720P, H=4)
    rng = np.random.default_rng(5)

    def units_of(H, NB, differ):
        u = set()
        for h in range(H):
            u |= {(0, h, 0), (0, h, NB - 1)}
            u |= {(0, h, int(i)) for i in rng.choice(NB, 10, replace=False)}
        u |= {tuple(int(x) for x in d) for d in differ}
        return sorted(u)

    _check(w, w.p[0], units_of, gather=gather)
