"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (all heads of a workload in one call).

Exact checks run on every element the oracle can afford (Hilbert order,
selection on all rows given the same float32 scores); the attention output
is compared on sampled query blocks that the oracle computes one by one
(the first and last block of sampled heads and random blocks between), and
the masks the GPU selects from its own scores are checked to be valid top-p
selections of those scores wherever they differ from the oracle's.
"""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api, configs
from block_sparse_attention_logits_b200.synthetic import drift_, make_qkv, random_bf16
from oracle import attention as oatt
from oracle import correction as ocor
from oracle import hilbert as ohil
from oracle import refresh as oref
from oracle import scoring as osco
from oracle import topp as otop

from .gpu_helpers import assert_attention_close, assert_probs_close, to_np

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda"


def _oracle_probs(qn, kn, blk):
    """Oracle block probabilities one head at a time (bounded float64 copies)."""
    B, H, L, D = qn.shape
    nb = (L + blk - 1) // blk
    P = np.empty((B, H, nb, nb), np.float32)
    for h in range(H):
        _, _, P[:, h:h + 1] = osco.score_blocks(qn[:, h:h + 1], kn[:, h:h + 1], blk)
    return P


def _valid_topp(P_row, p, kept):
    """Property check of a selection: mass reaches T, dropping its smallest
    member falls below T, and no dropped block outranks a kept one."""
    row = np.where(np.isnan(P_row) | (P_row <= 0), 0, np.minimum(P_row, 1)).astype(np.float32)
    u = np.floor(row.astype(np.float64) * 2.0 ** 40)
    T = math.ceil(float(np.float32(p)) * u.sum())
    if np.float32(p) == 1:
        return kept.size == row.size
    if u[kept].sum() < T:
        return False
    worst = min(kept, key=lambda j: (row[j], -j))
    if u[kept].sum() - u[worst] >= T:
        return False
    dropped = np.setdiff1d(np.arange(row.size), kept)
    return not dropped.size or max((row[j], -j) for j in dropped) < (row[worst], -worst)


def _sample_units(H, NB, rng, heads=3, per_head=4):
    hs = sorted(set([0, H - 1] + list(rng.choice(H, heads, replace=False))))[:heads + 1]
    units = []
    for h in hs:
        blocks = set([0, NB - 1]) | set(int(i) for i in rng.choice(NB, per_head, replace=False))
        units += [(0, h, i) for i in sorted(blocks)]
    return units


def _run_workload(w, p, correction):
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    q, k, v = t["q"], t["k"], t["v"]
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    perm_o = None
    if w.hilbert:
        perm, _ = api.reorder_tokens(*w.grid, device=DEV)
        perm_o, inv_o = ohil.hilbert_perm(*w.grid)
        torch.cuda.synchronize()
        assert np.array_equal(to_np(perm), perm_o)
        qd, kd, vd = (api.permute_tokens(x, perm) for x in (qd, kd, vd))
    qn, kn, vn = (x.float().numpy() for x in (q, k, v))
    if perm_o is not None:
        qn, kn, vn = (ohil.permute_rows(x, perm_o) for x in (qn, kn, vn))
    # scoring on the GPU against the oracle
    _, _, P = api.score_blocks(qd, kd, w.blk)
    Po = _oracle_probs(qn, kn, w.blk)
    torch.cuda.synchronize()
    Pg = to_np(P)
    assert_probs_close(Pg, Po, f"{w.name} probs")
    pvec = np.full(w.H, p, np.float32)
    # selection: bit-exact on the oracle's scores, all rows
    mask_o, idx_o, cnt_o = otop.select_topp_mask_fast(Po, pvec)
    mask_g, idx_g, cnt_g = api.select_topp_mask(torch.from_numpy(Po).to(DEV), list(pvec), w.L, w.blk, w.D)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(cnt_g), cnt_o)
    assert np.array_equal(to_np(mask_g), mask_o)
    # selection on the GPU's own scores: same rows almost everywhere, valid everywhere
    mask_s, idx_s, cnt_s = api.select_topp_mask(P, list(pvec), w.L, w.blk, w.D)
    torch.cuda.synchronize()
    ms, cs, ids = to_np(mask_s), to_np(cnt_s), to_np(idx_s)
    differ = np.argwhere(~np.all(ms == mask_o, axis=-1))
    assert len(differ) <= 0.005 * w.H * w.NB, f"{len(differ)} rows select differently"
    for (b, h, i) in differ[:200]:
        assert _valid_topp(Pg[b, h, i], pvec[h], ids[b, h, i, :cs[b, h, i]])
    # attention with the oracle's kept lists, fused correction when asked
    R = alpha = None
    if correction:
        R = random_bf16(q.shape, 4242, scale=0.05)
        alpha = torch.tensor(w.alpha(), dtype=torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd(qd, kd, vd, w.blk, torch.from_numpy(idx_o).to(DEV),
                                 torch.from_numpy(cnt_o).to(DEV),
                                 None if R is None else R.to(DEV), None if alpha is None else alpha.to(DEV),
                                 status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    units = _sample_units(w.H, w.NB, np.random.default_rng(7))
    O, LSE = oatt.masked_attention(qn, kn, vn, idx_o, cnt_o, w.blk, units=units)
    if correction:
        O = ocor.apply_correction(O, R.float().numpy(), alpha.numpy())
    assert_attention_close(to_np(o), to_np(lse), O, LSE, f"{w.name} sampled blocks")
    return 1.0 - cnt_o.sum() / (w.H * w.NB ** 2)


@pytest.mark.parametrize("p", [0.9, 0.97])
def test_fullsize_wan13b_480p(p):
    _run_workload(configs.WAN13B_480P, p, correction=False)


def test_fullsize_wan14b_720p():
    w = configs.WAN14B_720P
    sparsity = _run_workload(w, w.p[0], correction=False)
    assert 0.89 <= sparsity <= 0.91, sparsity


def test_fullsize_hunyuan_720p_with_fused_correction():
    w = configs.HUNYUAN_720P
    sparsity = _run_workload(w, w.p[0], correction=True)
    assert 0.94 <= sparsity <= 0.96, sparsity


def test_mask_reuse_sweep_720p_shape():
    """Ten drifting denoising steps on the 720P shape (4 heads): the mask is
    recomputed at steps 0, 3, 6, 9 and reused otherwise; a dense refresh at
    steps 0 and 5 renews R = bf16(O_dense - O_sparse); every other step runs
    sparse attention with the fused alpha*R.  Each step's output is checked
    on sampled query blocks against the oracle following the same schedule."""
    import dataclasses
    w = dataclasses.replace(configs.REUSE_SWEEP, H=4)
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    q, k, v = t["q"], t["k"], t["v"]
    perm, _ = api.reorder_tokens(*w.grid, device=DEV)
    perm_o, _ = ohil.hilbert_perm(*w.grid)
    vd = api.permute_tokens(v.to(DEV), perm)
    vn = ohil.permute_rows(v.float().numpy(), perm_o)
    alpha = torch.tensor(w.alpha(), dtype=torch.float32)
    pvec = np.full(w.H, w.p[0], np.float32)
    # one fixed row sample for the whole sweep, so the oracle carries its own
    # refinement R from a refresh to the later steps
    units = _sample_units(w.H, w.NB, np.random.default_rng(11), heads=2, per_head=2)
    ones = np.tile(np.arange(w.NB, dtype=np.int32), (w.B, w.H, w.NB, 1))
    full = np.full((w.B, w.H, w.NB), w.NB, np.int32)
    idx_o = cnt_o = None
    R_g = R_o = None
    for step in range(w.steps):
        if step > 0:
            drift_(q, w.drift, seed=101, step=step)
            drift_(k, w.drift, seed=202, step=step)
        qd = api.permute_tokens(q.to(DEV), perm)
        kd = api.permute_tokens(k.to(DEV), perm)
        qn = ohil.permute_rows(q.float().numpy(), perm_o)
        kn = ohil.permute_rows(k.float().numpy(), perm_o)
        if step % w.mask_every == 0:
            # the oracle's mask, applied by both sides (bit-exact selection is
            # covered by the other tests)
            Po = _oracle_probs(qn, kn, w.blk)
            _, idx_o, cnt_o = otop.select_topp_mask_fast(Po, pvec)
            idx_d, cnt_d = torch.from_numpy(idx_o).to(DEV), torch.from_numpy(cnt_o).to(DEV)
        Os, Ls = oatt.masked_attention(qn, kn, vn, idx_o, cnt_o, w.blk, units=units)
        if step % w.refresh_every == 0:
            # dense refresh: the step's output is the dense attention, and the
            # refinement R = bf16(O_dense - O_sparse) is renewed on both sides
            od, lse = api.sparse_attn_fwd(qd, kd, vd, w.blk)
            os_, _ = api.sparse_attn_fwd(qd, kd, vd, w.blk, idx_d, cnt_d)
            R_g = api.refresh_refinement(od, os_)
            out = od
            Od, Ld = oatt.masked_attention(qn, kn, vn, ones, full, w.blk, units=units)
            sel = ~np.isnan(Od)
            R_o = np.full(Od.shape, np.nan)
            R_o[sel] = ocor.refresh_refinement(ocor.bf16_round(Od[sel]), ocor.bf16_round(Os[sel]))
            ref_O, ref_L = Od, Ld
            torch.cuda.synchronize()
            # R from the GPU's two bf16 outputs vs R from the oracle's: the
            # outputs agree to the attention tolerance, so R does too
            got_R = to_np(R_g)
            assert np.max(np.abs(got_R[sel] - R_o[sel])) <= 2 * 2e-2
        else:
            out, lse = api.sparse_attn_fwd(qd, kd, vd, w.blk, idx_d, cnt_d, R_g, alpha.to(DEV))
            ref_O = ocor.apply_correction(Os, R_o, alpha.numpy())
            ref_L = Ls
        torch.cuda.synchronize()
        assert_attention_close(to_np(out), to_np(lse), ref_O, ref_L, f"sweep step {step}")


def test_fused_refresh_720p_shape():
    """The single-pass refresh on the 720P shape (4 heads, Hilbert order, the
    oracle's kept lists): dense and sparse outputs, R and the kept share on
    sampled query blocks against the oracle, and every element against the
    library's two-pass path (dense call, sparse call, refresh_refinement)."""
    import dataclasses
    w = dataclasses.replace(configs.WAN14B_720P, H=4)
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    perm, _ = api.reorder_tokens(*w.grid, device=DEV)
    perm_o, _ = ohil.hilbert_perm(*w.grid)
    qd, kd, vd = (api.permute_tokens(t[n].to(DEV), perm) for n in "qkv")
    qn, kn, vn = (ohil.permute_rows(t[n].float().numpy(), perm_o) for n in "qkv")
    Po = _oracle_probs(qn, kn, w.blk)
    _, idx_o, cnt_o = otop.select_topp_mask_fast(Po, np.full(w.H, w.p[0], np.float32))
    idx_d, cnt_d = torch.from_numpy(idx_o).to(DEV), torch.from_numpy(cnt_o).to(DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    od, ld, os_, ls, R, mass = api.sparse_attn_refresh(qd, kd, vd, w.blk, idx_d, cnt_d, status=status)
    o1, l1 = api.sparse_attn_fwd(qd, kd, vd, w.blk)
    o2, l2 = api.sparse_attn_fwd(qd, kd, vd, w.blk, idx_d, cnt_d)
    R2 = api.refresh_refinement(o1, o2)
    torch.cuda.synchronize()
    assert status.item() == 0
    units = _sample_units(w.H, w.NB, np.random.default_rng(13), heads=2, per_head=3)
    Od, Ld, Os, Ls, Rr, Mr = oref.fused_refresh(qn, kn, vn, idx_o, cnt_o, w.blk, units=units)
    assert_attention_close(to_np(od), to_np(ld), Od, Ld, "fused dense")
    assert_attention_close(to_np(os_), to_np(ls), Os, Ls, "fused sparse")
    sel = ~np.isnan(Od)
    assert np.max(np.abs(to_np(R)[sel] - Rr[sel])) <= 2 * 2e-2
    msel = ~np.isnan(Ld)
    assert np.max(np.abs(to_np(mass)[msel] - Mr[msel])) <= 2e-3
    # against the two-pass path, every element
    # one bf16 ulp of the output plus the accumulation-order difference
    assert bool(((od.float() - o1.float()).abs() <= 1e-2 + 2.0 ** -7 * o1.float().abs()).all())
    assert bool(((os_.float() - o2.float()).abs() <= 1e-2 + 2.0 ** -7 * o2.float().abs()).all())
    assert (R.float() - R2.float()).abs().max().item() <= 4e-2
    assert (ld - l1).abs().max().item() <= 1e-3 and (ls - l2).abs().max().item() <= 1e-3
