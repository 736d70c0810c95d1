"""GPU parity: every C-ABI call against the CPU oracle on the same seeded inputs.

Sizes here span several tiles and ragged tails while the oracle still
finishes in seconds; the full-size workloads are in test_gpu_fullsize.py.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api, configs
from block_sparse_attention_logits_b200.synthetic import (FieldParams, make_qkv, random_bf16,
                                                          random_probs)
from oracle import attention as oatt
from oracle import correction as ocor
from oracle import hilbert as ohil
from oracle import scoring as osco
from oracle import topp as otop

from .gpu_helpers import (assert_attention_close, assert_pool_close, assert_probs_close, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _qkv(B, H, grid, D, fp):
    t = make_qkv(B, H, grid, D, fp)
    return t["q"], t["k"], t["v"]


def _select_exact(P_np, p, L, blk, D):
    """GPU selection on the oracle's float32 P must equal the oracle's bit for bit."""
    mask_o, idx_o, cnt_o = otop.select_topp_mask_fast(P_np, p)
    P = torch.from_numpy(P_np).to(DEV)
    mask, idx, cnt = api.select_topp_mask(P, list(p), L, blk, D)
    torch.cuda.synchronize()
    mask, idx, cnt = to_np(mask), to_np(idx), to_np(cnt)
    assert np.array_equal(cnt, cnt_o), f"counts differ in {np.sum(cnt != cnt_o)} rows"
    assert np.array_equal(mask, mask_o), "masks differ"
    valid = np.arange(P_np.shape[-1])[None, None, None, :] < cnt[..., None]
    assert np.array_equal(np.where(valid, idx, -1), idx_o), "kept lists differ"
    return mask_o, idx_o, cnt_o


# ------------------------------------------------------------------ scoring

@pytest.mark.parametrize("case", ["tiny", "480p_2heads", "ragged", "rows_1200", "rows_4000"])
def test_score_blocks_matches_oracle(case):
    """rows_*: one head with 1200 and 4000 key blocks per row (the largest
    rows the exact selection takes are 4096 blocks), beyond the rows the block
    softmax normalises in registers (1024)."""
    if case.startswith("rows_"):
        nb = int(case[5:])
        L = nb * 128 - 37
        q = random_bf16((1, 1, L, 128), 7)
        k = random_bf16((1, 1, L, 128), 8)
        blk = 128
    elif case == "tiny":
        w = configs.TINY
        q, k, _ = _qkv(w.B, w.H, w.grid, w.D, w.fp)
        blk = w.blk
    elif case == "480p_2heads":
        w = configs.WAN13B_480P
        q, k, _ = _qkv(1, 2, w.grid, w.D, w.fp)
        blk = w.blk
    else:
        q = random_bf16((2, 3, 1000, 128), 5)
        k = random_bf16((2, 3, 1000, 128), 6)
        blk = 128
    qp, kp, P = api.score_blocks(q.to(DEV), k.to(DEV), blk)
    torch.cuda.synchronize()
    qo, ko, Po = osco.score_blocks(q.float().numpy(), k.float().numpy(), blk)
    assert_pool_close(to_np(qp), qo, "q_pool")
    assert_pool_close(to_np(kp), ko, "k_pool")
    assert_probs_close(to_np(P), Po, "probs")


# ---------------------------------------------------------------- selection

def test_select_exact_on_oracle_scores_tiny():
    w = configs.TINY
    q, k, _ = _qkv(w.B, w.H, w.grid, w.D, w.fp)
    _, _, P = osco.score_blocks(q.float().numpy(), k.float().numpy(), w.blk)
    _select_exact(P, np.array([0.9, 0.6], np.float32), w.L, w.blk, w.D)


@pytest.mark.parametrize("p", [0.9, 0.97])
def test_select_exact_on_oracle_scores_480p(p):
    w = configs.WAN13B_480P
    q, k, _ = _qkv(1, 2, w.grid, w.D, w.fp)
    _, _, P = osco.score_blocks(q.float().numpy(), k.float().numpy(), w.blk)
    _select_exact(P, np.array([p, p], np.float32), w.L, w.blk, w.D)


@pytest.mark.parametrize("nb,ties", [(37, True), (37, False), (929, False), (1, False), (300, True), (256, False),
                                     (257, True), (640, False), (641, True), (1024, False), (1100, True)])
def test_select_exact_random_rows(nb, ties):
    P = random_probs(2, 3, nb, seed=nb + 10 * ties, temperature=2.0, ties=ties)
    _select_exact(P, np.array([0.9, 0.35, 1.0], np.float32), nb * 128, 128, 128)


def test_select_exact_degenerate_rows():
    nb = 40
    P = random_probs(1, 2, nb, seed=3).copy()
    P[0, 0, 0] = 0.0                       # all-zero row
    P[0, 0, 1, :5] = np.nan                # NaNs clamp to 0
    P[0, 0, 2, 3] = 7.0                    # > 1 clamps to 1
    P[0, 0, 3] = 1.0 / nb                  # all equal
    P[0, 0, 4, :] = -1.0                   # all negative
    P[0, 0, 5, :] = 1e-30                  # below the fixed-point resolution
    P[0, 1, 6, :] = np.inf
    _select_exact(P, np.array([0.5, 0.999], np.float32), nb * 64, 64, 64)


# ----------------------------------------------------------------- reorder

@pytest.mark.parametrize("grid", [(2, 32, 32), (21, 30, 52), (21, 45, 80), (33, 45, 80), (3, 5, 7),
                                  (1, 1, 1), (1, 1, 256), (17, 1, 9)])
def test_reorder_tokens_exact(grid):
    perm, inv = api.reorder_tokens(*grid)
    torch.cuda.synchronize()
    perm_o, inv_o = ohil.hilbert_perm(*grid)
    assert np.array_equal(to_np(perm), perm_o)
    assert np.array_equal(to_np(inv), inv_o)


@pytest.mark.parametrize("D", [128, 64, 24])
def test_permute_tokens_exact(D):
    grid = (3, 5, 7)
    x = random_bf16((2, 3, 105, D), 11)
    perm_o, _ = ohil.hilbert_perm(*grid)
    perm = torch.from_numpy(perm_o).to(DEV)
    xd = x.to(DEV)
    y = api.permute_tokens(xd, perm)
    z = api.permute_tokens(y, perm, inverse=True)
    torch.cuda.synchronize()
    ref = ohil.permute_rows(x.view(torch.int16).numpy(), perm_o)
    assert np.array_equal(y.cpu().view(torch.int16).numpy(), ref)
    assert torch.equal(z.cpu(), x)


# --------------------------------------------------------------- attention

def _random_lists(B, H, nb, seed, density=0.3, empty_rows=()):
    rng = np.random.default_rng(seed)
    mask = rng.random((B, H, nb, nb)) < density
    mask[..., np.arange(nb), np.arange(nb)] = True
    for (b, h, i) in empty_rows:
        mask[b, h, i] = False
    cnt = mask.sum(-1).astype(np.int32)
    idx = np.full((B, H, nb, nb), -1, np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                kk = np.nonzero(mask[b, h, i])[0]
                idx[b, h, i, :kk.size] = kk
    return idx, cnt


def _run_attention(q, k, v, blk, idx, cnt, R=None, alpha=None):
    dev = lambda a: None if a is None else (torch.from_numpy(a).to(DEV) if isinstance(a, np.ndarray) else a.to(DEV))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd(dev(q), dev(k), dev(v), blk, dev(idx), dev(cnt), dev(R), dev(alpha),
                                 status=status)
    torch.cuda.synchronize()
    return to_np(o), to_np(lse), int(status.item())


@pytest.mark.parametrize("D,blk,L,H", [(128, 128, 1000, 2), (128, 128, 1300, 1), (64, 64, 2048, 2),
                                       (128, 64, 777, 2), (64, 128, 513, 2), (128, 128, 129, 1),
                                       (64, 64, 1, 1), (128, 128, 256, 3)])
def test_sparse_attention_random_lists(D, blk, L, H):
    B = 1
    q = random_bf16((B, H, L, D), 21 + L)
    k = random_bf16((B, H, L, D), 22 + L)
    v = random_bf16((B, H, L, D), 23 + L)
    nb = api.n_blocks(L, blk)
    idx, cnt = _random_lists(B, H, nb, seed=L, density=0.35)
    o, lse, st = _run_attention(q, k, v, blk, idx, cnt)
    assert st == 0
    O, LSE = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), idx, cnt, blk)
    assert_attention_close(o, lse, O, LSE, f"D={D} blk={blk} L={L}")


@pytest.mark.parametrize("D,blk,L", [(128, 128, 700), (64, 64, 650), (128, 64, 300)])
def test_dense_attention_matches_oracle(D, blk, L):
    q = random_bf16((1, 2, L, D), 31)
    k = random_bf16((1, 2, L, D), 32)
    v = random_bf16((1, 2, L, D), 33)
    o, lse, st = _run_attention(q, k, v, blk, None, None)
    assert st == 0
    O, LSE = oatt.dense_attention(q.float().numpy(), k.float().numpy(), v.float().numpy())
    assert_attention_close(o, lse, O, LSE, "dense")


def test_attention_empty_rows_and_bad_indices():
    D, blk, L, H = 128, 128, 900, 2
    q = random_bf16((1, H, L, D), 41)
    k = random_bf16((1, H, L, D), 42)
    v = random_bf16((1, H, L, D), 43)
    nb = api.n_blocks(L, blk)
    idx, cnt = _random_lists(1, H, nb, seed=4, empty_rows=[(0, 0, 1), (0, 1, 6), (0, 1, 2)])
    o, lse, st = _run_attention(q, k, v, blk, idx, cnt)
    assert st == 0
    O, LSE = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), idx, cnt, blk)
    assert_attention_close(o, lse, O, LSE, "empty rows")
    assert np.all(o[0, 0, 128:256] == 0) and np.all(np.isneginf(lse[0, 0, 128:256]))
    # out-of-range entries are skipped and flagged, never dereferenced
    bad = idx.copy()
    bad[0, 0, 0, 0] = nb + 5
    bad_cnt = cnt.copy()
    bad_cnt[0, 1, 3] = nb + 7
    _, _, st = _run_attention(q, k, v, blk, bad, bad_cnt)
    assert st & 2


def test_attention_tiny_config_with_oracle_masks_and_fused_correction():
    w = configs.TINY
    q, k, v = _qkv(w.B, w.H, w.grid, w.D, w.fp)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _, _, P = osco.score_blocks(qn, kn, w.blk)
    _, idx, cnt = otop.select_topp_mask(P, np.full(w.H, w.p[0], np.float32))
    o, lse, st = _run_attention(q, k, v, w.blk, idx, cnt)
    assert st == 0
    O, LSE = oatt.masked_attention(qn, kn, vn, idx, cnt, w.blk)
    assert_attention_close(o, lse, O, LSE, "tiny")
    # fused O + alpha_h R with a synthetic cached refinement
    R = random_bf16(q.shape, 51, scale=0.05)
    alpha = torch.tensor(w.alpha(), dtype=torch.float32)
    oc, lsec, st = _run_attention(q, k, v, w.blk, idx, cnt, R, alpha)
    assert st == 0
    Oc = ocor.apply_correction(O, R.float().numpy(), alpha.numpy())
    assert_attention_close(oc, lsec, Oc, LSE, "tiny fused correction")


def test_attention_480p_two_heads_sampled_blocks():
    w = configs.WAN13B_480P
    q, k, v = _qkv(1, 2, w.grid, w.D, w.fp)
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _, _, P = osco.score_blocks(qn, kn, w.blk)
    _, idx, cnt = otop.select_topp_mask_fast(P, np.full(2, 0.9, np.float32))
    o, lse, st = _run_attention(q, k, v, w.blk, idx, cnt)
    assert st == 0
    rng = np.random.default_rng(0)
    units = [(0, h, int(i)) for h in range(2) for i in rng.choice(w.NB, 12, replace=False)]
    units += [(0, 0, w.NB - 1), (0, 1, 0)]
    O, LSE = oatt.masked_attention(qn, kn, vn, idx, cnt, w.blk, units=units)
    assert_attention_close(o, lse, O, LSE, "480p sampled")


# -------------------------------------------------------------- correction

def test_refresh_refinement_bit_exact():
    od = random_bf16((1, 3, 333, 64), 61)
    os_ = (od.float() + 0.01 * random_bf16(od.shape, 62).float()).to(torch.bfloat16)
    R = api.refresh_refinement(od.to(DEV), os_.to(DEV))
    torch.cuda.synchronize()
    ref = ocor.refresh_refinement(od.float().numpy(), os_.float().numpy())
    assert np.array_equal(R.cpu().float().numpy().view(np.uint32), ref.view(np.uint32))


def test_apply_correction_matches_oracle():
    os_ = random_bf16((2, 3, 257, 128), 71)
    R = random_bf16(os_.shape, 72, scale=0.1)
    alpha = torch.tensor([0.0, 0.5, 1.0], dtype=torch.float32)
    out = api.apply_correction(os_.to(DEV), R.to(DEV), alpha.to(DEV))
    torch.cuda.synchronize()
    ref = ocor.apply_correction(os_.float().numpy(), R.float().numpy(), alpha.numpy())
    got = out.cpu().float().numpy()
    assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-30)
    assert torch.equal(out[:, 0].cpu(), os_[:, 0])
    # in place (o aliases o_sparse)
    inplace = os_.to(DEV)
    api.apply_correction(inplace, R.to(DEV), alpha.to(DEV), out=inplace)
    torch.cuda.synchronize()
    assert torch.equal(inplace.cpu(), out.cpu())


# ------------------------------------------------------------ whole path

def test_pipeline_tiny_end_to_end_through_the_abi():
    """GPU scoring -> GPU selection -> GPU attention, checked stage by stage."""
    w = configs.TINY
    q, k, v = _qkv(w.B, w.H, w.grid, w.D, w.fp)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    _, _, P = api.score_blocks(qd, kd, w.blk)
    mask, idx, cnt = api.select_topp_mask(P, w.p[0], w.L, w.blk, w.D)
    o, lse = api.sparse_attn_fwd(qd, kd, vd, w.blk, idx, cnt)
    torch.cuda.synchronize()
    qn, kn, vn = q.float().numpy(), k.float().numpy(), v.float().numpy()
    _, _, Po = osco.score_blocks(qn, kn, w.blk)
    assert_probs_close(to_np(P), Po)
    mask_o, idx_o, cnt_o = otop.select_topp_mask(Po, np.full(w.H, w.p[0], np.float32))
    same = np.all(to_np(mask) == mask_o, axis=-1)
    assert same.mean() >= 0.99, f"only {same.mean():.3f} of rows select identically"
    # attention of the rows whose selection agrees, from the oracle's own lists
    units = [tuple(int(x) for x in u) for u in np.argwhere(same)]
    O, LSE = oatt.masked_attention(qn, kn, vn, idx_o, cnt_o, w.blk, units=units)
    assert_attention_close(to_np(o), to_np(lse), O, LSE, "pipeline")
