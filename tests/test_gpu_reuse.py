"""GPU parity of the mask-reuse calls against the oracle: the per-head
query-key drift of the block means, scoring restricted to candidate blocks
and the restricted top-p selection (bit-exact given the same float32 scores),
with rows that have no candidates, candidates of zero mass, p = 1 heads and
ties.  Also the attention call that writes its output through a row map."""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api
from block_sparse_attention_logits_b200.synthetic import random_bf16
from oracle import reuse as oreu
from oracle import scoring as osco

from .gpu_helpers import assert_probs_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_drift_matches_oracle():
    rng = np.random.default_rng(50)
    B, H, NB, D, blk = 1, 4, 37, 128, 128
    L = NB * blk - 5
    ref_q = rng.standard_normal((B, H, NB, D)).astype(np.float32)
    ref_k = rng.standard_normal((B, H, NB, D)).astype(np.float32)
    q = ref_q + np.float32(0.05) * rng.standard_normal(ref_q.shape).astype(np.float32)
    k = ref_k.copy()
    k[0, 1] *= np.float32(1.3)   # head 1: the K change dominates
    q[0, 2] = ref_q[0, 2]        # head 2: no Q change
    k[0, 3] = ref_k[0, 3]
    q[0, 3] = ref_q[0, 3]        # head 3: identical -> exactly 0
    t = lambda a: torch.from_numpy(a).to(DEV)
    d = api.block_drift(t(ref_q), t(ref_k), t(q), t(k), L, blk)
    torch.cuda.synchronize()
    ref = oreu.block_drift(ref_q, ref_k, q, k).reshape(-1)
    got = to_np(d).astype(np.float64)
    assert np.allclose(got, ref, rtol=1e-5, atol=0)
    assert got[3] == 0
    z = np.zeros_like(ref_q)
    d0 = to_np(api.block_drift(t(z), t(z), t(z), t(z), L, blk))
    dinf = to_np(api.block_drift(t(z), t(ref_k), t(q), t(ref_k), L, blk))
    torch.cuda.synchronize()
    assert np.all(d0 == 0) and np.all(np.isinf(dinf))


def _candidates(B, H, NB, seed, frac=0.35):
    rng = np.random.default_rng(seed)
    c = (rng.random((B, H, NB, NB)) < frac).astype(np.uint8)
    c[0, 0, 2] = 0          # no candidates
    c[0, 1, 3] = 1          # every block a candidate
    return c


def test_restricted_scoring_matches_oracle():
    B, H, D, blk = 1, 2, 128, 128
    L = 9 * blk + 40
    q, k = random_bf16((B, H, L, D), 51, scale=1.5), random_bf16((B, H, L, D), 52, scale=1.5)
    NB = (L + blk - 1) // blk
    cand = _candidates(B, H, NB, 53)
    _, _, P = api.score_blocks(q.to(DEV), k.to(DEV), blk, candidates=torch.from_numpy(cand).to(DEV))
    torch.cuda.synchronize()
    qb, kb, _ = osco.score_blocks(q.float().numpy(), k.float().numpy(), blk)
    Pr = oreu.restricted_probs(qb, kb, cand)
    Pg = to_np(P)
    assert_probs_close(Pg, Pr, "restricted probs")
    assert np.all(Pg[cand == 0] == 0) and np.all(Pg[0, 0, 2] == 0)


@pytest.mark.parametrize("seed,NB", [(60, 45), (61, 45), (62, 600), (63, 1050)])
def test_restricted_selection_bit_exact(seed, NB):
    rng = np.random.default_rng(seed)
    B, H, blk, D = 1, 4, 128, 128
    L = NB * blk
    P = rng.dirichlet(np.full(NB, 0.3), size=(B, H, NB)).astype(np.float32)
    P[0, 1, 5, ::3] = P[0, 1, 5, 0]     # ties
    cand = _candidates(B, H, NB, seed + 1)
    P[0, 2, 7][cand[0, 2, 7] == 1] = 0  # candidates of zero mass (nothing to reach)
    pv = np.array([0.8, 0.9, 0.95, 1.0], np.float32)
    m, i, c = api.select_topp_mask(torch.from_numpy(P).to(DEV), list(pv), L, blk, D,
                                   candidates=torch.from_numpy(cand).to(DEV))
    torch.cuda.synchronize()
    mo, io, co = oreu.select_topp_mask_restricted(P, pv, cand)
    cg = to_np(c)
    assert np.array_equal(cg, co)
    assert np.array_equal(to_np(m), mo)
    ig = to_np(i)
    for b in range(B):
        for h in range(H):
            for r in range(NB):
                assert np.array_equal(ig[b, h, r, :cg[b, h, r]], io[b, h, r, :co[b, h, r]])
    assert cg[0, 0, 2] == 0
    assert np.all((to_np(m) == 1) <= (cand == 1))


def test_scatter_output_equals_attention_then_inverse_permute():
    """bsa_sparse_attn_fwd_scatter writes the same numbers as attention in curve
    order followed by the inverse permutation (both are this library's kernels;
    the curve-order attention itself is checked against the oracle elsewhere)."""
    from block_sparse_attention_logits_b200._lib import BSA_DEV_BAD_INDEX
    grid = (3, 9, 16)
    B, H, D, blk = 1, 2, 128, 128
    L = grid[0] * grid[1] * grid[2]
    NB = (L + blk - 1) // blk
    q, k, v = (random_bf16((B, H, L, D), 70 + j).to(DEV) for j in range(3))
    R = random_bf16((B, H, L, D), 73, scale=0.05).to(DEV)
    alpha = torch.tensor([0.3, 0.8], dtype=torch.float32, device=DEV)
    perm, _ = api.reorder_tokens(*grid, device=DEV)
    qh, kh, vh = (api.permute_tokens(x, perm) for x in (q, k, v))
    Rh = api.permute_tokens(R, perm)
    _, _, P = api.score_blocks(qh, kh, blk)
    _, idx, cnt = api.select_topp_mask(P, 0.9, L, blk, D)
    oh, lh = api.sparse_attn_fwd(qh, kh, vh, blk, idx, cnt, Rh, alpha)
    o_ref = api.permute_tokens(oh, perm, inverse=True)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd(qh, kh, vh, blk, idx, cnt, Rh, alpha, status=status, out_rows=perm)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(o, o_ref)
    lse_ref = torch.empty_like(lh)
    lse_ref[:, :, perm.long()] = lh
    assert torch.equal(lse, lse_ref)
    # an out-of-range row target is skipped and flagged
    bad = perm.clone()
    bad[5] = L + 3
    o2 = torch.zeros_like(o)
    api.sparse_attn_fwd(qh, kh, vh, blk, idx, cnt, Rh, alpha, o=o2, status=status, out_rows=bad)
    torch.cuda.synchronize()
    assert status.item() & BSA_DEV_BAD_INDEX
    keep = torch.ones(L, dtype=torch.bool, device=DEV)
    keep[perm[5].long()] = False
    assert torch.equal(o2[:, :, keep], o[:, :, keep])


def test_score_blocks_gather_equals_permute_then_score():
    """The gathering scorer gives the same bits as the two permutes followed by
    bsa_score_blocks (both this library's kernels; scoring itself is checked
    against the oracle elsewhere)."""
    grid = (3, 9, 16)
    B, H, D, blk = 1, 3, 128, 128
    L = grid[0] * grid[1] * grid[2]
    q, k = (random_bf16((B, H, L, D), 80 + j).to(DEV) for j in range(2))
    perm, _ = api.reorder_tokens(*grid, device=DEV)
    qh, kh = api.permute_tokens(q, perm), api.permute_tokens(k, perm)
    qp, kp, P = api.score_blocks(qh, kh, blk)
    q2, k2, qp2, kp2, P2 = api.score_blocks_gather(q, k, perm, blk)
    torch.cuda.synchronize()
    for a, b in ((qh, q2), (kh, k2), (qp, qp2), (kp, kp2), (P, P2)):
        assert torch.equal(a, b)
