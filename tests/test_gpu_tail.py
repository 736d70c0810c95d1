"""GPU parity of the coarse-tail calls against oracle/tail.py: block moments
(float32 against float64), the pooled covariance, the coarse tail, the
complement lists (bit-exact) and the reconstruction, which with a refinement
taken at the same step returns dense attention.

Two sizes: 677 tokens (6 blocks, one tile of pseudo-keys) and 38,350 tokens
(300 blocks: three tiles of 128 pseudo-keys, a ragged last block, and a
covariance split over 148 CTAs of which some get no tokens)."""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api
from block_sparse_attention_logits_b200.synthetic import random_bf16, random_kept_lists
from oracle import attention as oatt
from oracle import tail as otail

from .gpu_helpers import assert_attention_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bf16(a):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).float().numpy()


def _case(seed, L=5 * 128 + 37, H=2, keep=0.3):
    B, D, blk = 1, 128, 128
    NB = (L + blk - 1) // blk
    q = random_bf16((B, H, L, D), seed, scale=1.0)
    k = random_bf16((B, H, L, D), seed + 1, scale=1.0)
    # values that depend on the keys, so that the covariance term matters
    M = np.random.default_rng(seed + 5).standard_normal((D, D)) / np.sqrt(D)
    noise = random_bf16((B, H, L, D), seed + 2, scale=1.0).float().numpy()
    v = torch.from_numpy((0.8 * k.float().numpy() @ M.T + 0.5 * noise).astype(np.float32)).to(torch.bfloat16)
    idx, cnt = random_kept_lists(B, H, NB, seed + 3, keep, 1.5)
    mask = np.zeros((B, H, NB, NB), np.uint8)
    for pos in np.ndindex(B, H, NB):
        mask[pos + (idx[pos][:cnt[pos]].tolist(),)] = 1 if cnt[pos] else 0
    return q, k, v, idx, cnt, mask, blk


SIZES = [dict(L=5 * 128 + 37, H=2), dict(L=300 * 128 - 50, H=1)]


@pytest.mark.parametrize("size", SIZES, ids=["L677", "L38350"])
@pytest.mark.parametrize("seed", [1, 2])
def test_tail_stats_match_oracle(seed, size):
    q, k, v, idx, cnt, mask, blk = _case(10 * seed, **size)
    kbar, s2, vbar, C, _ = api.tail_stats(k.to(DEV), v.to(DEV), blk)
    torch.cuda.synchronize()
    kr, s2r, vr, n, Cr = otail.block_stats(k.float().numpy(), v.float().numpy(), blk)
    assert np.allclose(to_np(kbar), kr, rtol=1e-5, atol=1e-6)
    assert np.allclose(to_np(vbar), vr, rtol=1e-5, atol=1e-6)
    assert np.allclose(to_np(s2), s2r, rtol=1e-4, atol=1e-6)
    # C from bf16-rounded centred values with float32 accumulation: each product
    # is off by at most 2^-8 of its size
    kc = np.abs(k.float().numpy() - np.repeat(kr, blk, axis=2)[:, :, :k.shape[2]])
    vc = np.abs(v.float().numpy() - np.repeat(vr, blk, axis=2)[:, :, :k.shape[2]])
    bound = np.einsum("bhte,bhtd->bhed", vc, kc) / k.shape[2] * 2.0 ** -7 + 1e-6
    assert np.all(np.abs(to_np(C) - Cr) <= bound)


def test_complement_lists_bit_exact():
    q, k, v, idx, cnt, mask, blk = _case(5)
    ci, cc = api.complement_lists(torch.from_numpy(mask).to(DEV), q.shape[2], blk)
    torch.cuda.synchronize()
    from oracle.refresh import complement_lists
    ri, rc = complement_lists(idx, cnt, mask.shape[-1])
    assert np.array_equal(to_np(cc), rc)
    valid = np.arange(mask.shape[-1]) < rc[..., None]
    assert np.array_equal(np.where(valid, to_np(ci), -1), np.where(valid, ri, -1))


@pytest.mark.parametrize("size", SIZES, ids=["L677", "L38350"])
@pytest.mark.parametrize("seed", [3, 4])
def test_coarse_tail_matches_oracle_on_bf16_operands(seed, size):
    """The tail kernel multiplies bf16 operands: q, bf16(q^2), bf16(kbar),
    bf16(s2 / (2 sqrt D)), bf16(vbar), bf16(C).  The oracle evaluated on the
    same rounded operands differs only by float32 accumulation, exp2, the bf16
    weights of P.V and the bf16 output."""
    q, k, v, idx, cnt, mask, blk = _case(20 * seed, **size)
    dq = q.to(DEV)
    _, _, _, _, ws = api.tail_stats(k.to(DEV), v.to(DEV), blk)
    lbar, obar = api.coarse_tail(dq, torch.from_numpy(mask).to(DEV), blk, ws)
    torch.cuda.synchronize()
    kr, s2r, vr, n, Cr = otail.block_stats(k.float().numpy(), v.float().numpy(), blk)
    D = q.shape[-1]
    # the same rounded operands, expressed in the oracle's terms
    stats = (_bf16(kr), _bf16(s2r / (2 * np.sqrt(D))) * 2 * np.sqrt(D), _bf16(vr), n, _bf16(Cr))
    qf = q.float().numpy()
    lb_ref, ob_ref = otail.coarse_tail(qf, stats, idx, cnt, blk)
    lg, og = to_np(lbar), to_np(obar).astype(np.float64)
    fin = np.isfinite(lb_ref)
    assert np.array_equal(fin, np.isfinite(lg))
    # a model of the kernel's arithmetic lands within 5e-4 and 1.1e-3 of the
    # oracle here; a transposed C moves obar by ~0.5, a missing variance term
    # moves lbar by ~0.7
    assert np.abs(lg[fin] - lb_ref[fin]).max() <= 3e-3
    assert np.abs(og - ob_ref).max() <= 6e-3
    assert np.all(og[~fin] == 0)


def test_reconstruction_with_same_step_refinement_is_dense():
    q, k, v, idx, cnt, mask, blk = _case(7, keep=0.35)
    dq, dk, dv = q.to(DEV), k.to(DEV), v.to(DEV)
    ti, tc = torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV)
    tm = torch.from_numpy(mask).to(DEV)
    o_S, l_S = api.sparse_attn_fwd(dq, dk, dv, blk, ti, tc)
    ci, cc = api.complement_lists(tm, q.shape[2], blk)
    o_T, l_T = api.sparse_attn_fwd(dq, dk, dv, blk, ci, cc)
    _, _, _, _, ws = api.tail_stats(dk, dv, blk)
    lbar, obar = api.coarse_tail(dq, tm, blk, ws)
    d_l, d_o = api.tail_refinement(l_T, o_T, lbar, obar)
    o, lse = api.tail_reconstruct(l_S, o_S, lbar, obar, d_l, d_o)
    torch.cuda.synchronize()
    O, LSE = oatt.dense_attention(q.float().numpy(), k.float().numpy(), v.float().numpy())
    assert_attention_close(to_np(o), to_np(lse), O, LSE, "reconstruction")
