"""GPU parity of the single-pass dense refresh (bsa_sparse_attn_refresh)
against the oracle: dense and sparse outputs and LSEs, the refinement R and
the kept attention share, on several tiles with a ragged tail, D = 64 and 128,
rows that keep every block and rows that keep none, and malformed kept lists
(flagged, dense output unaffected)."""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api
from block_sparse_attention_logits_b200._lib import BSA_DEV_BAD_INDEX
from block_sparse_attention_logits_b200.synthetic import random_bf16
from oracle import refresh as oref

from .gpu_helpers import assert_attention_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
BLK = 128
MASS_ABS = 2e-3     # kept share: both sums are float32 over the same exponentials
R_MAX_ABS = 2 * 2e-2  # R is the difference of two outputs, each within 2e-2


def _lists(B, H, NB, seed, full_rows=(), empty_rows=()):
    rng = np.random.default_rng(seed)
    idx = np.zeros((B, H, NB, NB), np.int32)
    cnt = np.zeros((B, H, NB), np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(NB):
                if (h, i) in full_rows:
                    kept = np.arange(NB)
                elif (h, i) in empty_rows:
                    kept = np.zeros(0, np.int64)
                else:
                    kept = np.sort(rng.choice(NB, rng.integers(1, NB + 1), replace=False))
                idx[b, h, i, :len(kept)] = kept
                cnt[b, h, i] = len(kept)
    return idx, cnt


def _run(B, H, L, D, seed, full_rows=(), empty_rows=(), scale=1.0):
    NB = (L + BLK - 1) // BLK
    q, k, v = (random_bf16((B, H, L, D), seed + j, scale=scale if j < 2 else 1.0) for j in range(3))
    idx, cnt = _lists(B, H, NB, seed + 7, full_rows, empty_rows)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    outs = api.sparse_attn_refresh(q.to(DEV), k.to(DEV), v.to(DEV), BLK, torch.from_numpy(idx).to(DEV),
                                   torch.from_numpy(cnt).to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = oref.fused_refresh(q.float().numpy(), k.float().numpy(), v.float().numpy(), idx, cnt, BLK)
    return [to_np(t) for t in outs], ref, (q, k, v, idx, cnt)


@pytest.mark.parametrize("D,L", [(128, 5 * 128 + 37), (64, 4 * 128 + 1), (128, 3 * 128)])
def test_refresh_matches_oracle(D, L):
    (od, ld, os_, ls, R, mass), (Od, Ld, Os, Ls, Rr, Mr), _ = _run(1, 2, L, D, seed=100 + D, scale=1.5)
    assert_attention_close(od, ld, Od, Ld, "dense")
    assert_attention_close(os_, ls, Os, Ls, "sparse")
    assert np.max(np.abs(R.astype(np.float64) - Rr)) <= R_MAX_ABS
    assert np.max(np.abs(mass - Mr)) <= MASS_ABS
    assert np.all((mass > 0) & (mass <= 1))


def test_refresh_all_kept_and_empty_rows():
    full = {(0, 0), (1, 2)}
    empty = {(0, 1), (1, 3)}
    (od, ld, os_, ls, R, mass), (Od, Ld, Os, Ls, Rr, Mr), _ = _run(1, 2, 4 * 128 + 50, 128, seed=200,
                                                                   full_rows=full, empty_rows=empty)
    assert_attention_close(od, ld, Od, Ld, "dense")
    assert_attention_close(os_, ls, Os, Ls, "sparse")
    for h, i in full:
        rows = slice(i * BLK, min((i + 1) * BLK, od.shape[2]))
        # one set of accumulators: the two outputs are the same numbers
        assert np.array_equal(od[0, h, rows], os_[0, h, rows])
        assert np.array_equal(ld[0, h, rows], ls[0, h, rows])
        assert np.all(R[0, h, rows] == 0) and np.all(mass[0, h, rows] == 1.0)
    for h, i in empty:
        rows = slice(i * BLK, min((i + 1) * BLK, od.shape[2]))
        assert np.all(os_[0, h, rows] == 0) and np.all(np.isneginf(ls[0, h, rows]))
        assert np.all(mass[0, h, rows] == 0)


def test_refresh_agrees_with_the_two_pass_path():
    """The fused outputs against the library's own dense and sparse calls (same
    inputs): two GPU paths that share no accumulation order."""
    (od, ld, os_, ls, R, mass), _, (q, k, v, idx, cnt) = _run(1, 2, 6 * 128 + 9, 128, seed=300)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    o1, l1 = api.sparse_attn_fwd(qd, kd, vd, BLK)
    o2, l2 = api.sparse_attn_fwd(qd, kd, vd, BLK, torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV))
    torch.cuda.synchronize()
    # one bf16 ulp of the output plus the accumulation-order difference
    a1, a2 = to_np(o1), to_np(o2)
    assert np.all(np.abs(od - a1) <= 1e-2 + 2.0 ** -7 * np.abs(a1))
    assert np.all(np.abs(os_ - a2) <= 1e-2 + 2.0 ** -7 * np.abs(a2))
    assert np.max(np.abs(ld - to_np(l1))) <= 1e-3 and np.max(np.abs(ls - to_np(l2))) <= 1e-3


def test_refresh_flags_malformed_lists_and_keeps_dense_output():
    B, H, L, D = 1, 1, 5 * 128, 128
    NB = 5
    q, k, v = (random_bf16((B, H, L, D), 400 + j) for j in range(3))
    idx, cnt = _lists(B, H, NB, 407)
    idx[0, 0, 1, :4] = [3, 1, 4, 99]   # out of order, then out of range
    cnt[0, 0, 1] = 4
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    od, ld, *_ = api.sparse_attn_refresh(q.to(DEV), k.to(DEV), v.to(DEV), BLK, torch.from_numpy(idx).to(DEV),
                                         torch.from_numpy(cnt).to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() & BSA_DEV_BAD_INDEX
    fi, fc = oref.full_lists(B, H, NB)
    from oracle import attention as oatt
    Od, Ld = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), fi, fc, BLK)
    assert_attention_close(to_np(od), to_np(ld), Od, Ld, "dense with a malformed kept list")
