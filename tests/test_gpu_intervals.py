"""GPU parity of the interval (skip-list) calls against the oracle: runs per
row and their histogram, the width for a merge percentage, encoding at several
widths (rows with more runs are merged) and decoding back to the mask and kept
lists -- all bit-exact; malformed rows are flagged and emptied; attention over
decoded merged lists matches the oracle's masked attention over the merged
blocks; the attention walking the pairs itself equals the attention over the
decoded lists bit for bit, and attends malformed rows as empty."""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api
from block_sparse_attention_logits_b200._lib import BSA_DEV_BAD_INDEX
from block_sparse_attention_logits_b200.synthetic import random_bf16, random_kept_lists
from oracle import attention as oatt
from oracle import intervals as oint

from .gpu_helpers import assert_attention_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def _lists_equal(ki, kc, ki_ref, kc_ref):
    assert np.array_equal(kc, kc_ref)
    valid = np.arange(ki.shape[-1]) < kc[..., None]
    assert np.array_equal(np.where(valid, ki, -1), np.where(valid, ki_ref, -1))


@pytest.mark.parametrize("B,H,NB,seed,density,mean_run", [
    (1, 3, 37, 1, 0.3, 1.5), (2, 2, 100, 2, 0.1, 2.0), (1, 2, 591, 3, 0.1, 3.0), (1, 1, 591, 4, 0.45, 1.0)])
def test_runs_encode_decode_bit_exact(B, H, NB, seed, density, mean_run):
    blk = 128
    L = NB * blk - 17
    idx, cnt = random_kept_lists(B, H, NB, seed, density, mean_run)
    ti, tc = _dev(idx), _dev(cnt)
    n_runs, hist = api.interval_runs(ti, tc, L, blk)
    torch.cuda.synchronize()
    _, _, nr_ref = oint.kept_to_intervals(idx, cnt, oint.max_intervals(NB))
    hist_ref = oint.run_histogram(nr_ref, NB)
    assert np.array_equal(to_np(n_runs), nr_ref)
    assert np.array_equal(to_np(hist).astype(np.int64), hist_ref)
    for q in (0.5, 0.9, 0.95, 0.99, 1.0):
        assert api.interval_width_for_merge(hist, q) == oint.width_for_merge(hist_ref, q)
    widths = {1, 2, 3, oint.width_for_merge(hist_ref, 0.95), oint.width_for_merge(hist_ref, 0.99),
              oint.max_intervals(NB), NB}
    for W in sorted(widths):
        iv, n_int, nr = api.kept_to_intervals(ti, tc, W, L, blk)
        mask, ki, kc = api.intervals_to_kept(iv, n_int, L, blk)
        torch.cuda.synchronize()
        iv_ref, ni_ref, nr2_ref = oint.kept_to_intervals(idx, cnt, W)
        assert np.array_equal(to_np(iv), iv_ref), W
        assert np.array_equal(to_np(n_int), ni_ref), W
        assert np.array_equal(to_np(nr), nr2_ref), W
        m_ref, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_ref, NB)
        assert np.array_equal(to_np(mask), m_ref), W
        _lists_equal(to_np(ki), to_np(kc), ki_ref, kc_ref)
        # a merged row keeps a superset of its blocks
        m_in = np.zeros_like(m_ref)
        for pos in np.ndindex(*cnt.shape):
            m_in[pos + (idx[pos][: cnt[pos]].tolist(),)] = 1
        assert np.all(m_ref >= m_in)


def test_accumulated_histogram_and_decode_without_mask():
    NB, blk = 64, 64
    L = NB * blk
    hist = torch.zeros(oint.max_intervals(NB) + 1, dtype=torch.int32, device=DEV)
    total = np.zeros(oint.max_intervals(NB) + 1, np.int64)
    for seed in (11, 12, 13):   # e.g. three layers sharing one width
        idx, cnt = random_kept_lists(1, 2, NB, seed, 0.25, 2.0, special_rows=False)
        api.interval_runs(_dev(idx), _dev(cnt), L, blk, hist=hist)
        _, _, nr = oint.kept_to_intervals(idx, cnt, oint.max_intervals(NB))
        total += oint.run_histogram(nr, NB)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(hist).astype(np.int64), total)
    W = api.interval_width_for_merge(hist, 0.9)
    assert W == oint.width_for_merge(total, 0.9)
    iv, n_int, _ = api.kept_to_intervals(_dev(idx), _dev(cnt), W, L, blk)
    mask, ki, kc = api.intervals_to_kept(iv, n_int, L, blk, want_mask=False)
    torch.cuda.synchronize()
    assert mask is None
    iv_ref, ni_ref, _ = oint.kept_to_intervals(idx, cnt, W)
    _, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_ref, NB)
    _lists_equal(to_np(ki), to_np(kc), ki_ref, kc_ref)


def test_malformed_rows_are_flagged_and_emptied():
    NB, blk, W = 20, 128, 3
    L = NB * blk
    idx, cnt = random_kept_lists(1, 1, NB, 9, 0.4, 2.0, special_rows=False)
    bad = {0: ([], NB + 1), 1: ([], -1), 2: ([3, 2, 5], 3), 3: ([1, NB], 2), 4: ([4, 4], 2), 5: ([-1, 2], 2)}
    for r, (lst, c) in bad.items():
        idx[0, 0, r] = -1
        idx[0, 0, r, :len(lst)] = lst
        cnt[0, 0, r] = c
    good = idx.copy(), cnt.copy()
    for r in bad:                      # the oracle sees the malformed rows as empty
        good[0][0, 0, r] = -1
        good[1][0, 0, r] = 0
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    n_runs, hist = api.interval_runs(_dev(idx), _dev(cnt), L, blk, status=status)
    torch.cuda.synchronize()
    assert status.item() & BSA_DEV_BAD_INDEX
    _, _, nr_ref = oint.kept_to_intervals(*good, W)
    assert np.array_equal(to_np(n_runs), nr_ref)
    hist_ref = oint.run_histogram(nr_ref, NB)
    hist_ref[0] -= len(bad)            # malformed rows are not counted
    assert np.array_equal(to_np(hist).astype(np.int64), hist_ref)
    status.zero_()
    iv, n_int, _ = api.kept_to_intervals(_dev(idx), _dev(cnt), W, L, blk, status=status)
    torch.cuda.synchronize()
    assert status.item() & BSA_DEV_BAD_INDEX
    iv_ref, ni_ref, _ = oint.kept_to_intervals(*good, W)
    assert np.array_equal(to_np(iv), iv_ref) and np.array_equal(to_np(n_int), ni_ref)
    # malformed interval rows decode as empty
    iv_bad, ni_bad = iv_ref.copy(), ni_ref.copy()
    rows = [r for r in range(NB) if r not in bad and ni_ref[0, 0, r] >= 2][:4]
    assert len(rows) == 4
    ni_bad[0, 0, rows[0]] = W + 1                                          # count above the width
    iv_bad[0, 0, rows[1], 0] = (5, 5)                                      # empty pair
    iv_bad[0, 0, rows[2], 1, 0] = iv_bad[0, 0, rows[2], 0, 1] - 1          # overlaps its predecessor
    iv_bad[0, 0, rows[3], ni_ref[0, 0, rows[3]] - 1, 1] = NB + 1           # ends past the row
    status.zero_()
    mask, ki, kc = api.intervals_to_kept(_dev(iv_bad), _dev(ni_bad), L, blk, status=status)
    torch.cuda.synchronize()
    assert status.item() & BSA_DEV_BAD_INDEX
    ni_exp = ni_ref.copy()
    ni_exp[0, 0, rows] = 0
    m_ref, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_exp, NB)
    assert np.array_equal(to_np(mask), m_ref)
    _lists_equal(to_np(ki), to_np(kc), ki_ref, kc_ref)


def test_attention_over_decoded_merged_lists_matches_oracle():
    B, H, D, blk = 1, 2, 128, 128
    L = 9 * blk + 40
    NB = (L + blk - 1) // blk
    q, k, v = (random_bf16((B, H, L, D), 90 + j) for j in range(3))
    idx, cnt = random_kept_lists(B, H, NB, 93, 0.35, 1.5)
    W = 2
    iv, n_int, _ = api.kept_to_intervals(_dev(idx), _dev(cnt), W, L, blk)
    _, ki, kc = api.intervals_to_kept(iv, n_int, L, blk, want_mask=False)
    o, lse = api.sparse_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), blk, ki, kc)
    torch.cuda.synchronize()
    iv_ref, ni_ref, _ = oint.kept_to_intervals(idx, cnt, W)
    _, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_ref, NB)
    O, LSE = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), ki_ref, kc_ref, blk)
    assert_attention_close(to_np(o), to_np(lse), O, LSE, "attention over merged intervals")


@pytest.mark.parametrize("merge", [False, True], ids=["all-runs", "merged-W2"])
def test_attention_walking_intervals_matches_lists_and_oracle(merge):
    """bsa_sparse_attn_fwd_intervals walks the pairs itself: bit for bit the
    attention over the lists the same pairs decode to, and within tolerance of
    the oracle's masked attention over them.  6 x 40 rows over 148 SMs run
    several items per CTA; random rows include empty and full ones."""
    B, H, D, blk = 1, 6, 128, 128
    L = 39 * blk + 40
    NB = (L + blk - 1) // blk
    q, k, v = (random_bf16((B, H, L, D), 120 + j) for j in range(3))
    R = random_bf16((B, H, L, D), 124, scale=0.05)
    alpha = torch.linspace(0.0, 1.0, H, dtype=torch.float32)
    idx, cnt = random_kept_lists(B, H, NB, 125, 0.3, 2.0)
    W = 2 if merge else oint.max_intervals(NB)
    iv, n_int, _ = api.kept_to_intervals(_dev(idx), _dev(cnt), W, L, blk)
    _, ki, kc = api.intervals_to_kept(iv, n_int, L, blk, want_mask=False)
    qd, kd, vd, Rd, ad = q.to(DEV), k.to(DEV), v.to(DEV), R.to(DEV), alpha.to(DEV)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    o1, l1 = api.sparse_attn_fwd_intervals(qd, kd, vd, blk, iv, n_int, Rd, ad, status=st)
    o2, l2 = api.sparse_attn_fwd(qd, kd, vd, blk, ki, kc, Rd, ad, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(l1, l2)
    iv_ref, ni_ref, _ = oint.kept_to_intervals(idx, cnt, W)
    _, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_ref, NB)
    O, LSE = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), ki_ref, kc_ref, blk)
    O = O + alpha.numpy()[None, :, None, None] * R.float().numpy()
    assert_attention_close(to_np(o1), to_np(l1), O, LSE, "attention walking intervals")


def test_attention_walking_malformed_intervals_is_flagged_and_empty():
    B, H, D, blk = 1, 2, 128, 128
    L = 6 * blk
    NB = L // blk
    q, k, v = (random_bf16((B, H, L, D), 130 + j) for j in range(3))
    idx, cnt = random_kept_lists(B, H, NB, 133, 0.4, 1.5)
    W = oint.max_intervals(NB)
    iv_ref, ni_ref, _ = oint.kept_to_intervals(idx, cnt, W)
    bad = iv_ref.copy()
    nb = ni_ref.copy()
    nb[0, 0, 1] = W + 1                       # more pairs than the width
    bad[0, 1, 2, 0] = [3, 3]                  # an empty pair
    nb[0, 1, 2] = max(nb[0, 1, 2], 1)
    bad[0, 1, 3, 0] = [0, NB + 1]             # past NB
    nb[0, 1, 3] = max(nb[0, 1, 3], 1)
    bad[0, 0, 4, :2] = [[2, 4], [1, 3]]       # out of order
    nb[0, 0, 4] = 2
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd_intervals(q.to(DEV), k.to(DEV), v.to(DEV), blk, _dev(bad), _dev(nb), status=st)
    torch.cuda.synchronize()
    assert st.item() & BSA_DEV_BAD_INDEX
    on, ln = to_np(o), to_np(lse)
    for (h, i) in ((0, 1), (1, 2), (1, 3), (0, 4)):
        rows = slice(i * blk, (i + 1) * blk)
        assert not on[0, h, rows].any() and np.all(np.isneginf(ln[0, h, rows]))
    # the well-formed rows: the oracle over their decoded lists
    good = np.ones((B, H, NB), bool)
    for (h, i) in ((0, 1), (1, 2), (1, 3), (0, 4)):
        good[0, h, i] = False
    _, ki_ref, kc_ref = oint.intervals_to_kept(iv_ref, ni_ref, NB)
    units = [(0, h, i) for h in range(H) for i in range(NB) if good[0, h, i]]
    O, LSE = oatt.masked_attention(q.float().numpy(), k.float().numpy(), v.float().numpy(), ki_ref, kc_ref, blk,
                                   units=units)
    assert_attention_close(on, ln, O, LSE, "well-formed rows")
