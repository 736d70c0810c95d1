"""GPU parity of the gathering attention (bsa_sparse_attn_fwd_gather) and of
copy-free gathering scoring, against the oracle.

The attention runs over the tokens in Hilbert order (oracle.hilbert) while
q, k, v, R, o and lse stay in grid order; the kernel loads its tiles with
4-row TMA gathers.  Checked:
  * against oracle.attention on the reordered inputs, written back to grid
    order (oracle.hilbert.permute_rows inverse), with and without the fused
    correction (R read at each token's grid row), random kept lists with empty
    and full rows, dense, and a ragged last block;
  * bit for bit against the reordered-copies path of this library (the same
    arithmetic in the same order), so any gather fault shows as a difference;
  * a row map with an entry outside [0, L): zeros read, the output row
    skipped and BSA_DEV_BAD_INDEX raised;
  * block scores from score_blocks_gather without copies, against the oracle.
"""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import _lib, api
from block_sparse_attention_logits_b200.synthetic import random_bf16, random_kept_lists
from oracle import attention as oatt
from oracle import correction as ocor
from oracle import hilbert as ohil
from oracle import scoring as osco

from .gpu_helpers import assert_attention_close, assert_probs_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
GRID = (3, 9, 25)  # L = 675: 6 blocks, the last one 35 tokens


def _inputs(H, seed):
    L = GRID[0] * GRID[1] * GRID[2]
    q = random_bf16((1, H, L, 128), seed, scale=2.0)
    k = random_bf16((1, H, L, 128), seed + 1, scale=2.0)
    v = random_bf16((1, H, L, 128), seed + 2, scale=1.0)
    return q, k, v, L


@pytest.mark.parametrize("mode", ["sparse", "correction", "dense"])
def test_gather_attention_matches_oracle(mode):
    H = 3
    q, k, v, L = _inputs(H, 60)
    nb = (L + 127) // 128
    perm_o, _ = ohil.hilbert_perm(*GRID)
    perm = torch.from_numpy(perm_o.astype(np.int32)).to(DEV)
    idx, cnt = random_kept_lists(1, H, nb, 63, 0.4, 2.0)
    kept = (None, None) if mode == "dense" else (torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV))
    R = alpha = None
    if mode == "correction":
        R = random_bf16(q.shape, 64, scale=0.05)
        alpha = torch.tensor([0.0, 0.5, 1.0], dtype=torch.float32)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), 128, *kept,
                                 None if R is None else R.to(DEV), None if alpha is None else alpha.to(DEV),
                                 status=status, in_rows=perm)
    torch.cuda.synchronize()
    assert status.item() == 0
    qh, kh, vh = (ohil.permute_rows(x.float().numpy(), perm_o) for x in (q, k, v))
    if mode == "dense":
        O, LSE = oatt.dense_attention(qh, kh, vh)
    else:
        O, LSE = oatt.masked_attention(qh, kh, vh, idx, cnt, 128)
    if R is not None:
        O = ocor.apply_correction(O, ohil.permute_rows(R.float().numpy(), perm_o), alpha.numpy())
    O = ohil.permute_rows(O, perm_o, inverse=True)
    LSE = ohil.permute_rows(LSE[..., None], perm_o, inverse=True)[..., 0]
    assert_attention_close(to_np(o), to_np(lse), O, LSE, f"gather {mode}")


def test_gather_attention_bit_identical_to_reordered_copies():
    """480P-like item count (2 heads x 255 blocks, > 3 items per CTA): the
    gathering call and the reordered-copies call give the same bits."""
    grid = (21, 30, 52)
    L = grid[0] * grid[1] * grid[2]
    H = 2
    q = random_bf16((1, H, L, 128), 70, scale=2.0).to(DEV)
    k = random_bf16((1, H, L, 128), 71, scale=2.0).to(DEV)
    v = random_bf16((1, H, L, 128), 72, scale=1.0).to(DEV)
    R = random_bf16((1, H, L, 128), 73, scale=0.05).to(DEV)
    alpha = torch.tensor([0.25, 0.75], dtype=torch.float32, device=DEV)
    nb = (L + 127) // 128
    idx, cnt = (torch.from_numpy(a).to(DEV) for a in random_kept_lists(1, H, nb, 74, 0.1, 3.0))
    perm = api.reorder_tokens(*grid, device=DEV)[0]
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    o1, l1 = api.sparse_attn_fwd(q, k, v, 128, idx, cnt, R, alpha, status=st, in_rows=perm)
    qh, kh, vh, Rh = (api.permute_tokens(x, perm) for x in (q, k, v, R))
    o2, l2 = api.sparse_attn_fwd(qh, kh, vh, 128, idx, cnt, Rh, alpha, status=st, out_rows=perm)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(o1, o2)
    assert torch.equal(torch.nan_to_num(l1, neginf=-1e30), torch.nan_to_num(l2, neginf=-1e30))


def test_gather_attention_bad_row_index_is_flagged():
    H = 1
    q, k, v, L = _inputs(H, 80)
    perm_o, _ = ohil.hilbert_perm(*GRID)
    bad = perm_o.astype(np.int32).copy()
    bad[5] = L + 3  # outside [0, L)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    o = torch.full((1, H, L, 128), 7.0, dtype=torch.bfloat16, device=DEV)
    lse = torch.full((1, H, L), 7.0, dtype=torch.float32, device=DEV)
    api.sparse_attn_fwd(q.to(DEV), k.to(DEV), v.to(DEV), 128, o=o, lse=lse, status=st,
                        in_rows=torch.from_numpy(bad).to(DEV))
    torch.cuda.synchronize()
    assert st.item() & _lib.BSA_DEV_BAD_INDEX
    lse_h = to_np(lse)[0, 0]
    assert np.isfinite(lse_h).all()
    # grid row perm[5] receives no output (nothing maps to it); every other row does
    untouched = np.flatnonzero(lse_h == 7.0)
    assert untouched.tolist() == [int(perm_o[5])]


def test_copy_free_gather_scoring_matches_oracle():
    H = 2
    q, k, _, L = _inputs(H, 90)
    perm_o, _ = ohil.hilbert_perm(*GRID)
    perm = torch.from_numpy(perm_o.astype(np.int32)).to(DEV)
    qo, ko, qp, kp, P = api.score_blocks_gather(q.to(DEV), k.to(DEV), perm, 128, copies=False)
    torch.cuda.synchronize()
    assert qo is None and ko is None
    qh, kh = (ohil.permute_rows(x.float().numpy(), perm_o) for x in (q, k))
    _, _, Po = osco.score_blocks(qh, kh, 128)
    assert_probs_close(to_np(P), Po, "copy-free gather scoring")
