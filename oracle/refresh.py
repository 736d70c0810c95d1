"""Single-pass dense refresh -- oracle (test infrastructure only).

A dense refresh renews the cached refinement: at that step the dense output is
computed and R = bf16(O_dense - O_sparse) is stored for the following sparse
steps (RECAP section 1 and section 3.4 with Fig. 3: a dense refresh renews both
cache levels and reveals the error of the refinement it renews).  Computed in
one pass over all key blocks, the same pass also yields the sparse output over
the kept blocks and the exact share of the attention weight that the kept
blocks carry (GSRS abstract: exact attention weights evaluated within the
FlashAttention computation at negligible overhead).

Definitions (plain; nothing here is blocked or fused):
  O_dense, LSE_dense   masked attention with every key block kept
  O_sparse, LSE_sparse masked attention with the given kept blocks
  R                    bf16( bf16(O_dense) - bf16(O_sparse) )
  kept_mass            sum over kept keys of exp(s) / sum over all keys of exp(s)
                       = exp(LSE_sparse - LSE_dense), 0 for an empty kept set

Pinned by (tests/test_oracle.py): keeping every block gives kept_mass = 1,
O_sparse = O_dense and R = 0; with constant keys the mass is the kept token
count over L (closed form); the dense output is the mass-weighted mixture of
the sparse output and the attention over the complement blocks.
"""

import numpy as np

from .attention import masked_attention
from .correction import bf16_round, refresh_refinement


def full_lists(B, H, NB):
    """Kept lists that keep every key block (ascending)."""
    idx = np.tile(np.arange(NB, dtype=np.int32), (B, H, NB, 1))
    cnt = np.full((B, H, NB), NB, dtype=np.int32)
    return idx, cnt


def complement_lists(kept_idx, kept_cnt, NB):
    """Kept lists of the blocks that are NOT kept (ascending)."""
    B, H, NQ, _ = kept_idx.shape
    idx = np.zeros_like(kept_idx)
    cnt = np.zeros_like(kept_cnt)
    for b in range(B):
        for h in range(H):
            for i in range(NQ):
                kept = set(int(j) for j in kept_idx[b, h, i, :kept_cnt[b, h, i]])
                rest = [j for j in range(NB) if j not in kept]
                idx[b, h, i, :len(rest)] = rest
                cnt[b, h, i] = len(rest)
    return idx, cnt


def kept_mass(lse_sparse, lse_dense):
    """exp(LSE_sparse - LSE_dense); 0 where the kept set is empty."""
    ls = np.asarray(lse_sparse, dtype=np.float64)
    ld = np.asarray(lse_dense, dtype=np.float64)
    with np.errstate(invalid="ignore"):
        m = np.exp(ls - ld)
    return np.where(np.isneginf(ls), 0.0, m)


def fused_refresh(q, k, v, kept_idx, kept_cnt, blk, units=None):
    """(O_dense, LSE_dense, O_sparse, LSE_sparse, R, kept_mass), float64 except
    R (bf16 values as float32).  `units` restricts the work as in
    masked_attention (other rows stay NaN)."""
    B, H, L, _ = np.asarray(q).shape
    NB = (L + blk - 1) // blk
    fi, fc = full_lists(B, H, NB)
    Od, Ld = masked_attention(q, k, v, fi, fc, blk, units=units)
    Os, Ls = masked_attention(q, k, v, kept_idx, kept_cnt, blk, units=units)
    R = refresh_refinement(bf16_round(Od), bf16_round(Os))
    return Od, Ld, Os, Ls, R, kept_mass(Ls, Ld)
