"""Block-sparse (masked) softmax attention -- oracle.

Sources:
* CalibAtt abstract: compute the selected connections densely and skip the
  unselected ones; Fig. 5(b): skip the computation of unset blocks.
* RECAP, section 4.1: the Block Sparse Attention library for the selected
  interactions, FlashAttention-2 for dense refreshes.
* GSRS abstract: exact attention weights inside the FlashAttention pass.

Definition.  For query token r of query block i = r // blk, with kept key
blocks K(i) (from the selection stage) and key tokens c of those blocks
(c < L; the last block may be partial):
    s_c    = (q_r . k_c) / sqrt(D)
    LSE_r  = log( sum_{c} exp(s_c) )                (natural log)
    O_r    = sum_{c} exp(s_c - LSE_r) * v_c
i.e. exact softmax attention restricted to the kept blocks; the speed of the
method comes from skipping blocks, not from approximating inside them.  An
empty kept set (count 0) gives O_r = 0 and LSE_r = -inf.  All arithmetic is
float64; the bf16 inputs are widened exactly.

Pinned by (tests/test_oracle.py): keeping every block equals dense attention
computed by torch.nn.functional.scaled_dot_product_attention in float64 and
by a naive triple loop; the softmax weights of every row sum to 1; one kept
block with constant keys has the closed form LSE = q.k/sqrt(D) + log(n_j)
and O = mean of its values.
"""

import numpy as np


def _kept_tokens(kept_blocks, blk, L):
    cols = [np.arange(j * blk, min(L, (j + 1) * blk)) for j in kept_blocks]
    return np.concatenate(cols) if cols else np.zeros(0, dtype=np.int64)


def attend_rows(q_rows, k, v, token_cols):
    """Exact softmax attention of a set of query rows over given key tokens.

    q_rows [R, D]; k, v [L, D]; token_cols: key token indices.
    Returns (O [R, D] float64, LSE [R] float64).
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    R, D = q_rows.shape
    if token_cols.size == 0:
        return np.zeros((R, D)), np.full(R, -np.inf)
    kc = np.asarray(k, dtype=np.float64)[token_cols]
    vc = np.asarray(v, dtype=np.float64)[token_cols]
    s = q_rows @ kc.T / np.sqrt(D)
    m = s.max(axis=1, keepdims=True)
    lse = m[:, 0] + np.log(np.exp(s - m).sum(axis=1))
    w = np.exp(s - lse[:, None])
    return w @ vc, lse


def masked_attention_block(q, k, v, kept_blocks, blk, b, h, i):
    """O and LSE of query block i of head (b, h).  q, k, v: [B,H,L,D]."""
    L = q.shape[2]
    lo, hi = i * blk, min(L, (i + 1) * blk)
    cols = _kept_tokens(kept_blocks, blk, L)
    return attend_rows(q[b, h, lo:hi], k[b, h], v[b, h], cols)


def masked_attention(q, k, v, kept_idx, kept_cnt, blk, units=None):
    """Masked attention for all (b, h, i) or for a list of units.

    kept_idx [B,H,NB,NB] (first kept_cnt entries valid), kept_cnt [B,H,NB].
    units: optional iterable of (b, h, i); then only those query blocks are
    computed and the rest of O / LSE is left NaN.
    Returns O float64 [B,H,L,D], LSE float64 [B,H,L].
    """
    B, H, L, D = q.shape
    nb = (L + blk - 1) // blk
    O = np.full((B, H, L, D), np.nan)
    LSE = np.full((B, H, L), np.nan)
    if units is None:
        units = [(b, h, i) for b in range(B) for h in range(H) for i in range(nb)]
    for (b, h, i) in units:
        kb = kept_idx[b, h, i, : kept_cnt[b, h, i]]
        o, lse = masked_attention_block(q, k, v, kb, blk, b, h, i)
        lo, hi = i * blk, min(L, (i + 1) * blk)
        O[b, h, lo:hi] = o
        LSE[b, h, lo:hi] = lse
    return O, LSE


def dense_attention(q, k, v):
    """Full softmax attention (every block kept), float64."""
    q = np.asarray(q, dtype=np.float64)
    B, H, L, D = q.shape
    O = np.empty((B, H, L, D))
    LSE = np.empty((B, H, L))
    cols = np.arange(L)
    for b in range(B):
        for h in range(H):
            O[b, h], LSE[b, h] = attend_rows(q[b, h], k[b, h], v[b, h], cols)
    return O, LSE
