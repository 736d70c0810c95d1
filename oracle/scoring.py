"""Block importance scoring -- oracle.

Sources:
* RECAP (full text), section 3.2: coarse estimates of attention are formed
  from block means.
* DFSAttn ("Ride the Wave ..."), abstract: block scoring for block importance
  estimation.
* head-wise adaptive top-p abstract and GSRS abstract: the block scores are
  turned into a distribution over key blocks on which top-p acts.

Definition (one reading; the pages print no formula):
  pooled:  qbar[b,h,i,:] = (1/n_i) * sum_{t in block i} Q[b,h,t,:]
           with n_i the true number of tokens of block i (the last block of a
           sequence may be partial and is divided by its own count; there is
           no padding token).  Same for kbar from K.
  logits:  S[b,h,i,j] = (qbar_i . kbar_j) / sqrt(D)
           (the same 1/sqrt(D) scale as the attention it stands for)
  probs:   P[b,h,i,:] = softmax_j(S[b,h,i,:])

Precision: sums and dot products in float64, results stored float32 (the
dtype the GPU returns).

Pinned by (tests/test_oracle.py): pooling a constant gives the constant;
pooling an arithmetic ramp gives the closed-form block midpoints, including
the partial last block; rows of P sum to 1; a constant K gives P = 1/NB;
P agrees with scipy.special.softmax of independently formed logits.
"""

import numpy as np


def n_blocks(L, blk):
    return (L + blk - 1) // blk


def block_counts(L, blk):
    """True token count of every block: blk, ..., blk, L - (NB-1)*blk."""
    nb = n_blocks(L, blk)
    counts = np.full(nb, blk, dtype=np.int64)
    counts[-1] = L - (nb - 1) * blk
    return counts


def pool_blocks(x, blk):
    """Mean of every block of `blk` consecutive tokens along axis -2.

    x: [B, H, L, D] (any float dtype; bf16 callers pass float32 copies).
    Returns float32 [B, H, NB, D].
    """
    x = np.asarray(x, dtype=np.float64)
    B, H, L, D = x.shape
    nb = n_blocks(L, blk)
    out = np.empty((B, H, nb, D), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * blk, min(L, (i + 1) * blk)
        out[:, :, i, :] = x[:, :, lo:hi, :].sum(axis=2) / float(hi - lo)
    return out.astype(np.float32)


def block_logits(qbar, kbar):
    """S = qbar kbar^T / sqrt(D), float64 [B, H, NB, NB]."""
    qb = np.asarray(qbar, dtype=np.float64)
    kb = np.asarray(kbar, dtype=np.float64)
    D = qb.shape[-1]
    return np.einsum("bhid,bhjd->bhij", qb, kb) / np.sqrt(D)


def row_softmax(s):
    """Max-subtracted softmax along the last axis, float64."""
    s = np.asarray(s, dtype=np.float64)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def score_blocks(q, k, blk):
    """Full scoring stage: (qbar, kbar, P) with P float32 [B, H, NB, NB]."""
    qbar = pool_blocks(q, blk)
    kbar = pool_blocks(k, blk)
    probs = row_softmax(block_logits(qbar, kbar)).astype(np.float32)
    return qbar, kbar, probs
