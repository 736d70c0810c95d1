"""Mask reuse across denoising steps -- oracle (test infrastructure only).

Sources:
* head-wise adaptive top-p abstract: Temporal Mask Reuse skips mask
  prediction when the queries and keys have drifted little since the mask was
  predicted, judged by how far queries and keys have drifted.
* GSRS abstract: blocks selected early keep carrying most of the attention
  weight later, so later top-p searches are restricted to the early candidate
  set.

Definitions (readings: the pages name the quantities but print no formula):

  drift of head (b, h) between the step that predicted the mask (reference
  means qbar_ref, kbar_ref) and the current step (qbar, kbar), from the block
  means that scoring computes anyway:
      drift = max( ||qbar - qbar_ref||_F / ||qbar_ref||_F ,
                   ||kbar - kbar_ref||_F / ||kbar_ref||_F )
  (Frobenius norms over the head's [NB, D] means; 0 / 0 counts as 0 and a
  change from an all-zero reference as +inf).  The caller reuses the mask of
  a head while its drift stays at or below its threshold.

  restricted scoring: the per-query-block softmax of the block logits taken
  over the candidate key blocks only (the blocks outside are not scored and
  get P = 0); a row without candidates is all zeros.

  restricted selection: the top-p rule of topp.select_row applied to the
  candidate blocks of the row, with the target measured against the
  candidates' own mass; p = 1 keeps every candidate; a row without
  candidates keeps nothing.

Pinned by (tests/test_oracle.py): drift of identical means is 0, a uniform
scaling by c gives |c - 1| (closed form), a single perturbed entry gives its
size over the reference norm, and the larger of the Q and K changes wins;
with every block a candidate the restricted scoring and selection equal the
unrestricted ones; restricted rows sum to 1 over the candidates and match
scipy's softmax of the candidate logits; brute force over subsets of the
candidates on small rows; no non-candidate is ever kept.
"""

import numpy as np

from .scoring import block_logits
from .topp import clamp_probs, fixed_point_mass


def block_drift(qbar_ref, kbar_ref, qbar, kbar):
    """drift float64 [B, H] from block means [B, H, NB, D]."""
    def rel(x, ref):
        x = np.asarray(x, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        num = np.sqrt(((x - ref) ** 2).sum(axis=(-2, -1)))
        den = np.sqrt((ref ** 2).sum(axis=(-2, -1)))
        with np.errstate(divide="ignore", invalid="ignore"):
            r = num / den
        return np.where(num == 0, 0.0, r)
    return np.maximum(rel(qbar, qbar_ref), rel(kbar, kbar_ref))


def restricted_probs(qbar, kbar, candidates):
    """Softmax of the block logits over the candidate blocks, float32
    [B, H, NB, NB]; candidates: bool/uint8 [B, H, NB, NB]."""
    s = block_logits(qbar, kbar)
    c = np.asarray(candidates).astype(bool)
    out = np.zeros(s.shape, dtype=np.float64)
    B, H, NQ, _ = s.shape
    for b in range(B):
        for h in range(H):
            for i in range(NQ):
                sel = c[b, h, i]
                if not sel.any():
                    continue
                x = s[b, h, i, sel]
                e = np.exp(x - x.max())
                out[b, h, i, sel] = e / e.sum()
    return out.astype(np.float32)


def select_row_restricted(P_row, p, cand_row):
    """Top-p over the candidates of one row; returns (sorted kept, k)."""
    cand = np.flatnonzero(np.asarray(cand_row).astype(bool))
    if cand.size == 0:
        return np.zeros(0, dtype=np.int32), 0
    P = clamp_probs(P_row)[cand]
    if np.float32(p) == np.float32(1.0):
        return cand.astype(np.int32), int(cand.size)
    order = np.lexsort((cand, -P.astype(np.float64)))  # P desc, then block index asc
    u = fixed_point_mass(P)
    total = int(u.sum(dtype=np.uint64))
    T = int(np.ceil(np.float64(np.float32(p)) * np.float64(total)))
    csum = np.cumsum(u[order], dtype=np.uint64)
    k = int(np.argmax(csum >= np.uint64(T))) + 1
    kept = np.sort(cand[order[:k]]).astype(np.int32)
    return kept, k


def select_topp_mask_restricted(probs, p_per_head, candidates):
    """Restricted selection for all rows: (mask uint8, kept_idx int32 -1
    padded, kept_cnt int32), shapes as topp.select_topp_mask."""
    probs = np.asarray(probs, dtype=np.float32)
    c = np.asarray(candidates)
    B, H, NQ, NB = probs.shape
    mask = np.zeros((B, H, NQ, NB), dtype=np.uint8)
    idx = np.full((B, H, NQ, NB), -1, dtype=np.int32)
    cnt = np.zeros((B, H, NQ), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(NQ):
                kept, k = select_row_restricted(probs[b, h, i], p_per_head[h], c[b, h, i])
                mask[b, h, i, kept] = 1
                idx[b, h, i, :k] = kept
                cnt[b, h, i] = k
    return mask, idx, cnt
