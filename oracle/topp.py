"""Cumulative top-p block selection -- oracle.

Sources:
* head-wise adaptive top-p abstract: online top-p sparse attention with
  per-head top-p thresholds.
* GSRS abstract: top-p selection for adaptive sparsity control.
* CalibAtt, Fig. 5: threshold the top key blocks per query block; Fig. S8:
  an energy threshold.

Definition, per row (b, h, i) of block probabilities P[b,h,i,:] and the
head's threshold p = p_h in (0, 1]:
  1. clamp: P_j -> 0 if P_j is NaN or <= 0, -> 1 if P_j > 1.
  2. order the key blocks by (P_j descending, j ascending): the lowest index
     wins every tie, so the order is unique.
  3. fixed point: u_j = floor(P_j * 2**40), an exact integer (P_j is a float32
     in [0, 1], so P_j * 2**40 is exact in float64).  With NB <= 4096 the
     row total U = sum_j u_j <= 2**52 is exact in float64 and in uint64.
  4. target: T = ceil(float64(p) * float64(U)), computed in IEEE float64.
  5. k = min{ k >= 1 : sum of the first k ordered u_j >= T }  (">=" -- the kept
     mass reaches p inclusively; mass is measured against the row's own total,
     so float32 rounding of the softmax cannot put the target out of reach).
  6. p == 1 keeps every block, including blocks whose u_j is 0.
Outputs: mask[b,h,i,j] (uint8 0/1), the kept key-block indices of the row in
ascending order (padded to NB with -1 here; the GPU leaves the pad
unspecified) and the count k.

Readings (pages silent): ">=" is inclusive; mass relative to the row total;
the diagonal block is not forced; p is per head; fixed point 2**40 (the
integer prefix sum makes the selection independent of summation order).

Pinned by (tests/test_oracle.py): brute force over all subsets on rows with
NB <= 10 (no smaller subset reaches T, the chosen set is the ordered top-k);
kept mass >= T and dropping the last kept block falls below T; p = 1 keeps
all; equal P with p = 1/2 keeps the ceil(NB/2) lowest indices; hand-worked
rows in tests/golden/topp_cases.json.
"""

import numpy as np

FIXED_POINT_BITS = 40


def clamp_probs(P):
    P = np.asarray(P, dtype=np.float32)
    P = np.where(np.isnan(P) | (P <= 0), np.float32(0), P)
    return np.minimum(P, np.float32(1)).astype(np.float32)


def fixed_point_mass(P):
    """u = floor(P * 2**40) as uint64 (exact for float32 P in [0, 1])."""
    return np.floor(P.astype(np.float64) * float(1 << FIXED_POINT_BITS)).astype(np.uint64)


def select_row(P_row, p):
    """Selection for one row; returns (sorted kept indices, k)."""
    P_row = clamp_probs(P_row)
    nb = P_row.shape[0]
    p = np.float32(p)
    if p == np.float32(1.0):
        return np.arange(nb, dtype=np.int32), nb
    idx = np.arange(nb)
    order = np.lexsort((idx, -P_row.astype(np.float64)))  # P desc, then j asc
    u = fixed_point_mass(P_row)
    total = int(u.sum(dtype=np.uint64))
    T = int(np.ceil(np.float64(p) * np.float64(total)))
    csum = np.cumsum(u[order], dtype=np.uint64)
    k = int(np.argmax(csum >= np.uint64(T))) + 1  # first prefix reaching T
    kept = np.sort(order[:k]).astype(np.int32)
    return kept, k


def select_topp_mask(probs, p_per_head):
    """Top-p selection for all rows.

    probs: float32 [B, H, NB, NB]; p_per_head: float32 [H] in (0, 1].
    Returns mask uint8 [B,H,NB,NB], kept_idx int32 [B,H,NB,NB] (ascending,
    -1 padded), kept_cnt int32 [B,H,NB].
    """
    probs = np.asarray(probs, dtype=np.float32)
    B, H, NB, NB2 = probs.shape
    assert NB == NB2 and NB <= 4096
    p_per_head = np.asarray(p_per_head, dtype=np.float32)
    if np.any(~(p_per_head > 0)) or np.any(p_per_head > 1):
        raise ValueError("p must lie in (0, 1]")
    mask = np.zeros((B, H, NB, NB), dtype=np.uint8)
    kept_idx = np.full((B, H, NB, NB), -1, dtype=np.int32)
    kept_cnt = np.zeros((B, H, NB), dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(NB):
                kept, k = select_row(probs[b, h, i], p_per_head[h])
                mask[b, h, i, kept] = 1
                kept_idx[b, h, i, :k] = kept
                kept_cnt[b, h, i] = k
    return mask, kept_idx, kept_cnt


def select_topp_mask_fast(probs, p_per_head):
    """Same definition as select_topp_mask, vectorised over the rows of a head.

    Used for the large shapes where a Python loop per row is too slow.  Each
    step is the one above, applied along axis -1 of a [rows, NB] array.
    """
    probs = np.asarray(probs, dtype=np.float32)
    B, H, NB, _ = probs.shape
    assert NB <= 4096
    p_per_head = np.asarray(p_per_head, dtype=np.float32)
    if np.any(~(p_per_head > 0)) or np.any(p_per_head > 1):
        raise ValueError("p must lie in (0, 1]")
    mask = np.zeros((B, H, NB, NB), dtype=np.uint8)
    kept_idx = np.full((B, H, NB, NB), -1, dtype=np.int32)
    kept_cnt = np.zeros((B, H, NB), dtype=np.int32)
    idx = np.broadcast_to(np.arange(NB), (NB, NB))
    for b in range(B):
        for h in range(H):
            P = clamp_probs(probs[b, h])
            if np.float32(p_per_head[h]) == np.float32(1.0):
                mask[b, h] = 1
                kept_idx[b, h] = np.arange(NB, dtype=np.int32)[None, :]
                kept_cnt[b, h] = NB
                continue
            order = np.lexsort((idx, -P.astype(np.float64)), axis=-1)
            u = fixed_point_mass(P)
            total = u.sum(axis=-1, dtype=np.uint64)
            T = np.ceil(np.float64(p_per_head[h]) * total.astype(np.float64)).astype(np.uint64)
            csum = np.cumsum(np.take_along_axis(u, order, axis=-1), axis=-1, dtype=np.uint64)
            k = np.argmax(csum >= T[:, None], axis=-1) + 1
            sel = np.arange(NB)[None, :] < k[:, None]
            rows = np.broadcast_to(np.arange(NB)[:, None], (NB, NB))
            mask[b, h][rows[sel], order[sel]] = 1
            kept_cnt[b, h] = k
            # ascending kept indices: the mask's nonzero columns in order
            m = mask[b, h].astype(bool)
            pos = np.cumsum(m, axis=-1) - 1
            r, c = np.nonzero(m)
            kept_idx[b, h][r, pos[r, c]] = c
    return mask, kept_idx, kept_cnt
