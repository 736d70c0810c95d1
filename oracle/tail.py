"""Coarse estimate of the omitted attention tail and its reconstruction with a
cached refinement -- oracle (test infrastructure only).

Source: "RECAP: Reciprocal Sparse Attention and Hierarchical Caching for
Efficient Video Diffusion", section 3.2:
* the omitted (not kept) key blocks of a query start from block means of the
  keys and values (initial estimates of value and normalisation mass);
* the log-mass is refined by key variance through a second-order
  approximation (COBS), the value by a pooled value-key covariance through a
  first-order compensation (PISA, which the related-work section describes as
  block means plus a first-order value term common to all blocks);
* the log of the summed block masses is the coarse log-mass lbar_T, the block
  values weighted by their normalised masses give the coarse output obar_T;
  both are recomputed at every sparse evaluation;
* either tail quantity is written y_t = ybar_t + d_t; the reconstruction uses
  the refinement d_h cached at the last dense refresh, yhat_t = ybar_t + d_h.
Section 1 and the abstract: the sparse estimate over the kept blocks is exact;
the reconstructed tail completes it.

Definitions (readings: the pages print no formulas).  Per head, with a
query q (one token of query block i), a = q / sqrt(D), K(i) the kept blocks
and T(i) the omitted ones; per key block j with n_j tokens (the last block
its own count):
  kbar_j   mean key;  s2_j  per-dimension key variance (population, the
           block's own tokens)                     -- the key variance
  vbar_j   mean value
  C        pooled within-block value-key covariance of the head,
           C[e, d] = (1/L) sum_j sum_{c in j} (v_c - vbar_j)[e] (k_c - kbar_j)[d]
                                                   -- pooled over the blocks
  coarse block log-mass  log n_j + a . kbar_j + 1/2 sum_d a_d^2 s2_j[d]
           (the second-order cumulant expansion of log mean_c exp(a . k_c);
           exact for Gaussian keys with diagonal covariance)
  lbar_T = log sum_{j in T(i)} exp(coarse block log-mass)   (-inf if T(i) empty)
  obar_T = sum_{j in T(i)} w_j vbar_j + C a,   w_j the normalised block masses
           (C a is the first-order value-key compensation: exact for jointly
           Gaussian keys and values; 0 when T(i) is empty)
  exact tail (l_T, o_T): the attention over the omitted blocks' tokens
  refinement at a dense refresh: d_l = l_T - lbar_T, d_o = o_T - obar_T
           (0 where the tail is empty)
  reconstruction: lhat = lbar_T + d_l, ohat = obar_T + d_o, and with the
           exact sparse part (l_S, O_S) over the kept blocks
           LSE = logaddexp(l_S, lhat),
           O   = exp(l_S - LSE) O_S + exp(lhat - LSE) ohat.

Pinned by (tests/test_oracle.py): blocks of constant keys and values make the
coarse tail exact (closed form); for Gaussian keys the coarse block mass is
the Monte Carlo limit exp(a . kbar + 1/2 sum a^2 s2) (the variance term's sign
and factor), and for jointly Gaussian values the coarse output is the limit
vbar + C a (C's orientation and the 1/sqrt(D) scale); a refinement taken at
the same step reconstructs dense attention exactly; keeping every block gives
the sparse output; two planted mistakes.
"""

import numpy as np

from .attention import masked_attention
from .refresh import complement_lists


def block_stats(k, v, blk):
    """Per-block key means and variances, value means, token counts and the
    pooled value-key covariance.  k, v: [B,H,L,D].  Returns (kbar, s2, vbar
    float64 [B,H,NB,D], n int64 [NB], C float64 [B,H,D,D])."""
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, H, L, D = k.shape
    nb = (L + blk - 1) // blk
    kbar = np.empty((B, H, nb, D))
    s2 = np.empty((B, H, nb, D))
    vbar = np.empty((B, H, nb, D))
    n = np.empty(nb, dtype=np.int64)
    C = np.zeros((B, H, D, D))
    for j in range(nb):
        lo, hi = j * blk, min(L, (j + 1) * blk)
        kb, vb = k[:, :, lo:hi], v[:, :, lo:hi]
        n[j] = hi - lo
        kbar[:, :, j] = kb.mean(axis=2)
        vbar[:, :, j] = vb.mean(axis=2)
        dk = kb - kbar[:, :, j, None, :]
        dv = vb - vbar[:, :, j, None, :]
        s2[:, :, j] = (dk ** 2).mean(axis=2)
        C += np.einsum("bhce,bhcd->bhed", dv, dk)
    C /= L
    return kbar, s2, vbar, n, C


def coarse_tail(q, stats, kept_idx, kept_cnt, blk):
    """(lbar_T float64 [B,H,L], obar_T float64 [B,H,L,D]) over the omitted
    blocks of every query token."""
    kbar, s2, vbar, n, C = stats
    q = np.asarray(q, dtype=np.float64)
    B, H, L, D = q.shape
    nb = n.shape[0]
    lbar = np.full((B, H, L), -np.inf)
    obar = np.zeros((B, H, L, D))
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                kept = set(int(j) for j in kept_idx[b, h, i, : kept_cnt[b, h, i]])
                T = [j for j in range(nb) if j not in kept]
                if not T:
                    continue
                lo, hi = i * blk, min(L, (i + 1) * blk)
                a = q[b, h, lo:hi] / np.sqrt(D)
                logm = (np.log(n[T].astype(np.float64))[None, :] + a @ kbar[b, h, T].T
                        + 0.5 * (a * a) @ s2[b, h, T].T)
                mx = logm.max(axis=1, keepdims=True)
                lb = mx[:, 0] + np.log(np.exp(logm - mx).sum(axis=1))
                w = np.exp(logm - lb[:, None])
                lbar[b, h, lo:hi] = lb
                obar[b, h, lo:hi] = w @ vbar[b, h, T] + a @ C[b, h].T
    return lbar, obar


def exact_tail(q, k, v, kept_idx, kept_cnt, blk):
    """(l_T, o_T): the exact attention over the omitted blocks' tokens."""
    L = q.shape[2]
    nb = (L + blk - 1) // blk
    ci, cc = complement_lists(kept_idx, kept_cnt, nb)
    o, l = masked_attention(q, k, v, ci, cc, blk)
    return l, o


def refinement(l_T, o_T, lbar, obar):
    """(d_l, d_o) cached at a dense refresh; 0 where the tail is empty."""
    empty = np.isneginf(lbar)
    with np.errstate(invalid="ignore"):
        d_l = np.where(empty, 0.0, np.asarray(l_T) - lbar)
    d_o = np.where(empty[..., None], 0.0, np.asarray(o_T) - obar)
    return d_l, d_o


def reconstruct(l_S, O_S, lbar, obar, d_l, d_o):
    """(O, LSE) from the exact sparse part and the reconstructed tail."""
    l_S = np.asarray(l_S, dtype=np.float64)
    lhat = lbar + d_l
    ohat = obar + d_o
    lse = np.logaddexp(l_S, lhat)
    with np.errstate(invalid="ignore"):
        ws = np.where(np.isneginf(l_S), 0.0, np.exp(l_S - lse))
        wt = np.where(np.isneginf(lhat), 0.0, np.exp(lhat - lse))
    O = ws[..., None] * np.nan_to_num(np.asarray(O_S, dtype=np.float64)) + wt[..., None] * ohat
    return O, lse
