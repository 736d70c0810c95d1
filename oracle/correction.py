"""Cached dense refinement and its alpha-scaled correction -- oracle.

Sources:
* RECAP (full text), section 1 and the abstract: a cached dense refinement
  supplies the detail the current sparse estimate leaves unresolved, and
  fresh sparse statistics regulate how strongly the aging refinement is
  applied; section 3.2: the state is kept per layer and attention head;
  sections 3.4 / 4.3: the refinement is renewed only at dense refreshes.

Definitions (readings; the page's own reconstruction formula and its
coarse-tail terms are not printed):
  refinement at a dense-refresh step, from the two bf16 outputs:
      R = bf16( float(O_dense) - float(O_sparse) )
  correction at a later sparse step, per head h with alpha_h in [0, 1]
  supplied by the caller:
      O_corr = O_sparse + alpha_h * float(R)
  (the GPU rounds O_corr to bf16 once; the oracle keeps float64).  In the
  fused form, O_sparse is the float32 accumulator before its own rounding.

Pinned by (tests/test_oracle.py): alpha = 0 returns O_sparse; at the refresh
step alpha = 1 returns O_dense to within one bf16 rounding of R; R is exactly
the bf16 rounding of the difference (compared with torch's bf16 cast).
"""

import numpy as np


def bf16_round(x):
    """Round float64/float32 values to the nearest bfloat16 (ties to even),
    returned as float32.  Written out on the float32 bit pattern."""
    f = np.asarray(x, dtype=np.float32)
    bits = f.view(np.uint32).astype(np.uint64)
    lsb = (bits >> 16) & 1
    rounded = (bits + 0x7FFF + lsb) >> 16 << 16
    nan = np.isnan(f)
    out = rounded.astype(np.uint32).view(np.float32)
    return np.where(nan, np.float32(np.nan), out)


def refresh_refinement(o_dense_bf16, o_sparse_bf16):
    """R = bf16(O_dense - O_sparse); inputs are bf16 values given as float32."""
    d = np.asarray(o_dense_bf16, dtype=np.float32) - np.asarray(o_sparse_bf16, dtype=np.float32)
    return bf16_round(d)


def apply_correction(o_sparse, R, alpha):
    """O_corr[b,h,...] = O_sparse + alpha[h] * R, float64.  Shapes [B,H,L,D]."""
    o = np.asarray(o_sparse, dtype=np.float64)
    a = np.asarray(alpha, dtype=np.float64)[None, :, None, None]
    return o + a * np.asarray(R, dtype=np.float64)
