"""Shared helpers of the GPU parity tests: tolerances and comparisons.

Tolerances (from the accuracy contract of the path):
  * masks, kept lists, counts, permutations: bit-exact;
  * attention output O (bf16) against the float64 oracle: max-abs <= 2e-2 and
    mean-abs <= 2e-3;
  * LSE: relative error <= 1e-3;
  * block probabilities (float32, computed from float32 pooled means):
    |dP| <= 1e-4 * P + 1e-7.  The float32 logits differ from the float64
    ones by about D * 2^-24 * |qbar||kbar| (~1e-5 here), which moves P by the
    same relative amount; the absolute floor covers underflowing tails;
  * pooled means: |d| <= 1e-5 * (1 + |x|) (float32 sums of <= 128 bf16 values).
"""

import numpy as np
import torch

O_MAX_ABS = 2e-2
O_MEAN_ABS = 2e-3
LSE_REL = 1e-3


def to_np(t):
    return t.detach().float().cpu().numpy() if t.dtype == torch.bfloat16 else t.detach().cpu().numpy()


def assert_attention_close(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    o = np.asarray(o_gpu, dtype=np.float64)
    ref = np.asarray(o_ref, dtype=np.float64)
    finite = np.isfinite(ref)
    assert finite.any(), "no reference rows"
    err = np.abs(o[finite] - ref[finite])
    assert err.max() <= O_MAX_ABS, f"{what}: O max-abs {err.max():.3g}"
    assert err.mean() <= O_MEAN_ABS, f"{what}: O mean-abs {err.mean():.3g}"
    l = np.asarray(lse_gpu, dtype=np.float64)
    lr = np.asarray(lse_ref, dtype=np.float64)
    rows = ~np.isnan(lr)
    inf_rows = rows & np.isneginf(lr)
    assert np.all(np.isneginf(l[inf_rows])), f"{what}: empty rows must give -inf"
    fin = rows & np.isfinite(lr)
    rel = np.abs(l[fin] - lr[fin]) / np.maximum(np.abs(lr[fin]), 1e-30)
    assert rel.max() <= LSE_REL, f"{what}: LSE rel {rel.max():.3g}"
    return err.max(), err.mean(), rel.max() if rel.size else 0.0


def assert_probs_close(p_gpu, p_ref, what=""):
    p = np.asarray(p_gpu, dtype=np.float64)
    r = np.asarray(p_ref, dtype=np.float64)
    bad = np.abs(p - r) > 1e-4 * r + 1e-7
    assert not bad.any(), f"{what}: {bad.sum()} probs out of tolerance, worst {np.abs(p - r).max():.3g}"


def assert_pool_close(x_gpu, x_ref, what=""):
    x = np.asarray(x_gpu, dtype=np.float64)
    r = np.asarray(x_ref, dtype=np.float64)
    assert np.all(np.abs(x - r) <= 1e-5 * (1 + np.abs(r))), f"{what}: pooled means differ"
