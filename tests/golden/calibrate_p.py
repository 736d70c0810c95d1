"""Find the top-p threshold that gives a target block sparsity on a workload.

Used once to fix the p of the Wan2.1-14B 720P workload (target 90% +- 1%)
and of the HunyuanVideo 720p workload (target ~95%); the values live in
block_sparse_attention_logits_b200/configs.py and this script records the
evidence in tests/golden/p_star.json.  Only the oracle computes here: block
scores of the seeded inputs (in Hilbert order where the workload uses it)
and the top-p selection; p is bisected on a fine grid.

    python tests/golden/calibrate_p.py [workload ...]
"""

import json
import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

from block_sparse_attention_logits_b200 import configs  # noqa: E402
from block_sparse_attention_logits_b200.synthetic import make_qkv  # noqa: E402
from oracle import hilbert as ohil  # noqa: E402
from oracle import scoring as osco  # noqa: E402
from oracle import topp as otop  # noqa: E402

TARGETS = {"wan2.1-14b-720p": 0.90, "hunyuanvideo-720p-5s": 0.95}


def oracle_probs(w):
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp, with_v=False)
    q = t["q"].float().numpy()
    k = t["k"].float().numpy()
    if w.hilbert:
        perm, _ = ohil.hilbert_perm(*w.grid)
        q = ohil.permute_rows(q, perm)
        k = ohil.permute_rows(k, perm)
    P = np.empty((w.B, w.H, w.NB, w.NB), np.float32)
    for h in range(w.H):  # one head at a time keeps the float64 copies small
        _, _, P[:, h:h + 1] = osco.score_blocks(q[:, h:h + 1], k[:, h:h + 1], w.blk)
    return P


def sparsity(P, p):
    _, _, cnt = otop.select_topp_mask_fast(P, np.full(P.shape[1], p, np.float32))
    return 1.0 - cnt.sum() / (P.shape[0] * P.shape[1] * P.shape[2] ** 2)


def calibrate(name, target):
    w = configs.ALL[name]
    t0 = time.time()
    P = oracle_probs(w)
    lo, hi = 0.5, 0.999  # sparsity falls as p grows
    for _ in range(14):
        mid = round((lo + hi) / 2, 4)
        s = sparsity(P, mid)
        if s > target:
            lo = mid
        else:
            hi = mid
    best = min((lo, hi), key=lambda x: abs(sparsity(P, x) - target))
    best = round(best, 3)
    return {"workload": name, "target_sparsity": target, "p": best,
            "sparsity_at_p": round(float(sparsity(P, best)), 4),
            "seconds": round(time.time() - t0, 1)}


if __name__ == "__main__":
    names = sys.argv[1:] or list(TARGETS)
    out_path = os.path.join(HERE, "p_star.json")
    results = json.load(open(out_path)) if os.path.exists(out_path) else {}
    for n in names:
        r = calibrate(n, TARGETS[n])
        print(json.dumps(r))
        results[n] = r
    json.dump(results, open(out_path, "w"), indent=1)
