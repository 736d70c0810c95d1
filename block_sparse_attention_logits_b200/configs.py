"""The five named workloads: video-DiT latent grids with seeded synthetic
inputs (see synthetic.py for the recipe).

Shapes are the real latent grids of the models named: 2x32x32 (two small
frames), Wan2.1 480P 21x30x52 (L = 32760), Wan2.1 720P 21x45x80
(L = 75600), HunyuanVideo 720p 5 s 33x45x80 (L = 118800).  The field
parameters (s, A, sigma) are this library's choice, tuned once so that the
selection keeps a realistic, non-trivial fraction of blocks.
"""

from dataclasses import dataclass, field
from typing import Optional, Tuple

from .synthetic import FieldParams


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    D: int
    grid: Tuple[int, int, int]
    blk: int
    fp: FieldParams
    p: Tuple[float, ...]            # top-p values exercised (first one is the main one)
    hilbert: bool = False
    correction: bool = False        # fused O + alpha * R
    steps: int = 1                  # denoising steps (mask-reuse sweep)
    mask_every: int = 1
    refresh_every: int = 0
    drift: float = 0.0
    note: str = ""

    @property
    def L(self):
        T, Hh, W = self.grid
        return T * Hh * W

    @property
    def NB(self):
        return (self.L + self.blk - 1) // self.blk

    def alpha(self):
        """Per-head correction strength alpha_h = h / (H - 1) in [0, 1]."""
        H = self.H
        return [h / (H - 1) if H > 1 else 1.0 for h in range(H)]


# p for the 720P shape was found by bisection of the oracle's selection on the
# seeded inputs so that the global block sparsity is 90% +- 1% (Hunyuan: 95%)
# (tests/golden/calibrate_p.py reproduces it).
P_STAR_720P = 0.886
P_STAR_HUNYUAN = 0.846

TINY = Workload("tiny", 1, 2, 64, (2, 32, 32), 64, FieldParams(0.5, 8.0, 12.0, 1001), (0.9,))
WAN13B_480P = Workload("wan2.1-1.3b-480p", 1, 12, 128, (21, 30, 52), 128,
                       FieldParams(1.0, 8.0, 18.0, 2002), (0.9, 0.97))
WAN14B_720P = Workload("wan2.1-14b-720p", 1, 40, 128, (21, 45, 80), 128,
                       FieldParams(1.0, 8.0, 11.5, 3003), (P_STAR_720P,), hilbert=True)
HUNYUAN_720P = Workload("hunyuanvideo-720p-5s", 1, 24, 128, (33, 45, 80), 128,
                        FieldParams(1.0, 8.0, 18.0, 4004), (P_STAR_HUNYUAN,), correction=True)
REUSE_SWEEP = Workload("mask-reuse-sweep-wan2.1-14b-720p", 1, 40, 128, (21, 45, 80), 128,
                       FieldParams(1.0, 8.0, 11.5, 3003), (P_STAR_720P,), hilbert=True,
                       correction=True, steps=10, mask_every=3, refresh_every=5, drift=0.05)

ALL = {w.name: w for w in (TINY, WAN13B_480P, WAN14B_720P, HUNYUAN_720P, REUSE_SWEEP)}
