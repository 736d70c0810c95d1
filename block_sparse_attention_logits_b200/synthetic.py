"""Seeded synthetic video-token inputs shared by the tests, the bench and the
oracle checks.

This module holds no arithmetic of the attention method itself; it only draws
inputs with the structure of a video DiT's attention: queries and keys carry
a smooth positional field over the (T, Hh, W) latent grid, so attention is
local in space-time and block sparsity is real, plus Gaussian noise.

Recipe (per head h, seeded, float32 then rounded to bf16):
    x_n   = (t/T, y/Hh, x/W)                       normalised grid coordinate
    w ~ N(0, s^2 I_3) (F = D/2 draws), b ~ U(0, 2 pi)
    phi(x) = sqrt(1/F) [cos(w.x + b), sin(w.x + b)]   random Fourier features
             (Rahimi & Recht 2007): phi(x).phi(x') ~ Gaussian kernel of x - x'
    Q = A phi(x) + sigma N(0,1),  K = A phi(x) + sigma N(0,1),  V = N(0,1)
Tokens are flattened row-major, n = (t*Hh + y)*W + x.
"""

from dataclasses import dataclass

import numpy as np
import torch


@dataclass(frozen=True)
class FieldParams:
    sigma: float      # noise std of Q and K
    s: float          # std of the Fourier frequencies (locality scale)
    amp: float        # amplitude A of the positional field
    seed: int


def grid_coords(T, Hh, W):
    t, y, x = np.meshgrid(np.arange(T), np.arange(Hh), np.arange(W), indexing="ij")
    return np.stack([t.ravel() / T, y.ravel() / Hh, x.ravel() / W], axis=1).astype(np.float64)


def _head_field(coords, D, fp, h):
    F = D // 2
    rng = np.random.default_rng(fp.seed + h)
    w = rng.normal(0.0, fp.s, size=(3, F))
    b = rng.uniform(0.0, 2 * np.pi, size=F)
    ang = coords @ w + b
    phi = np.concatenate([np.cos(ang), np.sin(ang)], axis=1) * np.sqrt(1.0 / F)
    return (fp.amp * phi).astype(np.float32)


def make_qkv(B, H, grid, D, fp, with_v=True, out=None, h0=0):
    """Q, K (and V) as bf16 CPU tensors [B, H, L, D] in grid (row-major) order.

    `out` may pass preallocated bf16 tensors (e.g. pinned) to fill in place.
    h0: index of the first head, so that heads h0 .. h0+H-1 of a larger
    workload (one rank's head shard) get exactly that workload's values.
    """
    T, Hh, W = grid
    L = T * Hh * W
    coords = grid_coords(T, Hh, W)
    names = ("q", "k", "v") if with_v else ("q", "k")
    if out is None:
        out = {n: torch.empty((B, H, L, D), dtype=torch.bfloat16) for n in names}
    for hl in range(H):
        h = h0 + hl
        field = _head_field(coords, D, fp, h)
        for b in range(B):
            rng = np.random.default_rng([fp.seed, 7919, b, h])
            for n in names:
                noise = rng.standard_normal((L, D), dtype=np.float32)
                if n == "v":
                    val = noise
                else:
                    val = field + np.float32(fp.sigma) * noise
                out[n][b, hl].copy_(torch.from_numpy(val))
    return out


def drift_(x, std, seed, step):
    """In-place drift of a bf16 tensor by N(0, std) (mask-reuse sweep)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 1000003 + int(step))
    noise = torch.randn(x.shape, generator=g, dtype=torch.float32) * std
    x.copy_((x.float() + noise).to(torch.bfloat16))
    return x


def random_probs(B, H, NB, seed, temperature=1.0, ties=False):
    """Row-stochastic float32 [B,H,NB,NB] test rows for the selection stage.

    Drawn as a softmax of Gaussian logits computed in float64 and rounded to
    float32 (the rows sum to 1 only up to float32 rounding, as real scores
    do).  With ties=True every row repeats a few values so that the
    lowest-index tie rule is exercised.
    """
    rng = np.random.default_rng(seed)
    z = rng.standard_normal((B, H, NB, NB)) * temperature
    if ties:
        z = np.round(z * 2) / 2
    z -= z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32)


def random_bf16(shape, seed, scale=1.0):
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return (torch.randn(shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def random_kept_lists(B, H, NB, seed, density=0.1, mean_run=2.0, special_rows=True):
    """Ascending kept key-block lists for the list-encoding stages: int32
    [B,H,NB,NB] padded with -1 and int32 counts [B,H,NB].

    Each row is an on/off Markov chain along the key blocks: a kept run ends
    with probability 1/mean_run per block and a skipped run ends with
    probability density/(mean_run (1 - density)), so runs of kept blocks have
    mean length mean_run and a `density` share of the blocks is kept in the
    long run (the clustered rows top-p selection gives on video tokens).
    With special_rows, rows (0, 0, 0..3) are: empty, every block, every other
    block (the most runs a row can have) and only the last block.
    """
    assert 0.0 < density < 1.0 and mean_run >= 1.0
    rng = np.random.default_rng(seed)
    p_off = 1.0 / mean_run
    p_on = min(1.0, density * p_off / (1.0 - density))
    u = rng.random((B, H, NB, NB))
    state = rng.random((B, H, NB)) < density
    on = np.zeros((B, H, NB, NB), dtype=bool)
    for j in range(NB):
        state = np.where(state, u[..., j] >= p_off, u[..., j] < p_on)
        on[..., j] = state
    if special_rows and NB >= 4:
        on[0, 0, 0] = False
        on[0, 0, 1] = True
        on[0, 0, 2] = np.arange(NB) % 2 == 0
        on[0, 0, 3] = np.arange(NB) == NB - 1
    cnt = on.sum(axis=-1).astype(np.int32)
    order = np.argsort(~on, axis=-1, kind="stable")
    idx = np.where(np.arange(NB) < cnt[..., None], order, -1).astype(np.int32)
    return idx, cnt
