"""The seeded synthetic inputs and the named workloads (CPU): the generators
are deterministic per seed, the shapes are the latent grids the workloads
name, and the top-p values in the configs are the ones the committed
calibration record found."""

import json
import os

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import configs
from block_sparse_attention_logits_b200.synthetic import FieldParams, drift_, make_qkv, random_bf16, random_probs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_make_qkv_is_deterministic_and_per_head():
    fp = FieldParams(1.0, 8.0, 11.5, 77)
    a = make_qkv(1, 3, (2, 4, 8), 64, fp)
    b = make_qkv(1, 3, (2, 4, 8), 64, fp)
    for n in "qkv":
        assert a[n].dtype == torch.bfloat16 and tuple(a[n].shape) == (1, 3, 64, 64)
        assert torch.equal(a[n], b[n])
    assert not torch.equal(a["q"][:, 0], a["q"][:, 1])   # heads draw their own fields
    c = make_qkv(1, 3, (2, 4, 8), 64, FieldParams(1.0, 8.0, 11.5, 78))
    assert not torch.equal(a["q"], c["q"])


def test_positional_field_makes_nearby_tokens_similar():
    """The inputs stand in for video latents: queries of neighbouring tokens
    correlate more than those of distant tokens (the random-Fourier-feature
    field is a smooth kernel of position)."""
    t = make_qkv(1, 1, (1, 32, 32), 128, FieldParams(0.5, 4.0, 12.0, 5))
    q = t["q"][0, 0].float().numpy()
    qn = q / np.linalg.norm(q, axis=1, keepdims=True)
    near = np.mean([qn[r * 32 + c] @ qn[r * 32 + c + 1] for r in range(32) for c in range(31)])
    far = np.mean([qn[r * 32 + c] @ qn[((r + 16) % 32) * 32 + (c + 16) % 32] for r in range(32) for c in range(32)])
    assert near > far + 0.2


def test_other_generators_are_deterministic():
    assert torch.equal(random_bf16((2, 3, 5), 9), random_bf16((2, 3, 5), 9))
    assert not torch.equal(random_bf16((2, 3, 5), 9), random_bf16((2, 3, 5), 10))
    x, y = random_bf16((1, 2, 8, 8), 1), random_bf16((1, 2, 8, 8), 1)
    drift_(x, 0.05, seed=3, step=2)
    drift_(y, 0.05, seed=3, step=2)
    assert torch.equal(x, y)
    p1, p2 = random_probs(1, 2, 7, 4), random_probs(1, 2, 7, 4)
    assert np.array_equal(np.asarray(p1), np.asarray(p2))


@pytest.mark.parametrize("name,grid,L", [("tiny", (2, 32, 32), 2048), ("wan2.1-1.3b-480p", (21, 30, 52), 32760),
                                         ("wan2.1-14b-720p", (21, 45, 80), 75600),
                                         ("hunyuanvideo-720p-5s", (33, 45, 80), 118800)])
def test_workload_shapes(name, grid, L):
    w = configs.ALL[name]
    assert w.grid == grid and w.L == L and w.NB == -(-L // w.blk)
    assert all(0 < p <= 1 for p in w.p)
    a = w.alpha()
    assert len(a) == w.H and a[0] == 0.0 and a[-1] == 1.0


def test_configs_use_the_calibrated_top_p():
    rec = json.load(open(os.path.join(HERE, "golden", "p_star.json")))
    assert configs.WAN14B_720P.p[0] == rec["wan2.1-14b-720p"]["p"]
    assert abs(rec["wan2.1-14b-720p"]["sparsity_at_p"] - 0.90) <= 0.01
    assert configs.HUNYUAN_720P.p[0] == rec["hunyuanvideo-720p-5s"]["p"]
    assert abs(rec["hunyuanvideo-720p-5s"]["sparsity_at_p"] - 0.95) <= 0.01
    sw = configs.REUSE_SWEEP
    assert (sw.steps, sw.mask_every, sw.refresh_every, sw.drift) == (10, 3, 5, 0.05)
