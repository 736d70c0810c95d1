"""The Python binding on CPU: it only marshals, so every argument it cannot
hand to the library -- a host tensor, a wrong dtype, shape or layout, a
status word that is not one device int32 -- is refused with a Python error
before the C call; arguments it accepts reach the library, which without a GPU
refuses them with a status (there is no CPU fallback).  The host-only width
function runs here end to end."""

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import _lib, api
from oracle import intervals as oint

B, H, L, D, BLK = 1, 2, 300, 64, 64
NB = (L + BLK - 1) // BLK


def bf(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def f32(*shape):
    return torch.zeros(shape, dtype=torch.float32)


def i32(*shape):
    return torch.zeros(shape, dtype=torch.int32)


CALLS = {
    "score_blocks": lambda: api.score_blocks(bf(B, H, L, D), bf(B, H, L, D), BLK),
    "score_blocks_gather": lambda: api.score_blocks_gather(bf(B, H, L, D), bf(B, H, L, D), i32(L), BLK),
    "block_drift": lambda: api.block_drift(*(f32(B, H, NB, D) for _ in range(4)), L, BLK),
    "select_topp_mask": lambda: api.select_topp_mask(f32(B, H, NB, NB), 0.9, L, BLK, D),
    "permute_tokens": lambda: api.permute_tokens(bf(B, H, L, D), i32(L)),
    "sparse_attn_fwd": lambda: api.sparse_attn_fwd(bf(B, H, L, D), bf(B, H, L, D), bf(B, H, L, D), BLK),
    "sparse_attn_refresh": lambda: api.sparse_attn_refresh(bf(B, H, L, D), bf(B, H, L, D), bf(B, H, L, D), BLK,
                                                           i32(B, H, NB, NB), i32(B, H, NB)),
    "refresh_refinement": lambda: api.refresh_refinement(bf(B, H, L, D), bf(B, H, L, D)),
    "apply_correction": lambda: api.apply_correction(bf(B, H, L, D), bf(B, H, L, D), f32(H)),
    "interval_runs": lambda: api.interval_runs(i32(B, H, NB, NB), i32(B, H, NB), L, BLK, D),
    "kept_to_intervals": lambda: api.kept_to_intervals(i32(B, H, NB, NB), i32(B, H, NB), 2, L, BLK, D),
    "intervals_to_kept": lambda: api.intervals_to_kept(i32(B, H, NB, 2, 2), i32(B, H, NB), L, BLK, D),
}


@pytest.mark.parametrize("name", sorted(CALLS))
def test_host_tensors_are_refused_before_the_library(name):
    with pytest.raises(ValueError, match="CUDA"):
        CALLS[name]()


@pytest.fixture
def host_as_device(monkeypatch):
    """Let host tensors pass the binding's device check, so that the checks
    behind it can be reached on a machine without a GPU; the library itself
    still refuses to run without one."""
    orig = api._need

    def need(t, dtype, shape, name):
        if isinstance(t, torch.Tensor) and not t.is_cuda:
            if t.dtype != dtype:
                raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
            if tuple(t.shape) != tuple(shape):
                raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
            if not t.is_contiguous():
                raise ValueError(f"{name} must be contiguous")
            return t
        return orig(t, dtype, shape, name)
    monkeypatch.setattr(api, "_need", need)
    monkeypatch.setattr(api, "_stream", lambda: None)


def test_wrong_dtype_shape_layout_and_status_are_refused(host_as_device):
    q = bf(B, H, L, D)
    with pytest.raises(TypeError):
        api.score_blocks(q.float(), q, BLK)
    with pytest.raises(ValueError):
        api.score_blocks(q, bf(B, H, L + 1, D), BLK)
    with pytest.raises(ValueError):
        api.permute_tokens(bf(B, H, D, L).transpose(2, 3), i32(L))
    with pytest.raises(TypeError):
        api.sparse_attn_fwd(q, q, q, BLK, status=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError):
        api.sparse_attn_fwd(q, q, q, BLK, status=i32(2))
    with pytest.raises(ValueError):
        api.sparse_attn_refresh(q, q, q, BLK, i32(B, H, NB, NB), i32(B, H, NB), status=i32(1, 1))
    with pytest.raises(TypeError):
        api.refresh_refinement(q, q, out=f32(B, H, L, D))
    with pytest.raises(TypeError):
        api.apply_correction(q, q, f32(H), out=f32(B, H, L, D))
    with pytest.raises(TypeError):
        api.sparse_attn_fwd(q, q, q, BLK, kept_idx=i32(B, H, NB, NB))      # kept_cnt missing
    with pytest.raises(TypeError):
        api.reorder_tokens(2, 3, 5, device="cpu", perm=torch.zeros(30, dtype=torch.int64))
    with pytest.raises(ValueError):
        api.select_topp_mask(f32(B, H, NB, NB), [0.9], L, BLK, D)            # one p per head


def test_accepted_arguments_reach_the_library_which_needs_a_gpu(host_as_device):
    if torch.cuda.is_available():
        pytest.skip("checks the behaviour without a GPU")
    q = bf(B, H, L, D)
    with pytest.raises(_lib.BsaError) as e:
        api.apply_correction(q, q, f32(H))
    assert e.value.code == _lib.BSA_ENODEV
    with pytest.raises(_lib.BsaError) as e:
        api.sparse_attn_fwd(q, q, q, BLK, status=i32(1))
    assert e.value.code == _lib.BSA_ENODEV


def test_interval_width_for_merge_through_the_binding():
    rng = np.random.default_rng(3)
    for _ in range(50):
        hist = rng.integers(0, 30, size=int(rng.integers(2, 20)))
        for q in (0.5, 0.95, 1.0):
            assert api.interval_width_for_merge(torch.from_numpy(hist).to(torch.int32), q) == \
                oint.width_for_merge(hist, q)
            assert api.interval_width_for_merge(hist.tolist(), q) == oint.width_for_merge(hist, q)
    with pytest.raises(_lib.BsaError):
        api.interval_width_for_merge([1, 2], 1.5)
