"""The C-ABI library loads, exports every symbol include/bsa.h declares, and
rejects bad arguments on the host before touching the device (CPU only)."""

import ctypes
import os
import re

import pytest

from block_sparse_attention_logits_b200 import _lib
from block_sparse_attention_logits_b200._lib import Shape

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "bsa.h")


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(_lib.LIB_PATH):
        from block_sparse_attention_logits_b200 import build
        build.build()
    return _lib.load()


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("bsa_score_blocks", "bsa_select_topp_mask", "bsa_reorder_tokens", "bsa_permute_tokens",
                 "bsa_sparse_attn_fwd", "bsa_sparse_attn_refresh", "bsa_refresh_refinement", "bsa_apply_correction",
                 "bsa_strerror"):
        assert name in syms
    assert set(syms) == set(_lib.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {_lib.LIB_PATH}").read()
    exported = set(re.findall(r" T (bsa_\w+)", out))
    assert exported == set(declared_symbols())


def test_strerror_and_version(lib):
    assert lib.bsa_version() >= 10000
    for code in range(6):
        assert len(lib.bsa_strerror(code)) > 0
    assert lib.bsa_strerror(99) == b"unknown status"


NULL = ctypes.c_void_p(0)
FAKE = ctypes.c_void_p(1 << 20)     # aligned, never dereferenced on the host
MISALIGNED = ctypes.c_void_p((1 << 20) + 4)


def test_score_blocks_validation(lib):
    good = Shape(1, 2, 256, 128, 128)
    assert lib.bsa_score_blocks(good, NULL, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_score_blocks(good, MISALIGNED, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    for bad in (Shape(1, 2, 256, 96, 128), Shape(1, 2, 256, 128, 32), Shape(0, 2, 256, 128, 128),
                Shape(1, 2, 0, 128, 128), Shape(1, 1, 4097 * 64, 64, 64)):
        assert lib.bsa_score_blocks(bad, FAKE, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_ESHAPE
    # valid arguments, no GPU in this process: the device check answers
    import torch
    if not torch.cuda.is_available():
        assert lib.bsa_score_blocks(good, FAKE, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_ENODEV


def test_select_validation(lib):
    good = Shape(1, 3, 256, 128, 128)
    p_ok = (ctypes.c_float * 3)(0.9, 0.5, 1.0)
    for bad_p in ((0.0, 0.5, 0.5), (0.5, 1.5, 0.5), (0.5, float("nan"), 0.5), (-1.0, 0.5, 0.5)):
        arr = (ctypes.c_float * 3)(*bad_p)
        assert lib.bsa_select_topp_mask(good, FAKE, arr, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_select_topp_mask(good, FAKE, None, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_select_topp_mask(good, FAKE, p_ok, NULL, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    many = Shape(1, 513, 256, 128, 128)
    arr = (ctypes.c_float * 513)(*([0.9] * 513))
    assert lib.bsa_select_topp_mask(many, FAKE, arr, FAKE, FAKE, FAKE, NULL) == _lib.BSA_ESHAPE


def test_reorder_validation(lib):
    assert lib.bsa_reorder_workspace_bytes(21, 45, 80) == 512 * 4      # 128^3 cells / 4096 per chunk
    assert lib.bsa_reorder_workspace_bytes(2, 32, 32) == 8 * 4         # 32^3 / 4096
    assert lib.bsa_reorder_workspace_bytes(257, 1, 1) == 0
    assert lib.bsa_reorder_workspace_bytes(0, 4, 4) == 0
    assert lib.bsa_reorder_tokens(257, 2, 2, FAKE, FAKE, FAKE, 1 << 20, NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_reorder_tokens(21, 45, 80, FAKE, FAKE, FAKE, 100, NULL) == _lib.BSA_EWORKSPACE
    assert lib.bsa_reorder_tokens(21, 45, 80, FAKE, FAKE, NULL, 4096, NULL) == _lib.BSA_EWORKSPACE
    assert lib.bsa_reorder_tokens(21, 45, 80, NULL, FAKE, FAKE, 4096, NULL) == _lib.BSA_EINVAL


def test_attention_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    args = [FAKE] * 3
    # exactly one of kept_idx / kept_cnt
    assert lib.bsa_sparse_attn_fwd(s, *args, FAKE, NULL, NULL, NULL, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    # R without alpha
    assert lib.bsa_sparse_attn_fwd(s, *args, NULL, NULL, FAKE, NULL, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd(s, *args, NULL, NULL, NULL, NULL, NULL, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd(Shape(1, 2, 1000, 80, 128), *args, NULL, NULL, NULL, NULL, FAKE, FAKE,
                                   NULL, NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_fwd(Shape(70000, 1, 10, 64, 64), *args, NULL, NULL, NULL, NULL, FAKE, FAKE,
                                   NULL, NULL) == _lib.BSA_ESHAPE


def test_reuse_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    ph = (ctypes.c_float * 2)(0.9, 0.9)
    # restricted calls require the candidate mask
    assert lib.bsa_score_blocks_restricted(s, FAKE, FAKE, NULL, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_select_topp_mask_restricted(s, FAKE, ph, NULL, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_select_topp_mask_restricted(s, FAKE, (ctypes.c_float * 2)(0.9, 1.5), FAKE, FAKE, FAKE, FAKE,
                                               NULL) == _lib.BSA_EINVAL
    assert lib.bsa_score_blocks_restricted(Shape(1, 2, 1000, 96, 128), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE,
                                           NULL) == _lib.BSA_ESHAPE
    for miss in range(5):
        args = [FAKE] * 5
        args[miss] = NULL
        assert lib.bsa_block_drift(s, *args, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_block_drift(Shape(1, 2, 1000, 128, 96), FAKE, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_ESHAPE


def test_refresh_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    qkv = (FAKE, FAKE, FAKE)
    ok_out = (FAKE, FAKE, FAKE, FAKE)  # o_dense, lse_dense, o_sparse, lse_sparse
    # the kept lists are required
    assert lib.bsa_sparse_attn_refresh(s, *qkv, NULL, FAKE, *ok_out, NULL, NULL, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_refresh(s, *qkv, FAKE, NULL, *ok_out, NULL, NULL, NULL, NULL) == _lib.BSA_EINVAL
    # every output but R and kept_mass is required
    for miss in range(4):
        outs = list(ok_out)
        outs[miss] = NULL
        assert lib.bsa_sparse_attn_refresh(s, *qkv, FAKE, FAKE, *outs, NULL, NULL, NULL, NULL) == _lib.BSA_EINVAL
    # misaligned optional output
    assert lib.bsa_sparse_attn_refresh(s, *qkv, FAKE, FAKE, *ok_out, ctypes.c_void_p(FAKE.value + 2), NULL, NULL,
                                       NULL) == _lib.BSA_EINVAL
    # only 128-token blocks
    assert lib.bsa_sparse_attn_refresh(Shape(1, 2, 1000, 128, 64), *qkv, FAKE, FAKE, *ok_out, NULL, NULL, NULL,
                                       NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_refresh(Shape(1, 2, 1000, 96, 128), *qkv, FAKE, FAKE, *ok_out, NULL, NULL, NULL,
                                       NULL) == _lib.BSA_ESHAPE


def test_scatter_validation(lib):
    args = [FAKE] * 3
    ok = (NULL, NULL, NULL, NULL)  # kept_idx, kept_cnt, R, alpha
    # the row map needs 128-token blocks and 16-byte alignment
    assert lib.bsa_sparse_attn_fwd_scatter(Shape(1, 2, 1000, 128, 64), *args, *ok, FAKE, FAKE, FAKE, NULL,
                                           NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_fwd_scatter(Shape(1, 2, 1000, 128, 128), *args, *ok,
                                           ctypes.c_void_p(FAKE.value + 4), FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL


def test_gather_attention_validation(lib):
    qkv = [FAKE, ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20)]
    ok = (NULL, NULL, NULL, NULL)  # kept_idx, kept_cnt, R, alpha
    out = (ctypes.c_void_p(4 << 20), ctypes.c_void_p(5 << 20), NULL, NULL)  # o, lse, status, stream
    rows = ctypes.c_void_p(6 << 20)
    # rows required and 16-byte aligned; 128-token blocks and D = 128 only
    assert lib.bsa_sparse_attn_fwd_gather(Shape(1, 2, 1000, 128, 128), *qkv, NULL, *ok, *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_gather(Shape(1, 2, 1000, 128, 128), *qkv, ctypes.c_void_p(rows.value + 4), *ok,
                                          *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_gather(Shape(1, 2, 1000, 128, 64), *qkv, rows, *ok, *out) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_fwd_gather(Shape(1, 2, 1000, 64, 128), *qkv, rows, *ok, *out) == _lib.BSA_ESHAPE
    # row coordinates are int32: B*H*L must stay below 2^31
    assert lib.bsa_sparse_attn_fwd_gather(Shape(64, 64, 1 << 19, 128, 128), *qkv, rows, *ok,
                                          *out) == _lib.BSA_ESHAPE
    # kept_idx without kept_cnt
    assert lib.bsa_sparse_attn_fwd_gather(Shape(1, 2, 1000, 128, 128), *qkv, rows, FAKE, NULL, NULL, NULL,
                                          *out) == _lib.BSA_EINVAL


def test_gather_scoring_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    other = ctypes.c_void_p(2 << 20)
    third = ctypes.c_void_p(3 << 20)
    # perm required; outputs may not alias the inputs or each other
    assert lib.bsa_score_blocks_gather(s, FAKE, other, NULL, third, ctypes.c_void_p(4 << 20), FAKE, FAKE, FAKE,
                                       NULL) == _lib.BSA_EINVAL
    assert lib.bsa_score_blocks_gather(s, FAKE, other, FAKE, FAKE, third, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_score_blocks_gather(s, FAKE, other, FAKE, third, third, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    # no copies: both outputs NULL, never one
    assert lib.bsa_score_blocks_gather(s, FAKE, other, FAKE, third, NULL, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_score_blocks_gather(s, FAKE, other, FAKE, NULL, third, FAKE, FAKE, FAKE, NULL) == _lib.BSA_EINVAL


def test_elementwise_validation(lib):
    assert lib.bsa_refresh_refinement(Shape(1, 1, 10, 12, 0), FAKE, FAKE, FAKE, NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_refresh_refinement(Shape(1, 1, 10, 16, 0), FAKE, NULL, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_apply_correction(Shape(1, 1, 10, 16, 0), FAKE, FAKE, NULL, FAKE, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_permute_tokens(Shape(1, 1, 10, 16, 0), FAKE, FAKE, FAKE, 0, NULL) == _lib.BSA_EINVAL  # x == y


def test_interval_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)   # NB = 8
    # runs: kept lists and n_runs required; hist optional
    assert lib.bsa_interval_runs(s, NULL, FAKE, FAKE, NULL, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_interval_runs(s, FAKE, FAKE, NULL, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_interval_runs(s, FAKE, FAKE, FAKE, MISALIGNED, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_interval_runs(Shape(1, 2, 1000, 128, 96), FAKE, FAKE, FAKE, NULL, NULL, NULL) == _lib.BSA_ESHAPE
    # encode / decode: width in [1, NB]
    for W in (0, -1, 9):
        assert lib.bsa_kept_to_intervals(s, FAKE, FAKE, W, FAKE, FAKE, NULL, NULL, NULL) == _lib.BSA_EINVAL
        assert lib.bsa_intervals_to_kept(s, FAKE, FAKE, W, NULL, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_kept_to_intervals(s, FAKE, FAKE, 3, NULL, FAKE, NULL, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_kept_to_intervals(s, FAKE, FAKE, 3, FAKE, FAKE, MISALIGNED, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_intervals_to_kept(s, FAKE, NULL, 3, NULL, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_intervals_to_kept(s, FAKE, FAKE, 3, MISALIGNED, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_intervals_to_kept(Shape(0, 2, 1000, 128, 128), FAKE, FAKE, 3, NULL, FAKE, FAKE, NULL,
                                     NULL) == _lib.BSA_ESHAPE


def _width(lib, hist, q):
    arr = (ctypes.c_int32 * len(hist))(*hist)
    w = ctypes.c_int(-7)
    code = lib.bsa_interval_width_for_merge(arr, len(hist), q, ctypes.byref(w))
    return code, w.value


def test_interval_width_host_function_matches_oracle(lib):
    """bsa_interval_width_for_merge is host code of the library: it runs here,
    and agrees with the oracle on random and edge-case histograms."""
    import numpy as np
    from oracle import intervals as oint
    rng = np.random.default_rng(7)
    for _ in range(300):
        nb = int(rng.integers(2, 40))
        hist = rng.integers(0, 50, size=nb) * (rng.random(nb) < 0.6)
        for q in (1e-9, 0.3, 0.5, 0.9, 0.95, 0.99, 1.0, float(rng.random())):
            code, w = _width(lib, hist.tolist(), q)
            assert code == _lib.BSA_OK and w == oint.width_for_merge(hist, q), (hist, q)
    assert _width(lib, [0, 0, 0], 1.0) == (_lib.BSA_OK, 1)
    assert _width(lib, [5], 1.0)[0] == _lib.BSA_EINVAL           # fewer than 2 bins
    assert _width(lib, [1, -1, 3], 1.0)[0] == _lib.BSA_EINVAL      # negative count
    for q in (0.0, -0.5, 1.5, float("nan")):
        assert _width(lib, [1, 2, 3], q)[0] == _lib.BSA_EINVAL
    w = ctypes.c_int(0)
    assert lib.bsa_interval_width_for_merge(None, 3, 1.0, ctypes.byref(w)) == _lib.BSA_EINVAL


def test_status_and_alpha_need_word_alignment(lib):
    s = Shape(1, 2, 1000, 128, 128)
    odd = ctypes.c_void_p((1 << 20) + 2)      # not 4-byte aligned
    qkv = (FAKE, FAKE, FAKE)
    # status of the attention calls
    assert lib.bsa_sparse_attn_fwd(s, *qkv, NULL, NULL, NULL, NULL, FAKE, FAKE, odd, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_scatter(s, *qkv, NULL, NULL, NULL, NULL, NULL, FAKE, FAKE, odd,
                                           NULL) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_refresh(s, *qkv, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, NULL, odd,
                                       NULL) == _lib.BSA_EINVAL
    # alpha of the fused and the standalone correction
    assert lib.bsa_sparse_attn_fwd(s, *qkv, NULL, NULL, FAKE, odd, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_apply_correction(Shape(1, 2, 10, 16, 0), FAKE, FAKE, odd, FAKE, NULL) == _lib.BSA_EINVAL
    # status of the interval calls
    assert lib.bsa_interval_runs(s, FAKE, FAKE, FAKE, NULL, odd, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_kept_to_intervals(s, FAKE, FAKE, 3, FAKE, FAKE, NULL, odd, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_intervals_to_kept(s, FAKE, FAKE, 3, NULL, FAKE, FAKE, odd, NULL) == _lib.BSA_EINVAL


def test_wait_selftest_validation(lib):
    assert lib.bsa_wait_selftest(NULL, 1000, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_wait_selftest(ctypes.c_void_p((1 << 20) + 2), 1000, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_wait_selftest(FAKE, 0, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_wait_selftest(FAKE, 3_000_000_000, NULL) == _lib.BSA_EINVAL


def test_tail_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    need = lib.bsa_tail_workspace_bytes(s)
    assert need > 0 and lib.bsa_tail_workspace_bytes(Shape(1, 2, 1000, 64, 128)) == 0
    # statistics: every output required, D = 128, the workspace big enough
    assert lib.bsa_tail_stats(s, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, FAKE, need, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_tail_stats(Shape(1, 2, 1000, 64, 128), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need, NULL,
                              NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_tail_stats(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, need - 1, NULL,
                              NULL) == _lib.BSA_EWORKSPACE
    assert lib.bsa_tail_stats(s, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, need, NULL, NULL) == _lib.BSA_EWORKSPACE
    # the tail: 128-token blocks, D = 128, word-aligned status
    assert lib.bsa_coarse_tail(Shape(1, 2, 1000, 128, 64), FAKE, FAKE, FAKE, need, FAKE, FAKE, NULL,
                               NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_coarse_tail(s, FAKE, FAKE, FAKE, need - 1, FAKE, FAKE, NULL, NULL) == _lib.BSA_EWORKSPACE
    assert lib.bsa_coarse_tail(s, FAKE, NULL, FAKE, need, FAKE, FAKE, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_coarse_tail(s, FAKE, FAKE, FAKE, need, FAKE, FAKE, ctypes.c_void_p((1 << 20) + 2),
                               NULL) == _lib.BSA_EINVAL
    # elementwise refinement / reconstruction and the complement lists
    e = Shape(1, 2, 100, 12, 0)
    assert lib.bsa_tail_refinement(e, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_tail_refinement(Shape(1, 2, 100, 16, 0), FAKE, FAKE, NULL, FAKE, FAKE, FAKE,
                                   NULL) == _lib.BSA_EINVAL
    assert lib.bsa_tail_reconstruct(Shape(1, 2, 100, 16, 0), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, NULL, FAKE,
                                    NULL) == _lib.BSA_EINVAL
    assert lib.bsa_complement_lists(s, FAKE, NULL, FAKE, NULL) == _lib.BSA_EINVAL


def test_fp8_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)
    x, codes, scales = FAKE, ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20)
    # quantize: every pointer required and 16-byte aligned; the block shapes of the other calls
    assert lib.bsa_quantize_fp8(s, NULL, codes, scales, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_quantize_fp8(s, x, codes, NULL, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_quantize_fp8(s, x, ctypes.c_void_p(codes.value + 8), scales, NULL) == _lib.BSA_EINVAL
    assert lib.bsa_quantize_fp8(Shape(1, 2, 1000, 96, 128), x, codes, scales, NULL) == _lib.BSA_ESHAPE
    assert lib.bsa_quantize_fp8(Shape(1, 2, 1000, 128, 32), x, codes, scales, NULL) == _lib.BSA_ESHAPE
    # attention: codes, scales, v and outputs required; D = 128 and 128-token blocks only
    q8, qs, k8, ks, v = (ctypes.c_void_p(a << 20) for a in (4, 5, 6, 7, 8))
    out = (ctypes.c_void_p(9 << 20), ctypes.c_void_p(10 << 20), NULL, NULL)  # o, lse, status, stream
    none4 = (NULL, NULL, NULL, NULL)  # kept_idx, kept_cnt, R, alpha
    assert lib.bsa_sparse_attn_fwd_fp8(s, q8, NULL, k8, ks, v, *none4, *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_fp8(s, q8, qs, k8, ks, v, FAKE, NULL, NULL, NULL, *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_fp8(s, q8, qs, k8, ks, v, NULL, NULL, FAKE, NULL, *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_fp8(s, q8, ctypes.c_void_p(qs.value + 2), k8, ks, v, *none4,
                                       *out) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_fp8(Shape(1, 2, 1000, 64, 128), q8, qs, k8, ks, v, *none4,
                                       *out) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_fwd_fp8(Shape(1, 2, 1000, 128, 64), q8, qs, k8, ks, v, *none4,
                                       *out) == _lib.BSA_ESHAPE


def test_interval_attention_validation(lib):
    s = Shape(1, 2, 1000, 128, 128)  # NB = 8
    qkv = [FAKE, ctypes.c_void_p(2 << 20), ctypes.c_void_p(3 << 20)]
    iv, ni = ctypes.c_void_p(4 << 20), ctypes.c_void_p(5 << 20)
    tail = (NULL, NULL, ctypes.c_void_p(6 << 20), ctypes.c_void_p(7 << 20), NULL, NULL)  # R, alpha, o, lse, status, stream
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, NULL, ni, 2, *tail) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, iv, NULL, 2, *tail) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, ctypes.c_void_p(iv.value + 2), ni, 2, *tail) == _lib.BSA_EINVAL
    # the width: 1 <= W <= NB
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, iv, ni, 0, *tail) == _lib.BSA_EINVAL
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, iv, ni, 9, *tail) == _lib.BSA_EINVAL
    # 128-token blocks only; R without alpha
    assert lib.bsa_sparse_attn_fwd_intervals(Shape(1, 2, 1000, 128, 64), *qkv, iv, ni, 2, *tail) == _lib.BSA_ESHAPE
    assert lib.bsa_sparse_attn_fwd_intervals(s, *qkv, iv, ni, 2, FAKE, NULL, *tail[2:]) == _lib.BSA_EINVAL
