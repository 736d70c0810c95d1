"""bsa_reorder_tokens_noalloc: the allocation-free Hilbert reorder.

For callers that cannot allocate device memory (their memory belongs to a
host framework's allocator that hands over only input/output buffers, HBM is
already reserved, or cudaMalloc's implicit synchronisation is unacceptable),
the library keeps the reorder's scratch in a fixed array of its own.  This
test calls the new entry point through the C ABI, several times in a row on
different grids (the shared array keeps the previous call's contents), and
checks each result against the workspace-taking bsa_reorder_tokens on the
same grid and against the oracle's Hilbert order: permutations are
integers, so they must match bit for bit.  One grid, (2, 3, 200), has a
longest side between 129 and 256, so its 2^24-cell cube uses every one of
the array's 4096 chunk counts.

This file is collected last so that a run stopping at the first failure has
already run every other test; it also passes alone in a fresh process (the
first call on the device performs the array's address look-up).
"""

import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import _lib
from oracle import hilbert as ohil

pytestmark = pytest.mark.gpu


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _with_workspace(lib, grid, stream):
    L = grid[0] * grid[1] * grid[2]
    perm = torch.empty(L, dtype=torch.int32, device="cuda")
    inv = torch.empty(L, dtype=torch.int32, device="cuda")
    nbytes = lib.bsa_reorder_workspace_bytes(*grid)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    rc = lib.bsa_reorder_tokens(*grid, _ptr(perm), _ptr(inv), _ptr(ws), nbytes, stream)
    assert rc == 0, lib.bsa_strerror(rc)
    return perm, inv


def _no_alloc(lib, grid, stream):
    L = grid[0] * grid[1] * grid[2]
    perm = torch.full((L,), -7, dtype=torch.int32, device="cuda")
    inv = torch.full((L,), -7, dtype=torch.int32, device="cuda")
    rc = lib.bsa_reorder_tokens_noalloc(*grid, _ptr(perm), _ptr(inv), stream)
    assert rc == 0, lib.bsa_strerror(rc)
    return perm, inv


def test_noalloc_reorder_matches_workspace_reorder_twice():
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    # a large grid, one that fills the whole array, then a small one that
    # reuses part of it
    for grid in [(21, 45, 80), (2, 3, 200), (3, 5, 7)]:
        ref_perm, ref_inv = _with_workspace(lib, grid, stream)
        perm, inv = _no_alloc(lib, grid, stream)
        torch.cuda.synchronize()
        assert torch.equal(perm, ref_perm), grid
        assert torch.equal(inv, ref_inv), grid
        o_perm, o_inv = ohil.hilbert_perm(*grid)
        assert np.array_equal(perm.cpu().numpy(), o_perm), grid
        assert np.array_equal(inv.cpu().numpy(), o_inv), grid


def test_noalloc_reorder_rejects_grids_beyond_its_limit():
    lib = _lib.load()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    dummy = torch.empty(16, dtype=torch.int32, device="cuda")
    assert lib.bsa_reorder_tokens_noalloc(257, 2, 2, _ptr(dummy), _ptr(dummy), stream) == _lib.BSA_ESHAPE
    assert lib.bsa_reorder_tokens_noalloc(2, 2, 2, ctypes.c_void_p(0), _ptr(dummy), stream) == _lib.BSA_EINVAL
