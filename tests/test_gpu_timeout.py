"""A bounded wait that runs out on the GPU: a wait on a barrier that nothing
arrives at gives up after its limit, the status word carries
BSA_DEV_TIMEOUT, and the context stays usable (a kernel launched afterwards
runs and its result is correct)."""

import time

import pytest
import torch

from block_sparse_attention_logits_b200 import _lib, api

pytestmark = pytest.mark.gpu


def test_wait_runs_out_and_reports_timeout():
    lib = _lib.load()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.time()
    rc = lib.bsa_wait_selftest(status.data_ptr(), 50_000_000, stream)   # 50 ms
    assert rc == 0
    torch.cuda.synchronize()
    assert time.time() - t0 < 5.0
    assert status.item() & _lib.BSA_DEV_TIMEOUT
    # the context is still usable
    o = api.refresh_refinement(torch.ones((1, 1, 8, 8), dtype=torch.bfloat16, device="cuda"),
                               torch.zeros((1, 1, 8, 8), dtype=torch.bfloat16, device="cuda"))
    torch.cuda.synchronize()
    assert torch.equal(o.cpu(), torch.ones((1, 1, 8, 8), dtype=torch.bfloat16))
