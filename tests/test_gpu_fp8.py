"""GPU parity of the FP8 Q.K^T path against the oracle (oracle/fp8.py,
oracle/attention.py).

* bsa_quantize_fp8: E4M3 codes bit-exact and scales equal to the oracle's
  (integer / byte work), ragged blocks, an all-zero block, negative values.
* bsa_sparse_attn_fwd_fp8: the block-sparse attention of the dequantized Q
  and K (codes x block scale, exactly what the tensor cores multiply), at the
  bf16 path's tolerance: O max-abs 2e-2, mean-abs 2e-3, LSE relative 1e-3.
  Ragged tail, random kept lists (empty and full rows), the fused correction,
  dense; and the 480P shape with 2 heads (512 work items, >= 3 per CTA) on
  sampled query blocks.
The cost of the format itself (dequantized against unquantized Q and K, on
the oracle alone) is checked in tests/test_oracle_fp8.py.
"""

import dataclasses

import numpy as np
import pytest
import torch

from block_sparse_attention_logits_b200 import api, configs
from block_sparse_attention_logits_b200.synthetic import make_qkv, random_bf16, random_kept_lists
from oracle import attention as oatt
from oracle import correction as ocor
from oracle import fp8 as ofp8
from oracle import scoring as osco
from oracle import topp as otop

from .gpu_helpers import assert_attention_close, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("D", [128, 64])
def test_quantize_matches_oracle_bit_exact(D):
    B, H, L, blk = 1, 2, 5 * 128 + 37, 128
    x = random_bf16((B, H, L, D), 31, scale=3.0)
    x[0, 1, 128:256] = 0  # an all-zero block
    x[0, 0, 300, 5] = -40.0  # one large magnitude in block 2
    codes, scales = api.quantize_fp8(x.to(DEV), blk)
    torch.cuda.synchronize()
    oc, osc = ofp8.quantize_blocks(x.float().numpy(), blk)
    assert np.array_equal(to_np(codes), oc)
    assert np.array_equal(to_np(scales), osc)


def _dequant(codes, scales, blk):
    return ofp8.dequantize_blocks(to_np(codes), to_np(scales), blk)


def _case(seed, L, H, density):
    B, D, blk = 1, 128, 128
    nb = (L + blk - 1) // blk
    q = random_bf16((B, H, L, D), seed, scale=2.0)
    k = random_bf16((B, H, L, D), seed + 1, scale=2.0)
    v = random_bf16((B, H, L, D), seed + 2, scale=1.0)
    idx, cnt = random_kept_lists(B, H, nb, seed + 3, density, 2.0)
    return q, k, v, idx, cnt, blk


@pytest.mark.parametrize("mode", ["sparse", "correction", "dense"])
def test_fp8_attention_matches_dequantized_oracle(mode):
    q, k, v, idx, cnt, blk = _case(40, 5 * 128 + 37, 2, 0.4)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    q8, qs = api.quantize_fp8(qd, blk)
    k8, ks = api.quantize_fp8(kd, blk)
    R = alpha = None
    if mode == "correction":
        R = random_bf16(q.shape, 44, scale=0.05)
        alpha = torch.tensor([0.3, 1.0], dtype=torch.float32)
    kept = (None, None) if mode == "dense" else (torch.from_numpy(idx).to(DEV), torch.from_numpy(cnt).to(DEV))
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd_fp8(q8, qs, k8, ks, vd, blk, *kept, None if R is None else R.to(DEV),
                                     None if alpha is None else alpha.to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    qh, kh = _dequant(q8, qs, blk), _dequant(k8, ks, blk)
    vn = v.float().numpy()
    if mode == "dense":
        O, LSE = oatt.dense_attention(qh, kh, vn)
    else:
        O, LSE = oatt.masked_attention(qh, kh, vn, idx, cnt, blk)
    if R is not None:
        O = ocor.apply_correction(O, R.float().numpy(), alpha.numpy())
    assert_attention_close(to_np(o), to_np(lse), O, LSE, f"fp8 {mode}")


def test_fp8_attention_480p_2heads_sampled():
    w = dataclasses.replace(configs.WAN13B_480P, H=2)
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    qn, kn = t["q"].float().numpy(), t["k"].float().numpy()
    _, _, P = osco.score_blocks(qn, kn, w.blk)
    _, idx, cnt = otop.select_topp_mask_fast(P, np.full(w.H, 0.9, np.float32))
    q8, qs = api.quantize_fp8(t["q"].to(DEV), w.blk)
    k8, ks = api.quantize_fp8(t["k"].to(DEV), w.blk)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    o, lse = api.sparse_attn_fwd_fp8(q8, qs, k8, ks, t["v"].to(DEV), w.blk, torch.from_numpy(idx).to(DEV),
                                     torch.from_numpy(cnt).to(DEV), status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    rng = np.random.default_rng(9)
    units = [(0, h, int(i)) for h in range(w.H) for i in sorted(set([0, w.NB - 1]) | set(rng.choice(w.NB, 14)))]
    O, LSE = oatt.masked_attention(_dequant(q8, qs, w.blk), _dequant(k8, ks, w.blk), t["v"].float().numpy(), idx,
                                   cnt, w.blk, units=units)
    assert_attention_close(to_np(o), to_np(lse), O, LSE, "fp8 480P")
