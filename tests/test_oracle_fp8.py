"""Pins of the FP8 (E4M3) quantization oracle (oracle/fp8.py) to the format's
definition: every code round-trips, the encoder is the nearest finite value
by brute force (ties to the even code, saturation at 448), known codes, and
the per-block scale maps each block's largest magnitude to 448."""

import dataclasses

import numpy as np

from block_sparse_attention_logits_b200 import configs
from block_sparse_attention_logits_b200.synthetic import make_qkv
from oracle import attention as oatt
from oracle import fp8
from oracle import scoring as osco
from oracle import topp as otop


def _table():
    codes = np.arange(256, dtype=np.uint8)
    vals = fp8.e4m3_value(codes)
    keep = ~np.isnan(vals)
    return codes[keep], vals[keep]


def test_known_values():
    assert fp8.e4m3_value(np.uint8(0x38)) == 1.0
    assert fp8.e4m3_value(np.uint8(0x7E)) == 448.0
    assert fp8.e4m3_value(np.uint8(0x01)) == 2.0 ** -9
    assert fp8.e4m3_value(np.uint8(0x08)) == 2.0 ** -6      # smallest normal
    assert np.isnan(fp8.e4m3_value(np.uint8(0x7F))) and np.isnan(fp8.e4m3_value(np.uint8(0xFF)))
    enc = fp8.e4m3_encode(np.array([1.0, 448.0, 2.0 ** -9, -1.0, 0.0, -0.0, 1e9, -1e9, np.nan], np.float32))
    assert enc.tolist() == [0x38, 0x7E, 0x01, 0xB8, 0x00, 0x80, 0x7E, 0xFE, 0x7F]
    # ties go to the even code: half of 2^-9 -> 0, 1.5 * 2^-9 -> 2 * 2^-9, 1 + 1/16 -> 1
    assert fp8.e4m3_encode(np.array([2.0 ** -10, 1.5 * 2.0 ** -9, 1.0625, 1.1875], np.float32)).tolist() == \
        [0x00, 0x02, 0x38, 0x3A]


def test_every_code_round_trips():
    codes, vals = _table()
    assert len(codes) == 254
    back = fp8.e4m3_encode(vals.astype(np.float32))
    # -0 and +0 keep their sign bit; every other finite code maps to itself
    assert np.array_equal(back, codes)


def test_encoder_is_the_nearest_value_by_brute_force():
    codes, vals = _table()
    rng = np.random.default_rng(3)
    x = np.concatenate([np.linspace(-460, 460, 40001), rng.standard_normal(20000) * 3,
                        rng.standard_normal(20000) * 2.0 ** -8, (vals[:-1] + vals[1:]) / 2]).astype(np.float32)
    got = fp8.e4m3_encode(x)
    xd = np.clip(x.astype(np.float64), -448.0, 448.0)
    dist = np.abs(xd[:, None] - vals[None, :])
    best = dist.min(axis=1)
    cand = dist == best[:, None]
    # among equally near codes: the even one (the value with an even mantissa);
    # at 0 both signed zeros are nearest: keep the sign of x
    want = np.empty(len(x), np.uint8)
    for i in range(len(x)):
        cs = codes[cand[i]]
        if len(cs) > 1:
            cs = cs[(cs & 1) == 0]
        if len(cs) > 1:  # +0 and -0
            cs = cs[(cs >= 0x80) == bool(np.signbit(x[i]))]
        want[i] = cs[0]
    assert np.array_equal(got, want)


def test_block_scale_maps_the_block_maximum_to_448():
    rng = np.random.default_rng(4)
    x = (rng.standard_normal((1, 2, 300, 16)) * rng.uniform(0.01, 50, (1, 2, 300, 1))).astype(np.float32)
    x[0, 1, 128:256] = 0.0  # an all-zero block
    codes, scales = fp8.quantize_blocks(x, 128)
    assert scales.shape == (1, 2, 3) and scales[0, 1, 1] == 1.0
    deq = fp8.dequantize_blocks(codes, scales, 128)
    for j in range(3):
        blk = slice(128 * j, min(300, 128 * (j + 1)))
        for h in range(2):
            amax = np.abs(x[0, h, blk]).max()
            if amax == 0:
                assert not deq[0, h, blk].any()
                continue
            assert np.abs(codes[0, h, blk] & 0x7F).max() == 0x7E        # the largest maps to 448
            assert abs(np.abs(deq[0, h, blk]).max() - amax) <= 2.0 ** -20 * amax
    # relative error of one E4M3 rounding on normal-range values
    ok = np.abs(x) >= 2.0 ** -6 * np.repeat(scales, 128, axis=2)[:, :, :300, None]
    rel = np.abs(deq - x)[ok] / np.abs(x)[ok]
    assert rel.max() <= 2.0 ** -4 + 1e-9


def test_format_cost_on_the_720p_inputs_is_bounded():
    """Oracle only (no GPU result enters): E4M3 Q and K against bf16 Q and K
    on one head of the 720P workload, sampled query blocks.  The bounds are
    the measured cost (O max-abs 0.19, mean-abs 0.0074, LSE abs 0.21) with
    about 1.5x margin, so a format or scaling change that loses precision is
    caught."""
    w = dataclasses.replace(configs.WAN14B_720P, H=1, hilbert=False)
    t = make_qkv(w.B, w.H, w.grid, w.D, w.fp)
    qn, kn, vn = (t[n].float().numpy() for n in "qkv")
    _, _, P = osco.score_blocks(qn, kn, w.blk)
    _, idx, cnt = otop.select_topp_mask_fast(P, np.full(w.H, w.p[0], np.float32))
    q8, qs = fp8.quantize_blocks(qn, w.blk)
    k8, ks = fp8.quantize_blocks(kn, w.blk)
    units = [(0, 0, int(i)) for i in np.random.default_rng(0).choice(w.NB, 20, replace=False)]
    O1, L1 = oatt.masked_attention(qn, kn, vn, idx, cnt, w.blk, units=units)
    O2, L2 = oatt.masked_attention(fp8.dequantize_blocks(q8, qs, w.blk), fp8.dequantize_blocks(k8, ks, w.blk), vn,
                                   idx, cnt, w.blk, units=units)
    m = ~np.isnan(O1)
    err = np.abs(O1 - O2)[m]
    lm = ~np.isnan(L1)
    assert err.max() <= 0.3 and err.mean() <= 0.012
    assert np.abs(L1 - L2)[lm].max() <= 0.32
