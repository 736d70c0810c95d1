"""FP8 (e4m3) quantization of Q and K per token block -- oracle.

Source: the abstract on the page titled RECAP (a distilled pipeline that
runs its sparse attention in FP8 with fused kernels).  The pages give no
format, granularity or scaling rule; the reading here is:

* format: FP8 E4M3 as OCP defines it -- 1 sign bit, 4 exponent bits (bias
  7), 3 mantissa bits; normal values 2^(e-7) * (1 + m/8) for e = 1..15
  except the pattern e = 15, m = 7 (NaN), so the largest finite value is
  448; subnormals (e = 0) m/8 * 2^-6, the smallest 2^-9;
* encoding: round to the nearest E4M3 value, ties to the even mantissa,
  saturating to +-448 (no infinities);
* granularity: one scale per (batch, head, 128-token block) of Q and of K
  (the attention's own blocks): s = amax / 448 over the block's tokens and
  dimensions (s = 1 for an all-zero block), codes = E4M3(x * (448 / amax))
  with the reciprocal and the product each rounded to float32;
* only Q and K are quantized: the logits are (s_q * s_k) * (q8 . k8), the
  softmax and P.V stay as in the bf16 path.
The attention of the quantized inputs is then the plain masked attention of
the dequantized Q and K (oracle.attention), so the FP8 kernel is checked
against that definition at the bf16 path's tolerance, and against the
unquantized attention at a looser, stated tolerance.

Pinned by (tests/test_oracle_fp8.py): the codes of every representable value
decode to themselves; the encoder equals the nearest of the 255 finite
values found by brute force (ties to the even code) on a dense sweep; known
values (1.0 = 0x38, 448 = 0x7E, 2^-9 = 0x01, -0 / 0); saturation; the block
scale maps the block's largest magnitude to 448 exactly.
"""

import numpy as np

E4M3_MAX = 448.0


def e4m3_value(code):
    """Value of E4M3 code(s) (uint8) as float64; the NaN pattern gives nan."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return sign * val


def _finite_table():
    codes = np.arange(256, dtype=np.uint8)
    vals = e4m3_value(codes)
    keep = ~np.isnan(vals)
    return codes[keep], vals[keep]


def e4m3_encode(x):
    """Nearest E4M3 code of float32 values, ties to the even code, saturating
    to +-448; NaN gives the NaN code 0x7F.  Written on the exponent and
    mantissa of each value."""
    f = np.asarray(x, dtype=np.float32).astype(np.float64)
    sign = np.signbit(f)
    a = np.abs(f)
    out = np.zeros(f.shape, dtype=np.uint8)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, a)
    a = np.minimum(a, E4M3_MAX)
    # spacing of the E4M3 grid at a: 2^-9 below 2^-6 (subnormals), else
    # 2^(floor(log2 a) - 3)
    with np.errstate(divide="ignore"):
        ex = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    ex = np.maximum(ex, -6.0)
    step = np.exp2(ex - 3.0)
    q = a / step                      # exact in float64 (a is a float32 value)
    r = np.floor(q)
    frac = q - r
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2.0) == 1.0))
    r = r + up
    v = r * step                      # the rounded magnitude (may reach the next binade)
    v = np.minimum(v, E4M3_MAX)
    # code from the rounded magnitude
    with np.errstate(divide="ignore"):
        e2 = np.floor(np.log2(np.where(v > 0, v, 1.0)))
    sub = v < 2.0 ** -6
    mant_sub = np.round(v / 2.0 ** -9)
    e_field = np.where(sub, 0.0, e2 + 7.0)
    m_field = np.where(sub, mant_sub, v / np.exp2(e2) * 8.0 - 8.0)
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = np.where(v == 0, 0, code)
    code = code | np.where(sign, 0x80, 0)
    out[...] = code.astype(np.uint8)
    out[nan] = 0x7F
    return out


def quantize_blocks(x, blk):
    """Per (b, h, token block) E4M3 quantization of x [B,H,L,D] (bf16 values
    given as float32).  Returns (codes uint8 [B,H,L,D], scales float32
    [B,H,NB]): x ~= e4m3_value(codes) * scale within its block."""
    x = np.asarray(x, dtype=np.float32)
    B, H, L, D = x.shape
    nb = (L + blk - 1) // blk
    codes = np.empty(x.shape, dtype=np.uint8)
    scales = np.empty((B, H, nb), dtype=np.float32)
    for j in range(nb):
        lo, hi = j * blk, min(L, (j + 1) * blk)
        xb = x[:, :, lo:hi]
        amax = np.abs(xb).max(axis=(2, 3)).astype(np.float32)
        safe = np.where(amax > 0, amax, np.float32(1.0))
        inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
        inv = np.where(amax > 0, inv, np.float32(1.0)).astype(np.float32)
        scales[:, :, j] = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(1.0))
        codes[:, :, lo:hi] = e4m3_encode((xb * inv[:, :, None, None]).astype(np.float32))
    return codes, scales


def dequantize_blocks(codes, scales, blk):
    """float64 values e4m3_value(codes) * scale of the token's block."""
    B, H, L, D = codes.shape
    s = np.repeat(np.asarray(scales, dtype=np.float64), blk, axis=2)[:, :, :L]
    return e4m3_value(codes) * s[..., None]
