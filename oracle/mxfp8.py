"""MXFP8 quantisation and the MXFP8 output projection, in float64 (oracle).

TEST INFRASTRUCTURE ONLY: used by ``tests/`` (and nothing on the product
path).  It shares no code with the CUDA library.

Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation", implementation section ("Other optimizations": MXFP8 for the QKV,
output and feed-forward GEMMs, with the recurrent states and the inverses kept
in FP32).  The pages name the format and nothing more; the format itself is
the OCP Microscaling (MX) one, taken here from its published definition:

* a block of 32 consecutive elements along the contraction dimension shares
  one scale X = 2^e, stored as an unsigned 8-bit exponent (UE8M0, e + 127);
* e = floor(log2(max |v| over the block)) - 8, where 8 is the exponent of the
  largest normal E4M3 value (448 = 1.75 * 2^8); an all-zero block takes the
  smallest scale;
* each element is v / X rounded to E4M3 (1 sign, 4 exponent bits with bias 7,
  3 mantissa bits, subnormals down to 2^-9, largest finite 448, no infinity)
  to nearest, ties to even, saturating at +-448.

Reading (M1): the library forms its projection operands in fp16 first (the
gated branch outputs x and W, as on its default path); the MXFP8 mode quantises
those fp16 values.  This oracle does the same: x and W are rounded to fp16,
then quantised, then multiplied exactly (float64).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64
E4M3_MAX = 448.0
E4M3_EMAX = 8      # exponent of the largest normal E4M3 value
E4M3_EMIN = -6     # exponent of the smallest normal
E4M3_MBITS = 3
BLOCK = 32


def e4m3_round(y):
    """Round to the nearest E4M3 value (ties to even), saturating at +-448."""
    y = np.asarray(y, F64)
    a = np.abs(y)
    # quantum of the binade (normal: 2^(e-3); subnormal: 2^-9)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, E4M3_EMIN)
    q = np.exp2(e - E4M3_MBITS)
    r = np.round(a / q) * q          # numpy rounds halves to even
    r = np.minimum(r, E4M3_MAX)
    return np.sign(y) * np.where(a > 0, r, 0.0)


def e4m3_values():
    """Every finite E4M3 value, from the format's definition (254 codes:
    +-0, 2 * (7 subnormals + 15 binades * 8 mantissas - 1 for NaN))."""
    vals = [0.0]
    for m in range(1, 8):                        # subnormals m * 2^-9
        vals.append(m * 2.0 ** -9)
    for e in range(-6, 9):                       # normals (1 + m/8) * 2^e
        for m in range(8):
            v = (1 + m / 8) * 2.0 ** e
            if v <= E4M3_MAX:
                vals.append(v)
    vals = np.array(vals)
    return np.concatenate([-vals[:0:-1], vals])


def block_exponents(v, axis=-1):
    """Shared exponent e of every block of 32 along ``axis`` (length a
    multiple of 32): floor(log2(amax)) - 8, or -127 for an all-zero block.
    Returns an array with the blocked axis of length n / 32."""
    v = np.moveaxis(np.asarray(v, F64), axis, -1)
    n = v.shape[-1]
    assert n % BLOCK == 0
    amax = np.abs(v.reshape(v.shape[:-1] + (n // BLOCK, BLOCK))).max(axis=-1)
    e = np.where(amax > 0, np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - E4M3_EMAX, -127.0)
    e = np.clip(e, -127.0, 127.0)
    return np.moveaxis(e, -1, axis)


def mxfp8_quantize(v, axis=-1):
    """(elements, exponents): the E4M3 elements (as float64 values) of v
    scaled by its blocks' scales, and the blocks' shared exponents.  The
    dequantised value is elements * 2^exponent (per block)."""
    v = np.moveaxis(np.asarray(v, F64), axis, -1)
    e = block_exponents(v, -1)
    scale = np.repeat(np.exp2(e), BLOCK, axis=-1)
    el = e4m3_round(v / scale)
    return np.moveaxis(el, -1, axis), np.moveaxis(e, -1, axis)


def mxfp8_dequantize(v, axis=-1):
    """v rounded through MXFP8 (quantised, then scaled back)."""
    el, e = mxfp8_quantize(v, axis)
    el = np.moveaxis(el, axis, -1)
    e = np.moveaxis(e, axis, -1)
    return np.moveaxis(el * np.repeat(np.exp2(e), BLOCK, axis=-1), -1, axis)


def to_fp16(v):
    return np.asarray(v, F64).astype(np.float16).astype(F64)


def output_projection_mxfp8(o_s, o_l, g_s, g_l, W_soft, W_lin, eps=1e-6):
    """out = deq(x) deq(W), x = [g_s * o_s | g_l * RMS(o_l)] per token
    (the concatenated operand of the two projections, heads in order), W =
    [W_soft; W_lin]: both rounded to fp16 (reading M1) and quantised in blocks
    of 32 along the contraction dimension (x along its row, W along its
    column), products and sums exact."""
    o_s = np.asarray(o_s, F64)
    o_l = np.asarray(o_l, F64)
    B, R, H, dv = o_s.shape
    ms = np.mean(o_l * o_l, axis=-1, keepdims=True)
    xs = (np.asarray(g_s, F64) * o_s).reshape(B, R, H * dv)
    xl = (np.asarray(g_l, F64) * o_l / np.sqrt(ms + eps)).reshape(B, R, H * dv)
    x = np.concatenate([xs, xl], axis=-1)
    W = np.concatenate([np.asarray(W_soft, F64), np.asarray(W_lin, F64)], axis=0)
    xq = mxfp8_dequantize(to_fp16(x), axis=-1)
    Wq = mxfp8_dequantize(to_fp16(W), axis=0)
    return xq @ Wq
