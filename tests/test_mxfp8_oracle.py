"""Pins of the MXFP8 oracle (oracle/mxfp8.py) against the format's definition
and an independent conversion (torch's float8_e4m3fn)."""
import numpy as np
import pytest
import torch

from oracle import mxfp8 as MX


def test_e4m3_grid_has_the_formats_values():
    v = MX.e4m3_values()
    assert len(v) == 253  # +-(7 subnormals + 119 normals up to 448) and 0
    assert v.max() == 448.0 and v.min() == -448.0
    assert np.min(v[v > 0]) == 2.0 ** -9
    # every grid value rounds to itself
    np.testing.assert_array_equal(MX.e4m3_round(v), v)
    # and agrees with torch's float8_e4m3fn encoding of the same values
    t = torch.tensor(v, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(t, v)


def test_e4m3_rounding_matches_torch_inside_the_range():
    rng = np.random.default_rng(3)
    y = np.concatenate([rng.normal(size=20000) * s for s in (1e-3, 0.05, 1, 30, 200)])
    y = y[np.abs(y) <= 448]
    # midpoints between grid values: ties go to the even mantissa
    g = MX.e4m3_values()
    mids = (g[1:] + g[:-1]) / 2
    y = np.concatenate([y, mids[np.abs(mids) <= 448]]).astype(np.float32).astype(np.float64)
    want = torch.tensor(y, dtype=torch.float32).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(MX.e4m3_round(y), want)


def test_e4m3_saturates():
    np.testing.assert_array_equal(MX.e4m3_round([449.0, 500.0, 1e9, -1e9]), [448, 448, 448, -448])


def test_block_scale_rule():
    v = np.zeros(64)
    v[3] = 1.0       # block 0: amax 1 -> e = 0 - 8
    v[40] = -300.0   # block 1: amax 300 -> floor(log2 300) = 8 -> e = 0
    e = MX.block_exponents(v)
    np.testing.assert_array_equal(e, [-8, 0])
    assert MX.block_exponents(np.zeros(32))[0] == -127
    # the block maximum lands in [256, 512) before rounding (448 saturates)
    rng = np.random.default_rng(4)
    w = rng.normal(size=(50, 32)) * np.exp(rng.normal(size=(50, 1)) * 4)
    e = MX.block_exponents(w)
    top = np.abs(w).max(axis=1) / np.exp2(e[:, 0])
    assert np.all((top >= 256) & (top < 512))


def test_representable_values_survive_the_round_trip():
    rng = np.random.default_rng(5)
    g = MX.e4m3_values()
    el = rng.choice(g[np.abs(g) <= 255], size=(8, 64))
    el[:, 0] = 256.0  # fixes the scale of block 0 to 2^0 * ...
    el[:, 32] = -320.0
    for s in (-20, 0, 7):
        v = el * 2.0 ** s
        np.testing.assert_array_equal(MX.mxfp8_dequantize(v), v)


@pytest.mark.parametrize("seed", range(3))
def test_round_trip_error_bound(seed):
    """Elements not clipped at 448 and in the normal range of their block keep
    a relative error <= 2^-4 (3 mantissa bits, round to nearest)."""
    rng = np.random.default_rng(seed)
    v = rng.normal(size=(64, 256)) * np.exp(rng.normal(size=(64, 1)))
    q = MX.mxfp8_dequantize(v)
    e = np.repeat(MX.block_exponents(v), 32, axis=-1)
    y = np.abs(v) / np.exp2(e)
    ok = (y >= 2.0 ** -6) & (y <= 448)
    rel = np.abs(q - v)[ok] / np.abs(v)[ok]
    assert rel.max() <= 2.0 ** -4 + 1e-15
    # clipped elements are exactly 448 times the scale
    clip = y > 448
    np.testing.assert_array_equal(np.abs(q[clip]), (448 * np.exp2(e))[clip])


def test_quantisation_axis_is_the_contraction_axis():
    rng = np.random.default_rng(6)
    W = rng.normal(size=(64, 5))
    W[:32, 2] *= 1000  # a large first block in column 2 only
    q = MX.mxfp8_dequantize(W, axis=0)
    for c in range(5):
        np.testing.assert_array_equal(q[:, c], MX.mxfp8_dequantize(W[:, c]))


def test_mxfp8_projection_is_the_product_of_quantised_operands():
    """Pins the operand assembly: with gates and inputs whose fp16 values and
    MXFP8 values coincide, the MXFP8 projection is the exact projection."""
    rng = np.random.default_rng(7)
    B, R, H, dv, Do = 1, 3, 2, 32, 6
    g = MX.e4m3_values()
    pick = lambda *s: rng.choice(g[(np.abs(g) >= 1) & (np.abs(g) <= 255)], size=s)
    o_s = pick(B, R, H, dv)
    o_s[..., 0] = 256.0
    o_l = pick(B, R, H, dv)
    W_soft, W_lin = pick(H * dv, Do), pick(H * dv, Do)
    W_soft[::32] = 256.0
    W_lin[::32] = 256.0
    one = np.ones((B, R, H, dv))
    # g_l = 0: only the Softmax half, whose operand is exactly representable
    got = MX.output_projection_mxfp8(o_s, o_l, one, 0 * one, W_soft, W_lin)
    want = o_s.reshape(B, R, H * dv) @ W_soft
    np.testing.assert_array_equal(got, want)
