"""Pins of the VDA-Prep oracle (linear-branch feature map) against closed
forms, a library correlation and brute force, independent of its own code."""
import numpy as np
import pytest
import scipy.ndimage
import scipy.special

from oracle import vda_prep as P


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _tiny(seed=0, B=2, T=4, gh=3, gw=5, H=2, d=3):
    x = _rand((B, T * gh * gw, H, d), seed)
    ws = _rand((H * d, 3, 3), seed + 1)
    wt = _rand((H * d, 5), seed + 2)
    return x, ws, wt, T, gh, gw


def test_conv_equals_library_3d_correlation():
    """Separable depthwise conv = scipy's 3-D correlation with the outer-product
    kernel w_t[tau] * w_s[i, j], per channel, zero boundary."""
    x, ws, wt, T, gh, gw = _tiny()
    B, L, H, d = x.shape
    got = P.short_conv(x, ws, wt, T, gh, gw).reshape(B, T, gh, gw, H * d)
    X = x.reshape(B, T, gh, gw, H * d)
    for b in range(B):
        for c in range(H * d):
            k3 = wt[c][:, None, None] * ws[c][None, :, :]
            want = scipy.ndimage.correlate(X[b, :, :, :, c], k3, mode="constant", cval=0.0)
            np.testing.assert_allclose(got[b, :, :, :, c], want, rtol=1e-12, atol=1e-12)


def test_conv_brute_force_loops():
    """Every output point summed over its 45 taps with explicit bounds checks."""
    x, ws, wt, T, gh, gw = _tiny(seed=5, B=1, T=3, gh=2, gw=4, H=1, d=2)
    got = P.short_conv(x, ws, wt, T, gh, gw)
    N = gh * gw
    for t in range(T):
        for y in range(gh):
            for xx in range(gw):
                for c in range(2):
                    s = 0.0
                    for tau in range(5):
                        for i in range(3):
                            for j in range(3):
                                tt, yy, x2 = t + tau - 2, y + i - 1, xx + j - 1
                                if 0 <= tt < T and 0 <= yy < gh and 0 <= x2 < gw:
                                    s += wt[c, tau] * ws[c, i, j] * x[0, tt * N + yy * gw + x2, 0, c]
                    assert abs(got[0, t * N + y * gw + xx, 0, c] - s) < 1e-12


def test_delta_filters_are_identity():
    x, ws, wt, T, gh, gw = _tiny(seed=9)
    ws = np.zeros_like(ws)
    ws[:, 1, 1] = 1.0
    wt = np.zeros_like(wt)
    wt[:, 2] = 1.0
    np.testing.assert_array_equal(P.short_conv(x, ws, wt, T, gh, gw), x)


def test_temporal_tap_is_a_frame_shift():
    """Tap 0 alone (offset -2): out[t] = in[t - 2], zero for the first two frames."""
    x, ws, wt, T, gh, gw = _tiny(seed=11, T=5)
    ws = np.zeros_like(ws)
    ws[:, 1, 1] = 1.0
    wt = np.zeros_like(wt)
    wt[:, 0] = 1.0
    N = gh * gw
    got = P.short_conv(x, ws, wt, T, gh, gw)
    np.testing.assert_array_equal(got[:, :2 * N], 0.0)
    np.testing.assert_array_equal(got[:, 2 * N:], x[:, :(T - 2) * N])


def test_spatial_tap_is_a_column_shift():
    """Spatial tap (row 1, col 0), offset (0, -1): out[y, x] = in[y, x - 1]."""
    x, ws, wt, T, gh, gw = _tiny(seed=12)
    B, L, H, d = x.shape
    ws = np.zeros_like(ws)
    ws[:, 1, 0] = 1.0
    wt = np.zeros_like(wt)
    wt[:, 2] = 1.0
    got = P.short_conv(x, ws, wt, T, gh, gw).reshape(B, T, gh, gw, H, d)
    X = x.reshape(B, T, gh, gw, H, d)
    np.testing.assert_array_equal(got[:, :, :, 0], 0.0)
    np.testing.assert_array_equal(got[:, :, :, 1:], X[:, :, :, :-1])


def test_silu_closed_form():
    assert P.silu(0.0) == 0.0
    assert abs(P.silu(1.0) - 0.7310585786300049) < 1e-15
    assert abs(P.silu(-1.0) + 0.2689414213699951) < 1e-15
    z = np.linspace(-30, 30, 101)
    np.testing.assert_allclose(P.silu(z), z * scipy.special.expit(z), rtol=1e-14, atol=1e-300)


def test_l2_normalize_norm_and_direction():
    x = _rand((7, 3, 16), 3)
    y = P.l2_normalize(x, eps=1e-6)
    s = np.sum(x * x, -1)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.sqrt(s / (s + 1e-6)), rtol=1e-13)
    cos = np.sum(x * y, -1) / (np.linalg.norm(x, axis=-1) * np.linalg.norm(y, axis=-1))
    np.testing.assert_allclose(cos, 1.0, rtol=1e-13)
    assert np.all(P.l2_normalize(np.zeros((2, 4))) == 0.0)


def test_prep_with_delta_filters():
    """With identity filters: q_l = L2(q), k_l = L2(SiLU(k)), v_l = SiLU(v);
    k_l and q_l have unit norm up to eps."""
    x, ws, wt, T, gh, gw = _tiny(seed=21)
    q, k, v = x, _rand(x.shape, 22), _rand(x.shape, 23)
    ws = np.zeros_like(ws)
    ws[:, 1, 1] = 1.0
    wt = np.zeros_like(wt)
    wt[:, 2] = 1.0
    ql, kl, vl = P.vda_prep(q, k, v, ws, wt, ws, wt, T, gh, gw)
    sk = k * scipy.special.expit(k)
    np.testing.assert_allclose(vl, v * scipy.special.expit(v), rtol=1e-13)
    nk = np.sqrt(np.sum(sk * sk, -1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(kl * nk, sk, rtol=1e-13)
    nq = np.sum(q * q, -1)
    np.testing.assert_allclose(np.linalg.norm(ql, axis=-1), np.sqrt(nq / (nq + 1e-6)),
                               rtol=1e-13)


def test_conv_order_commutes():
    """Spatial and temporal filters act on different axes: applying the
    temporal filter first gives the same result (property of the separable
    form)."""
    x, ws, wt, T, gh, gw = _tiny(seed=31)
    ident_s = np.zeros_like(ws)
    ident_s[:, 1, 1] = 1.0
    ident_t = np.zeros_like(wt)
    ident_t[:, 2] = 1.0
    a = P.short_conv(P.short_conv(x, ident_s, wt, T, gh, gw), ws, ident_t, T, gh, gw)
    np.testing.assert_allclose(a, P.short_conv(x, ws, wt, T, gh, gw), rtol=1e-12, atol=1e-12)
