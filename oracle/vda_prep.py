"""Plain float64 CPU oracle for VDA-Prep, the linear branch's feature map.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or runs
this module; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU legs of
``bench.py`` may use it.  It shares no code with the CUDA library.

Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation", method section (the paragraph on the two branches' inputs: the
linear branch takes the same pretrained Q, K, V projections and applies its
own feature map, a separable short convolution of K and V followed by SiLU,
with L2 normalisation of Q and K; the released convolution is a depthwise
spatial filter followed by a five-tap temporal filter) and implementation
section ("Fused VDA kernels": VDA-Prep fuses the convolution, SiLU, L2
normalisation and the layout conversion for K and V).

Readings where the pages are silent (each listed with its reason in the design
notes):
  P1  the N tokens of a frame form a row-major grid_h x grid_w grid
      (token n = y * grid_w + x); the spatial filter is depthwise (one filter
      per channel of every head), ks x ks with ks = 3, zero padding, output the
      same size;
  P2  the temporal filter is depthwise with 5 taps centred on the frame
      (offsets -2..+2), zero padding at the clip ends;
  P3  both filters are cross-correlations (out[y] = sum_i w[i] in[y + i - r]),
      the deep-learning convention; no bias;
  P4  order: short convolution -> SiLU for K and V, then L2 over the d
      channels of each (token, head) for K; Q gets the L2 normalisation only;
      L2(x) = x / sqrt(sum x^2 + eps), eps = 1e-6;
  P5  the text tokens have no spatial or temporal grid, so VDA-Prep covers the
      video tokens only.

Layouts: q, k, v [B, L, H, d] with L = T * grid_h * grid_w, token index
t * N + y * grid_w + x; spatial filters [H*d, ks, ks]; temporal filters
[H*d, 5] (channel c = h * d + i).
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + exp(-x))."""
    x = np.asarray(x, F64)
    return x / (1.0 + np.exp(-x))


def l2_normalize(x, eps=1e-6):
    """x / sqrt(sum_d x^2 + eps) over the last (channel) axis (P4)."""
    x = np.asarray(x, F64)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def short_conv(x, w_s, w_t, T, grid_h, grid_w):
    """Depthwise ks x ks spatial filter, then depthwise temporal filter, both
    with zero padding and 'same' output size (P1-P3).

    x [B, T*grid_h*grid_w, H, d]; w_s [H*d, ks, ks]; w_t [H*d, kt].
    """
    x = np.asarray(x, F64)
    w_s = np.asarray(w_s, F64)
    w_t = np.asarray(w_t, F64)
    B, L, H, d = x.shape
    C = H * d
    X = x.reshape(B, T, grid_h, grid_w, C)
    ks = w_s.shape[-1]
    r = ks // 2
    Xp = np.pad(X, ((0, 0), (0, 0), (r, r), (r, r), (0, 0)))
    Y = np.zeros_like(X)
    for i in range(ks):          # y offset i - r
        for j in range(ks):      # x offset j - r
            Y += Xp[:, :, i:i + grid_h, j:j + grid_w, :] * w_s[:, i, j]
    kt = w_t.shape[-1]
    rt = kt // 2
    Yp = np.pad(Y, ((0, 0), (rt, rt), (0, 0), (0, 0), (0, 0)))
    Z = np.zeros_like(Y)
    for tau in range(kt):        # frame offset tau - rt
        Z += Yp[:, tau:tau + T] * w_t[:, tau]
    return Z.reshape(B, L, H, d)


def vda_prep(q, k, v, wk_s, wk_t, wv_s, wv_t, T, grid_h, grid_w, eps=1e-6):
    """The linear branch's q, k, v from the raw projections (P4):
    q_l = L2(q), k_l = L2(SiLU(conv_k(k))), v_l = SiLU(conv_v(v))."""
    q_l = l2_normalize(q, eps)
    k_l = l2_normalize(silu(short_conv(k, wk_s, wk_t, T, grid_h, grid_w)), eps)
    v_l = silu(short_conv(v, wv_s, wv_t, T, grid_h, grid_w))
    return q_l, k_l, v_l
