"""Seeded synthetic workloads shaped like the pages' 768p video latents.

Video DeltaNet (paper "Video DeltaNet: A Video-Native Hybrid Attention for
Livestream Video Generation", Experiments / Implementation) measures on
MiniMax-H3 latents of a 14.3 s 768p clip with 42-102 latent frames.  Those
latents are not available, so every workload here is drawn from fixed
distributions with a seeded CPU generator, in a fixed order:

  1. q      [B, L, H, d]   ~ N(0, 1); L2-normalised per (token, head) when
                             ``q_norm`` is set
  2. k      [B, L, H, d]   ~ N(0, 1), always L2-normalised per (token, head)
  3. v      [B, L, H, d]   ~ N(0, 1)
  4. text_k [B, n_text, H, d] (L2-normalised), then text_v [B, n_text, H, d]
  5. beta   [B, H, 1+T]    = sigmoid(N(0, 1)); index 0 is the text frame
  6. W_soft, W_lin [H*d, D_out] ~ N(0, 1/d)   (d = head dim)
  7. gates  [2, B, L, H, d] = 0.5 (post-sigmoid; [0] Softmax, [1] linear)

All draws are float32; the result is then rounded once to the workload dtype
(round-to-nearest-even for bf16).  alpha (the decay gate) is None for the
standard workloads (alpha == 1); ``alpha_range`` draws alpha ~ U[lo, hi]
per (b, h, frame, channel) as an extra draw after the gates;
``beta_per_token`` then draws one write gate per token,
sigmoid(N(0, 1)) [B, H, n_text + L] (text tokens first), replacing beta.
``gates="random"`` replaces the constant gates with independent per-element
draws g_s, g_l = sigmoid(N(0, 1)) [B, L, H, d] each (Softmax gate first), taken
after every other draw so that nothing else changes.

L = T * N and token index = t * N + n (frame-major, token-minor).
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    B: int
    H: int
    T: int
    N: int
    d: int
    n_text: int
    dtype: str  # "f32" or "bf16"
    seed: int
    q_norm: bool
    chunk: int = 5
    window_radius: int = 1

    @property
    def L(self) -> int:
        return self.T * self.N

    @property
    def D(self) -> int:
        return self.H * self.d

    def replace(self, **kw) -> "Config":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny_f32": Config("tiny_f32", B=1, H=2, T=15, N=16, d=32, n_text=8,
                       dtype="f32", seed=0, q_norm=False),
    "small_bf16": Config("small_bf16", B=1, H=8, T=40, N=256, d=64, n_text=128,
                         dtype="bf16", seed=1, q_norm=False),
    "768p_bf16": Config("768p_bf16", B=1, H=24, T=75, N=1536, d=128, n_text=512,
                        dtype="bf16", seed=2, q_norm=True),
    "long_bf16": Config("long_bf16", B=1, H=24, T=300, N=1536, d=128, n_text=512,
                        dtype="bf16", seed=3, q_norm=True),
    "batched_bf16": Config("batched_bf16", B=16, H=16, T=20, N=576, d=128,
                           n_text=256, dtype="bf16", seed=4, q_norm=True),
    # the batched workload's short clip (T=15): run with chunk=5, and with
    # chunk=15 (one chunk, the window spans the clip) for the dense check
    "span_bf16": Config("span_bf16", B=16, H=16, T=15, N=576, d=128,
                        n_text=256, dtype="bf16", seed=4, q_norm=True),
    # the 768p shape with 4 heads: the profiler workload (inputs > L2, ~1.5 GB
    # on the device in total)
    "768p_h4_bf16": Config("768p_h4_bf16", B=1, H=4, T=75, N=1536, d=128, n_text=512,
                           dtype="bf16", seed=2, q_norm=True),
    # the batched clips with 4 of their 16 batch items: the profiler workload
    # of the VDA state kernels (inputs > L2, about 1.5 GB on the device)
    "batched_b4_bf16": Config("batched_b4_bf16", B=4, H=16, T=20, N=576, d=128,
                              n_text=256, dtype="bf16", seed=4, q_norm=True),
}

_TORCH_DTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def _l2n(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_inputs(cfg: Config, *, alpha_range: Optional[tuple] = None,
                beta_override: Optional[torch.Tensor] = None, beta_per_token: bool = False,
                gates: str = "const", device: str = "cpu") -> dict:
    """Draw one workload.  Returns torch tensors in the workload dtype
    (beta, alpha always float32) on ``device``.

    The draws always happen on the CPU generator, so the values do not depend
    on ``device``.
    """
    g = torch.Generator(device="cpu").manual_seed(cfg.seed)
    B, H, T, N, d, L = cfg.B, cfg.H, cfg.T, cfg.N, cfg.d, cfg.L
    dt = _TORCH_DTYPE[cfg.dtype]

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    out = {}
    q = randn(B, L, H, d)
    if cfg.q_norm:
        q = _l2n(q)
    out["q"] = q.to(dt)
    del q
    out["k"] = _l2n(randn(B, L, H, d)).to(dt)
    out["v"] = randn(B, L, H, d).to(dt)
    out["text_k"] = _l2n(randn(B, cfg.n_text, H, d)).to(dt)
    out["text_v"] = randn(B, cfg.n_text, H, d).to(dt)
    beta = torch.sigmoid(randn(B, H, 1 + T))
    out["beta"] = beta if beta_override is None else beta_override.float()
    std = 1.0 / np.sqrt(d)
    out["W_soft"] = (randn(H * d, H * d) * std).to(dt)
    out["W_lin"] = (randn(H * d, H * d) * std).to(dt)
    out["gates"] = torch.full((2, B, L, H, d), 0.5, dtype=dt)
    if alpha_range is not None:
        lo, hi = alpha_range
        u = torch.rand(B, H, T, d, generator=g, dtype=torch.float32)
        out["alpha"] = lo + (hi - lo) * u
    else:
        out["alpha"] = None
    if beta_per_token:
        out["beta"] = torch.sigmoid(randn(B, H, cfg.n_text + L))
    if gates == "random":
        g_s = torch.sigmoid(randn(B, L, H, d))
        g_l = torch.sigmoid(randn(B, L, H, d))
        out["gates"] = torch.stack([g_s, g_l]).to(dt)
        del g_s, g_l
    elif gates != "const":
        raise ValueError(f"gates must be 'const' or 'random', not {gates!r}")
    if device != "cpu":
        out = {k: (v.to(device) if v is not None else None) for k, v in out.items()}
    return out


def sample_rows(cfg: Config, per_frame: int = 4, extra_frac: float = 0.0,
                seed: int = 12345, chunks=None) -> np.ndarray:
    """Seeded sample of query token indices (within one batch item).

    Takes ``per_frame`` tokens (the first, the last and random ones) from:
    frames 0 and T-1 (the anchors) and the first and last frame of every
    chunk (or of the chunks listed in ``chunks``), plus a random
    ``extra_frac`` of all other tokens.  Sorted, unique.
    """
    rng = np.random.default_rng(seed)
    T, N, C = cfg.T, cfg.N, cfg.chunk
    frames = {0, T - 1}
    nc = (T + C - 1) // C
    for c in (range(nc) if chunks is None else [c % nc for c in chunks]):
        frames.add(c * C)
        frames.add(min(T, (c + 1) * C) - 1)
    rows = []
    for f in sorted(frames):
        pick = {0, N - 1}
        if N > 2:
            pick |= set(rng.choice(np.arange(1, N - 1), size=min(N - 2, max(0, per_frame - 2)),
                                   replace=False).tolist())
        rows += [f * N + n for n in sorted(pick)]
    if extra_frac > 0:
        n_extra = int(extra_frac * cfg.L)
        rows += rng.choice(cfg.L, size=n_extra, replace=False).tolist()
    return np.unique(np.asarray(rows, dtype=np.int64))


def grid_shape(N: int) -> tuple:
    """Spatial token grid (grid_h, grid_w) of a frame of N tokens: the factor
    pair with grid_h <= grid_w closest to square (1536 -> 32 x 48,
    576 -> 24 x 24, 256 -> 16 x 16)."""
    h = int(np.floor(np.sqrt(N)))
    while N % h:
        h -= 1
    return h, N // h


def make_prep_inputs(cfg: Config, *, grid: Optional[tuple] = None, device: str = "cpu") -> dict:
    """Raw inputs of the linear branch's feature map (VDA-Prep), drawn from a
    second seeded generator (seed + 7919) so that ``make_inputs`` is unchanged:

      1. q_raw, k_raw, v_raw [B, L, H, d] ~ N(0, 1)  (pretrained projections,
         before any normalisation), rounded once to the workload dtype
      2. wk_s [H*d, 3, 3] ~ N(0, 1) / 3,   wk_t [H*d, 5] ~ N(0, 1) / sqrt(5)
      3. wv_s, wv_t likewise                (float32; random stand-ins for the
         released depthwise spatial and five-tap temporal filters)

    ``grid`` is the frame's (grid_h, grid_w); default ``grid_shape(N)``.
    """
    g = torch.Generator(device="cpu").manual_seed(cfg.seed + 7919)
    B, H, d, L = cfg.B, cfg.H, cfg.d, cfg.L
    dt = _TORCH_DTYPE[cfg.dtype]
    gh, gw = grid_shape(cfg.N) if grid is None else grid
    assert gh * gw == cfg.N

    def randn(*shape):
        return torch.randn(*shape, generator=g, dtype=torch.float32)

    out = {"grid_h": gh, "grid_w": gw}
    for name in ("q_raw", "k_raw", "v_raw"):
        out[name] = randn(B, L, H, d).to(dt)
    out["wk_s"] = randn(H * d, 3, 3) / 3.0
    out["wk_t"] = randn(H * d, 5) / np.sqrt(5.0)
    out["wv_s"] = randn(H * d, 3, 3) / 3.0
    out["wv_t"] = randn(H * d, 5) / np.sqrt(5.0)
    if device != "cpu":
        out = {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in out.items()}
    return out


def make_text_queries(cfg: Config, *, device: str = "cpu") -> torch.Tensor:
    """Text-token queries [B, n_text, H, d] for the text rows of the joint
    Softmax, from a third seeded generator (seed + 104729, so no other draw
    changes): N(0, 1), L2-normalised per (token, head) when ``q_norm`` is set,
    rounded once to the workload dtype."""
    g = torch.Generator(device="cpu").manual_seed(cfg.seed + 104729)
    tq = torch.randn(cfg.B, cfg.n_text, cfg.H, cfg.d, generator=g, dtype=torch.float32)
    if cfg.q_norm:
        tq = _l2n(tq)
    return tq.to(_TORCH_DTYPE[cfg.dtype]).to(device)
