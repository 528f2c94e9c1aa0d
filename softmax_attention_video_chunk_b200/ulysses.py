"""Head-sharded (Ulysses) VDN hybrid attention forward over P ranks.

"Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation", implementation section: for multi-GPU inference VDA is sharded by
attention head, following Ulysses sequence parallelism.  Every step of the
forward is independent per head except the output projection, which
contracts over heads.  With P ranks:

  1. each rank holds a contiguous shard of L/P tokens of q, k, v and the gates;
  2. one all-to-all per tensor turns token shards into head shards: every rank
     then holds all L tokens of H/P heads;
  3. the rank computes the projection operand of its heads,
     x = [g_s * o_s, g_l * RMS(o_l)]  ([B, L, 2, H/P, d], fp16 on the library
     path: vdn_hybrid_attn_operand);
  4. one all-to-all turns that head shard back into a token shard holding every
     head: [B, L/P, 2, H, d];
  5. the rank projects its own tokens with the whole W_soft and W_lin
     (vdn_output_projection): its output rows [B, L/P, D_out].

Bytes each rank sends in step 4: B * L * 2 * (H/P) * d fp16 values, 1/P of
what a reduce-scatter of full-width float32 partial projections would move
(B * L * D_out * 4 bytes per rank), and no rank holds a [B, L, D_out] partial.

The per-head inputs (beta, alpha, text_k, text_v) are passed whole to every
rank (they are small) and sliced here.  The collectives are torch.distributed
calls (NCCL on GPUs, gloo on CPU).  ``operand`` and ``project`` default to the
library's two calls; the CPU tests pass float64 oracle versions.
"""
from __future__ import annotations

from typing import Callable, Optional


def _world(group):
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized():
        return 1, 0
    return dist.get_world_size(group), dist.get_rank(group)


def seq_to_heads(x, group=None):
    """[B, L/P, H, d] token shard -> [B, L, H/P, d] head shard (all-to-all).

    Rank r's shard holds tokens [r L/P, (r+1) L/P); the result holds heads
    [r H/P, (r+1) H/P) of every token."""
    import torch
    import torch.distributed as dist
    P, _ = _world(group)
    if P == 1:
        return x
    B, Ls, H, d = x.shape
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    # [P (destination rank), B, Ls, Hp, d]
    send = x.reshape(B, Ls, P, Hp, d).permute(2, 0, 1, 3, 4).contiguous()
    recv = torch.empty_like(send)  # [P (source rank), B, Ls, Hp, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3, 4).reshape(B, P * Ls, Hp, d)


def heads_to_seq(x, group=None):
    """[B, L, 2, H/P, d] operand of this rank's heads -> [B, L/P, 2, H, d], the
    operand of every head for this rank's tokens (all-to-all).  Heads keep
    their global order: rank r's heads are [r H/P, (r+1) H/P)."""
    import torch
    import torch.distributed as dist
    P, _ = _world(group)
    if P == 1:
        return x
    B, L, two, Hp, d = x.shape
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    Ls = L // P
    # [P (destination rank = token shard), B, Ls, 2, Hp, d]
    send = x.reshape(B, P, Ls, two, Hp, d).permute(1, 0, 2, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)  # [P (source rank = head block), B, Ls, 2, Hp, d]
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(B, Ls, two, P * Hp, d)


def head_slice(P: int, r: int, H: int):
    """Heads of rank r: [r H/P, (r+1) H/P)."""
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    return slice(r * Hp, (r + 1) * Hp)


def head_inputs(beta, alpha, text_k, text_v, hs):
    """The per-head inputs of heads `hs` (beta [B, H, ...], alpha [B, H, T, d],
    text_k / text_v [B, n_text, H, d])."""
    return (beta[:, hs].contiguous(), None if alpha is None else alpha[:, hs].contiguous(),
            None if text_k is None else text_k[:, :, hs].contiguous(),
            None if text_v is None else text_v[:, :, hs].contiguous())


def _library_operand(q, k, v, beta, text_k, text_v, gates, T, *, alpha=None, **kw):
    from . import hybrid_attn_operand
    return hybrid_attn_operand(q, k, v, beta, text_k, text_v, gates, T, alpha=alpha, **kw)


def _library_project(x, W_soft, W_lin, **kw):
    from . import make_params, output_projection
    B, Ls, _, H, d = x.shape
    p = make_params(B, H, 1, Ls, d, 0, "bf16", D_out=W_soft.shape[1],
                    out_dtype=kw.get("out_dtype", "f32"))
    return output_projection(x, W_soft, W_lin, p)


def ulysses_forward(q, k, v, beta, text_k, text_v, W_soft, W_lin, gates, T, *, alpha=None,
                    group=None, operand: Optional[Callable] = None,
                    project: Optional[Callable] = None, **kw):
    """Head-sharded forward; returns this rank's output rows [B, L/P, D_out].

    q, k, v: [B, L/P, H, d] (this rank's tokens); gates [2, B, L/P, H, d];
    beta [B, H, ...] and alpha [B, H, T, d] (or None), text_k / text_v
    [B, n_text, H, d], W_soft / W_lin [H*d, D_out]: whole, on every rank.
    ``operand(q, k, v, beta, text_k, text_v, gates, T, alpha=, **kw)`` returns
    [B, L, 2, h, d] for the h heads it is given; ``project(x, W_soft, W_lin)``
    returns [..., D_out]."""
    operand = operand or _library_operand
    project = project or _library_project
    P, r = _world(group)
    H = q.shape[2]
    hs = head_slice(P, r, H)
    qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
    gh = gates.new_empty((2,) + qh.shape) if P > 1 else gates
    if P > 1:
        for i in range(2):
            gh[i] = seq_to_heads(gates[i], group)
    b_h, a_h, tk_h, tv_h = head_inputs(beta, alpha, text_k, text_v, hs)
    x_heads = operand(qh, kh, vh, b_h, tk_h, tv_h, gh.contiguous(), T, alpha=a_h, **kw)
    x_tok = heads_to_seq(x_heads, group)
    return project(x_tok.contiguous(), W_soft, W_lin)
