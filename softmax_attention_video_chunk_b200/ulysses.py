"""Head-sharded (Ulysses) VDN hybrid attention forward over P ranks.

"Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation", implementation section: for multi-GPU inference VDA is sharded by
attention head, following Ulysses sequence parallelism.  Every step of the
forward is independent per head except the output projection, which
contracts over heads.  So with P ranks:

  1. each rank holds a contiguous shard of L/P tokens of q, k, v and the gates;
  2. one all-to-all per tensor turns token shards into head shards: every rank
     then holds all L tokens of H/P heads;
  3. the rank runs the whole forward on its heads with its H/P * d rows of
     W_soft and W_lin, which gives a partial sum of the projection;
  4. one reduce-scatter over the token dimension adds the P partial sums and
     hands each rank the output rows of its own token shard.

The per-head inputs (beta, alpha, text_k, text_v) are passed whole to every
rank (they are small) and sliced here.  The collectives are torch.distributed
calls (NCCL on GPUs, gloo on CPU).  The per-rank forward is
softmax_attention_video_chunk_b200.hybrid_attn_fwd unless ``fwd`` is given.
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


def partial_to_seq(y, group=None):
    """[B, L, D_out] partial sums (one per rank) -> [B, L/P, D_out], the sum
    over ranks of this rank's token shard (reduce-scatter)."""
    import torch
    import torch.distributed as dist
    P, _ = _world(group)
    if P == 1:
        return y
    B, L, Do = y.shape
    if L % P:
        raise ValueError(f"{L} tokens do not split over {P} ranks")
    Ls = L // P
    # [P * B, Ls, Do]: rank r's rows are block r along dim 0
    send = y.reshape(B, P, Ls, Do).permute(1, 0, 2, 3).reshape(P * B, Ls, Do).contiguous()
    recv = torch.empty((B, Ls, Do), dtype=y.dtype, device=y.device)
    dist.reduce_scatter_tensor(recv, send, group=group)
    return recv


def head_slice(P: int, r: int, H: int):
    """Heads of rank r: [r H/P, (r+1) H/P)."""
    if H % P:
        raise ValueError(f"{H} heads do not split over {P} ranks")
    Hp = H // P
    return slice(r * Hp, (r + 1) * Hp)


def ulysses_forward(q, k, v, beta, text_k, text_v, W_soft, W_lin, gates, T, *, alpha=None,
                    group=None, fwd: Optional[Callable] = None, **kw):
    """Head-sharded forward; returns this rank's output rows [B, L/P, D_out].

    q, k, v: [B, L/P, H, d] (this rank's tokens); gates [2, B, L/P, H, d];
    beta [B, H, ...] and alpha [B, H, T, d] (or None), text_k / text_v
    [B, n_text, H, d], W_soft / W_lin [H*d, D_out]: whole, on every rank.
    ``fwd`` has the signature of hybrid_attn_fwd and returns [B, L, D_out]."""
    if fwd is None:
        from . import hybrid_attn_fwd as fwd
    P, r = _world(group)
    H, d = q.shape[2], q.shape[3]
    hs = head_slice(P, r, H)
    qh, kh, vh = (seq_to_heads(x, group) for x in (q, k, v))
    gh = gates.new_empty((2,) + qh.shape) if P > 1 else gates
    if P > 1:
        for i in range(2):
            gh[i] = seq_to_heads(gates[i], group)
    rows = slice(hs.start * d, hs.stop * d)
    part = fwd(qh, kh, vh, beta[:, hs].contiguous(),
               None if text_k is None else text_k[:, :, hs].contiguous(),
               None if text_v is None else text_v[:, :, hs].contiguous(),
               W_soft[rows].contiguous(), W_lin[rows].contiguous(), gh.contiguous(), T,
               alpha=None if alpha is None else alpha[:, hs].contiguous(), **kw)
    return partial_to_seq(part, group)
