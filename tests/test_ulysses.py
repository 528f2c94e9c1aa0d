"""Head-sharded (Ulysses) forward on CPU ranks with the gloo backend: the
token -> head all-to-all, the per-rank projection operand of its heads, the
head -> token all-to-all of that operand and the token-sharded projection,
with float64 oracle versions of the two per-rank calls, must reproduce the
unsharded forward."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _cfg(H=4):
    from synth import CONFIGS
    return CONFIGS["tiny_f32"].replace(H=H)


def _oracle_operand(cfg):
    """x [B, L, 2, h, d] = [g_s * o_s, g_l * RMS(o_l)] of the h heads given,
    from the float64 oracle's two branches."""
    from oracle import vdn_oracle as O

    def operand(q, k, v, beta, text_k, text_v, gates, T, alpha=None, **kw):
        _, o_s, o_l = O.hybrid_forward(
            dict(q=q, k=k, v=v, beta=beta, alpha=alpha, text_k=text_k, text_v=text_v,
                 W_soft=torch.zeros(q.shape[2] * q.shape[3], 8, dtype=q.dtype),
                 W_lin=torch.zeros(q.shape[2] * q.shape[3], 8, dtype=q.dtype), gates=gates),
            T, cfg.N, cfg.chunk, cfg.window_radius, **kw)
        g = O._to_np(gates)
        xs = g[0] * o_s
        xl = g[1] * O.rms_norm(o_l)
        return torch.from_numpy(np.stack([xs, xl], axis=2))
    return operand


def _oracle_project(x, W_soft, W_lin):
    B, Ls, _, H, d = x.shape
    xs = x[:, :, 0].reshape(B, Ls, H * d).double()
    xl = x[:, :, 1].reshape(B, Ls, H * d).double()
    return xs @ W_soft.double() + xl @ W_lin.double()


def _oracle_fwd(cfg):
    from oracle import vdn_oracle as O

    def fwd(q, k, v, beta, text_k, text_v, W_soft, W_lin, gates, T, alpha=None, **kw):
        inp = dict(q=q, k=k, v=v, beta=beta, alpha=alpha, text_k=text_k, text_v=text_v,
                   W_soft=W_soft, W_lin=W_lin, gates=gates)
        out, _, _ = O.hybrid_forward(inp, T, cfg.N, cfg.chunk, cfg.window_radius, **kw)
        return torch.from_numpy(out)
    return fwd


def _rank(rank, world, port, out, alpha, gates="const", H=4):
    import datetime

    import torch.distributed as dist

    from softmax_attention_video_chunk_b200 import ulysses
    from synth import make_inputs
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        cfg = _cfg(H)
        inp = make_inputs(cfg, alpha_range=(0.8, 1.0) if alpha else None, gates=gates)
        Ls = cfg.L // world
        tok = slice(rank * Ls, (rank + 1) * Ls)
        y = ulysses.ulysses_forward(
            inp["q"][:, tok], inp["k"][:, tok], inp["v"][:, tok], inp["beta"], inp["text_k"],
            inp["text_v"], inp["W_soft"], inp["W_lin"], inp["gates"][:, :, tok], cfg.T,
            alpha=inp["alpha"], operand=_oracle_operand(cfg), project=_oracle_project)
        parts = [torch.empty_like(y) for _ in range(world)]
        dist.all_gather(parts, y)
        if rank == 0:
            out["y"] = torch.cat(parts, dim=1).numpy()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,alpha,gates,H", [(2, False, "const", 4), (4, True, "random", 4),
                                                 (3, True, "random", 6)])
def test_head_sharded_forward_equals_unsharded(world, alpha, gates, H):
    from synth import make_inputs
    cfg = _cfg(H)
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, _free_port(), out, alpha, gates, H), nprocs=world,
                 join=True)
        got = out["y"]
    inp = make_inputs(cfg, alpha_range=(0.8, 1.0) if alpha else None, gates=gates)
    want = _oracle_fwd(cfg)(inp["q"], inp["k"], inp["v"], inp["beta"], inp["text_k"],
                            inp["text_v"], inp["W_soft"], inp["W_lin"], inp["gates"], cfg.T,
                            alpha=inp["alpha"]).numpy()
    rms = np.sqrt(np.mean(want ** 2))
    assert got.shape == want.shape
    assert np.max(np.abs(got - want)) <= 1e-12 * rms


def test_one_rank_is_the_plain_forward():
    from softmax_attention_video_chunk_b200 import ulysses
    from synth import make_inputs
    cfg = _cfg()
    inp = make_inputs(cfg, gates="random")
    fwd = _oracle_fwd(cfg)
    args = (inp["q"], inp["k"], inp["v"], inp["beta"], inp["text_k"], inp["text_v"],
            inp["W_soft"], inp["W_lin"], inp["gates"], cfg.T)
    got = ulysses.ulysses_forward(*args, operand=_oracle_operand(cfg),
                                  project=_oracle_project).numpy()
    want = fwd(*args).numpy()
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())


def test_heads_to_seq_layout_on_one_process():
    """The reassembly order of heads_to_seq: simulated with the all-to-all
    replaced by the list of every rank's send buffer."""
    from softmax_attention_video_chunk_b200 import ulysses
    B, L, H, d, P = 2, 12, 6, 3, 3
    full = torch.arange(B * L * 2 * H * d, dtype=torch.float64).reshape(B, L, 2, H, d)
    Ls, Hp = L // P, H // P
    # rank r's operand covers heads hs(r) for every token
    per_rank = [full[:, :, :, ulysses.head_slice(P, r, H)] for r in range(P)]
    for dst in range(P):
        # what rank dst receives from rank src: tokens of dst, heads of src
        recv = torch.stack([per_rank[src].reshape(B, P, Ls, 2, Hp, d)[:, dst]
                            for src in range(P)])
        got = recv.permute(1, 2, 3, 0, 4, 5).reshape(B, Ls, 2, P * Hp, d)
        assert torch.equal(got, full[:, dst * Ls:(dst + 1) * Ls])


def test_head_split_must_divide():
    from softmax_attention_video_chunk_b200 import ulysses
    with pytest.raises(ValueError):
        ulysses.head_slice(3, 0, 4)
    assert ulysses.head_slice(4, 3, 8) == slice(6, 8)
