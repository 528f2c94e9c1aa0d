"""The forward inside a CUDA graph: the library enqueues only kernels and a
memset on the caller's stream and allocates nothing, so one forward can be
captured once and replayed; a replay equals a direct call bit for bit, and
follows new inputs copied into the captured buffers."""
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from synth import CONFIGS, make_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu

KEYS = ("q", "k", "v", "beta", "text_k", "text_v", "W_soft", "W_lin", "gates", "alpha")


@pytest.mark.parametrize("mxfp8", [False, True], ids=["fp16_projection", "mxfp8_projection"])
def test_forward_replays_from_a_cuda_graph(mxfp8):
    cfg = CONFIGS["small_bf16"].replace(H=2, T=13, N=72, n_text=16, seed=9)
    d = to_dev(make_inputs(cfg, gates="random", alpha_range=(0.9, 1.0)))
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], proj_mxfp8=mxfp8)
    ws = vdn.alloc_workspace(p)
    out = torch.empty(cfg.B, cfg.L, p.D_out, dtype=torch.float32, device="cuda")

    def run(o):
        return vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                   d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"],
                                   out=o, workspace=ws, params=p)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up off the default stream, as capture wants
        run(out)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    want = out.clone()

    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run(out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, want)
    assert vdn.device_status(p, ws) == 0

    # new inputs in the same buffers: the replay computes them
    d2 = to_dev(make_inputs(cfg.replace(seed=10), gates="random", alpha_range=(0.9, 1.0)))
    for key in KEYS:
        d[key].copy_(d2[key])
    g.replay()
    direct = torch.empty_like(out)
    run(direct)
    torch.cuda.synchronize()
    assert torch.equal(out, direct)
    assert not torch.equal(out, want)
