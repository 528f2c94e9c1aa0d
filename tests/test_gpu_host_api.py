"""The host-buffer entry points (the end-to-end path of the bench): pinned host
inputs -> device -> forward -> host output must give exactly the device
forward's result, and report the bytes each step moves."""
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from synth import CONFIGS, make_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu


def _cfg(seed):
    return CONFIGS["small_bf16"].replace(H=2, T=12, N=64, n_text=16, seed=seed)


def _device_forward(inp, cfg):
    d = to_dev(inp)
    out = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                              d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"])
    torch.cuda.synchronize()
    return out.cpu()


def _pinned(inp):
    return {k: (v.pin_memory() if v is not None else None) for k, v in inp.items()}


def test_host_call_equals_device_forward_and_counts_bytes():
    cfg = _cfg(31)
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0))
    host = _pinned(inp)
    out_host, h2d, d2h = vdn.hybrid_attn_fwd_host(host, cfg.T)
    torch.cuda.synchronize()
    assert out_host.is_pinned()
    assert torch.equal(out_host, _device_forward(inp, cfg))
    want_h2d = sum(v.numel() * v.element_size() for n, v in inp.items()
                   if v is not None and n in vdn.INPUT_NAMES)
    assert h2d == want_h2d
    assert d2h == out_host.numel() * out_host.element_size()


def test_pipeline_alternating_inputs_matches_each_step():
    """Four pipelined steps over two different workloads (the two slots
    alternate): every step's output is exactly that workload's forward."""
    cfgs = [_cfg(41), _cfg(42)]
    inps = [make_inputs(c) for c in cfgs]
    hosts = [_pinned(i) for i in inps]
    pipe = vdn.HostPipeline(hosts[0], cfgs[0].T)
    outs = []
    for step in range(4):
        o = torch.empty(1, cfgs[0].L, cfgs[0].D, dtype=torch.float32).pin_memory()
        pipe.submit(hosts[step % 2], o)
        outs.append(o)
    pipe.synchronize()
    want = [_device_forward(inps[i], cfgs[i]) for i in range(2)]
    for step, o in enumerate(outs):
        assert torch.equal(o, want[step % 2]), step
    assert not torch.equal(want[0], want[1])
