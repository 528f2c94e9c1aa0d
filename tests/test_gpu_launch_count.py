"""The kernel count the library reports for a forward (vdn_forward_launches,
which bench.py multiplies into gpu_launches) against the kernels a profiler
sees one forward launch."""
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from synth import CONFIGS, make_inputs

from _parity import to_dev

pytestmark = pytest.mark.gpu

# kernels of this library (device function names as the profiler reports them)
OURS = ("vda_", "attn_", "readout_", "convert_", "gemm_tc", "mx_", "proj_simt", "rms_inv",
        "combine_splits", "prep_")


def _kernels_of_one_forward(d, cfg, p):
    ws = vdn.alloc_workspace(p)
    out = torch.empty(cfg.B, cfg.L, p.D_out, dtype=torch.float32, device="cuda")
    run = lambda: vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"],
                                      d["text_v"], d["W_soft"], d["W_lin"], d["gates"], cfg.T,
                                      alpha=d["alpha"], out=out, workspace=ws, params=p)
    run()
    torch.cuda.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        run()
        torch.cuda.synchronize()
    names = [e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA]
    return [n for n in names if any(k in n for k in OURS)]


CASES = [
    ("frames", dict(T=20, N=64, H=2, d=128, n_text=16), vdn.FLAG_SCAN_FRAMES),
    ("chunks", dict(T=20, N=64, H=2, d=128, n_text=16), vdn.FLAG_SCAN_CHUNKS),
    ("mxfp8", dict(T=12, N=64, H=2, d=64, n_text=16), vdn.FLAG_PROJ_MXFP8),
    ("text_softmax", dict(T=12, N=64, H=2, d=64, n_text=16), vdn.FLAG_TEXT_SOFTMAX),
    ("simt", dict(T=12, N=64, H=2, d=64, n_text=16), vdn.FLAG_SIMT),
]


@pytest.mark.parametrize("name,over,flags", CASES, ids=[c[0] for c in CASES])
def test_reported_launch_count_matches_the_profiler(name, over, flags):
    cfg = CONFIGS["small_bf16"].replace(seed=5).replace(**over)
    d = to_dev(make_inputs(cfg))
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"])
    p.flags |= flags
    ours = _kernels_of_one_forward(d, cfg, p)
    if not ours:
        pytest.skip("the profiler recorded no kernel activity on this box")
    assert len(ours) == vdn.forward_launches(p), ours
