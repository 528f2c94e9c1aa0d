"""The boundary-state entry point that allocates nothing.

vdn_vda_boundary_states_noalloc serves callers that cannot allocate device
memory (a host framework that owns every allocation, a plugin without an
allocator, code that must not call cudaMalloc while a stream is captured): it
runs the same kernels as vdn_vda_boundary_states with its scratch in a static
device array of the library.  This file is collected last so that a run that
stops at the first failure has run every other test first.
"""
import ctypes

import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from synth import CONFIGS, make_inputs
from tests._parity import rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,over,tol", [
    ("tiny_f32", {}, 1e-5),
    ("small_bf16", dict(T=16, N=96, H=4), 1e-4),
    ("d128_bf16", dict(T=12, N=136, H=2, d=128), 1e-4),
])
def test_noalloc_matches_workspace_entry_twice(cuda_ok, name, over, tol):
    base = CONFIGS["tiny_f32"] if name == "tiny_f32" else CONFIGS["small_bf16"].replace(seed=11)
    cfg = base.replace(**over)
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0))
    d = to_dev(inp)
    F_ref, G_ref = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                           cfg.T, alpha=d["alpha"], chunk=cfg.chunk)
    torch.cuda.synchronize()
    for _ in range(2):  # the static scratch keeps the previous call's contents
        F, G = vdn.vda_boundary_states_noalloc(d["k"], d["v"], d["beta"], d["text_k"],
                                               d["text_v"], cfg.T, alpha=d["alpha"],
                                               chunk=cfg.chunk)
        torch.cuda.synchronize()
        assert rel_err(F.double().cpu(), F_ref.double().cpu()) <= tol
        assert rel_err(G.double().cpu(), G_ref.double().cpu()) <= tol


def test_noalloc_rejects_problems_beyond_the_static_scratch(cuda_ok):
    cfg = CONFIGS["768p_bf16"]
    p = vdn.make_params(cfg.B, cfg.H, cfg.T, cfg.N, cfg.d, cfg.n_text, "bf16")
    dummy = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ptr = dummy.data_ptr()
    rc = vdn.lib().vdn_vda_boundary_states_noalloc(ctypes.byref(p), ptr, ptr, ptr, None, ptr,
                                                   ptr, ptr, ptr, None)
    assert vdn.STATUS[rc] == "VDN_ERR_WORKSPACE"
