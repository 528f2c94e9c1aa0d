"""Parity of the CUDA path (through the C ABI) against the CPU oracle.

Small workloads are compared element by element on every output; the
full-size workloads (768p, long clip, batched clips) are run in the launch
configuration the benchmark times and compared on seeded samples of query
rows that the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from oracle import vdn_oracle as O
from synth import CONFIGS, make_inputs, make_text_queries, sample_rows
from tests._parity import TOL_OUT, gpu_rows, oracle_forward, rel_err, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    return vdn.lib()


def _fwd(d, cfg, **kw):
    return vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                               d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"],
                               chunk=cfg.chunk, window_radius=cfg.window_radius, **kw)


def _branches(d, cfg, **kw):
    return vdn.hybrid_attn_branches(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                    cfg.T, alpha=d["alpha"], chunk=cfg.chunk,
                                    window_radius=cfg.window_radius, **kw)


# ----------------------------------------------------------------------------
# full comparison on small workloads
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("gates", ["const", "random"])
@pytest.mark.parametrize("simt", [False, True])
def test_tiny_f32_full(simt, gates):
    cfg = CONFIGS["tiny_f32"]
    inp = make_inputs(cfg, gates=gates)
    d = to_dev(inp)
    out = _fwd(d, cfg, simt=simt)
    o_s, o_l = _branches(d, cfg, simt=simt)
    F, G = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"], cfg.T,
                                   chunk=cfg.chunk)
    torch.cuda.synchronize()
    want, ws_, wl_ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    assert rel_err(out.double().cpu(), want) <= TOL_OUT["f32"]
    assert rel_err(o_s.double().cpu(), ws_) <= 1e-5
    assert rel_err(o_l.double().cpu(), wl_) <= 1e-5
    Fo, Go = O.boundary_states(inp["k"], inp["v"], inp["beta"], inp["text_k"], inp["text_v"],
                               cfg.T, cfg.N, cfg.chunk)
    assert rel_err(F.double().cpu(), Fo) <= 1e-5
    assert rel_err(G.double().cpu(), Go) <= 1e-5


@pytest.mark.parametrize("gates", ["const", "random"])
@pytest.mark.parametrize("simt", [False, True])
def test_small_bf16_full(simt, gates):
    cfg = CONFIGS["small_bf16"]
    inp = make_inputs(cfg, gates=gates)
    d = to_dev(inp)
    out = _fwd(d, cfg, simt=simt)
    o_s, o_l = _branches(d, cfg, simt=simt)
    torch.cuda.synchronize()
    want, ws_, wl_ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    e_out = rel_err(out.double().cpu(), want)
    e_s = rel_err(o_s.double().cpu(), ws_)
    e_l = rel_err(o_l.double().cpu(), wl_)
    print(f"small_bf16 simt={simt} gates={gates}: out {e_out:.2e} o_soft {e_s:.2e} "
          f"o_lin {e_l:.2e}")
    assert e_out <= TOL_OUT["bf16"]
    assert e_s <= 2e-3
    assert e_l <= 1e-4


# (name, overrides, make_inputs kwargs, extra fwd kwargs)
EDGE = [
    ("T1", dict(T=1, N=40), {}, {}),
    ("T2", dict(T=2, N=24), {}, {}),
    ("T7_N5_partial_chunk", dict(T=7, N=5), {}, {}),
    ("T12_N200_c3_r2", dict(T=12, N=200, chunk=3, window_radius=2), {}, {}),
    ("T9_N130_c1_r0", dict(T=9, N=130, chunk=1, window_radius=0), {}, {}),
    ("T23_N96_c4", dict(T=23, N=96, chunk=4), {}, {}),
    ("no_text", dict(T=16, N=64, n_text=0), {}, {}),
    ("decay_alpha", dict(T=18, N=48), dict(alpha_range=(0.85, 1.0)), {}),
    ("text_full", dict(T=16, N=64), {}, dict(text_full=True)),
    ("text_softmax", dict(T=13, N=72, n_text=200), {}, dict(text_softmax=True)),
    ("text_softmax_d128", dict(T=9, N=130, d=128, H=2, n_text=77), {}, dict(text_softmax=True)),
    ("beta_per_token", dict(T=14, N=72), dict(beta_per_token=True, alpha_range=(0.9, 1.0)),
     dict(beta_per_token=True)),
    ("beta_per_token_d128_N5", dict(T=8, N=5, d=128, H=2, n_text=37),
     dict(beta_per_token=True), dict(beta_per_token=True)),
    ("d128", dict(T=11, N=136, d=128, H=2), {}, {}),
    ("d32", dict(T=11, N=40, d=32, H=3), {}, {}),
    # independent per-element gates of the two branches (sigmoid(N(0,1)))
    ("gates_d128", dict(T=11, N=136, d=128, H=2), dict(gates="random"), {}),
    ("gates_ragged_N", dict(T=13, N=37, d=64, H=3), dict(gates="random"), {}),
    ("gates_text_softmax_d128", dict(T=9, N=130, d=128, H=2, n_text=77),
     dict(gates="random", alpha_range=(0.9, 1.0)), dict(text_softmax=True)),
]


def _edge_cfg(over):
    base = CONFIGS["small_bf16"].replace(H=3, T=15, N=32, n_text=16, seed=7)
    return base.replace(**over)


def _oracle_inputs_nontext(inp, cfg):
    if cfg.n_text == 0:
        B, H, d = cfg.B, cfg.H, cfg.d
        inp = dict(inp)
        inp["text_k"] = torch.zeros(B, 0, H, d, dtype=inp["q"].dtype)
        inp["text_v"] = torch.zeros(B, 0, H, d, dtype=inp["q"].dtype)
    return inp


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("name,over,mk,kw", EDGE, ids=[e[0] for e in EDGE])
def test_edge_cases(name, over, mk, kw, simt):
    cfg = _edge_cfg(over)
    inp = make_inputs(cfg, **mk)
    inp = _oracle_inputs_nontext(inp, cfg)
    d = to_dev(inp)
    if cfg.n_text == 0:
        d["text_k"] = d["text_v"] = None
    out = _fwd(d, cfg, simt=simt, **kw)
    o_s, o_l = _branches(d, cfg, simt=simt, **kw)
    torch.cuda.synchronize()
    want, ws_, wl_ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius,
                                    text_full=kw.get("text_full", False),
                                    text_softmax=kw.get("text_softmax", False),
                                    beta_per_token=kw.get("beta_per_token", False))
    e_out = rel_err(out.double().cpu(), want)
    e_s = rel_err(o_s.double().cpu(), ws_)
    e_l = rel_err(o_l.double().cpu(), wl_)
    print(f"{name} simt={simt}: out {e_out:.2e} o_soft {e_s:.2e} o_lin {e_l:.2e}")
    assert e_out <= TOL_OUT["bf16"]
    assert e_s <= 2e-3
    assert e_l <= 1e-4


def _frozen_inputs(cfg):
    """Inputs for the frozen-state comparison rule: keys scaled by 1/sqrt(N),
    one reading of SANA-WM's frame-size key scaling, so that the frame
    transitions I - A stay near the unit ball over the clip."""
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0))
    inp["k"] = (inp["k"].float() / np.sqrt(cfg.N)).to(inp["k"].dtype)
    return inp


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("over", [dict(T=14, N=72), dict(T=9, N=130, d=128, H=2, n_text=37)],
                         ids=["d64", "d128"])
def test_frozen_state_rule(over, simt):
    """Comparison mode: every frame update follows the frozen-state rule."""
    cfg = _edge_cfg(over)
    inp = _frozen_inputs(cfg)
    d = to_dev(inp)
    out = _fwd(d, cfg, simt=simt, frozen_state=True)
    _, o_l = _branches(d, cfg, simt=simt, frozen_state=True, want_soft=False)
    torch.cuda.synchronize()
    want, _, wl_ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, frozen=True)
    e_out, e_l = rel_err(out.double().cpu(), want), rel_err(o_l.double().cpu(), wl_)
    # and it is a different rule: VDA's o_lin differs from it
    _, vda_l = _branches(d, cfg, simt=simt, want_soft=False)
    torch.cuda.synchronize()
    gap = rel_err(vda_l.double().cpu(), wl_)
    print(f"frozen {over} simt={simt}: out {e_out:.2e} o_lin {e_l:.2e} (VDA gap {gap:.2e})")
    assert e_out <= TOL_OUT["bf16"]
    assert e_l <= 1e-4
    assert gap > 1e-2


@pytest.mark.parametrize("over", [dict(T=23, N=96, d=64, H=2), dict(T=12, N=136, d=128, H=2)],
                         ids=["d64", "d128"])
def test_boundary_states_frozen(over):
    cfg = _edge_cfg(over)
    inp = _frozen_inputs(cfg)
    d = to_dev(inp)
    F, G = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"], cfg.T,
                                   alpha=d["alpha"], chunk=cfg.chunk, frozen_state=True)
    torch.cuda.synchronize()
    Fo, Go = O.boundary_states(inp["k"], inp["v"], inp["beta"], inp["text_k"], inp["text_v"],
                               cfg.T, cfg.N, cfg.chunk, alpha=inp["alpha"], frozen=True)
    eF, eG = rel_err(F.double().cpu(), Fo), rel_err(G.double().cpu(), Go)
    print(f"frozen states {over}: F {eF:.2e} G {eG:.2e}")
    assert eF <= 1e-4 and eG <= 1e-4


@pytest.mark.parametrize("simt", [False, True])
@pytest.mark.parametrize("over", [dict(T=13, N=72, n_text=200), dict(T=9, N=130, d=128, H=2,
                                  n_text=300), dict(T=5, N=16, n_text=3)],
                         ids=["d64_nt200", "d128_nt300", "nt3"])
def test_text_query_rows(over, simt):
    """Text tokens as queries, dense over every video key and text key."""
    cfg = _edge_cfg(over)
    inp = make_inputs(cfg)
    tq = make_text_queries(cfg)
    d = to_dev(inp)
    o = vdn.text_query_attn(tq.cuda(), d["k"], d["v"], d["text_k"], d["text_v"], cfg.T, simt=simt)
    torch.cuda.synchronize()
    want = O.text_query_branch(O._to_np(tq), O._to_np(inp["k"]), O._to_np(inp["v"]),
                               O._to_np(inp["text_k"]), O._to_np(inp["text_v"]))
    e = rel_err(o.double().cpu(), want)
    print(f"text rows {over} simt={simt}: {e:.2e}")
    # tensor cores: P rounded once to fp16 (as for the video rows); FP32 kernel: exact
    assert e <= (1e-5 if simt else 2e-3)


def test_text_query_rows_768p_sampled():
    """768p: 512 text queries over 115200 video keys + 512 text keys; sampled rows."""
    cfg = CONFIGS["768p_bf16"]
    inp = make_inputs(cfg)
    tq = make_text_queries(cfg)
    d = to_dev(inp)
    o = vdn.text_query_attn(tq.cuda(), d["k"], d["v"], d["text_k"], d["text_v"], cfg.T)
    torch.cuda.synchronize()
    rows = np.array([0, 1, 137, 255, 256, 400, 510, 511])
    got = o[:, rows].double().cpu().numpy()
    del d, o
    torch.cuda.empty_cache()
    want = O.text_query_branch(O._to_np(tq), O._to_np(inp["k"]), O._to_np(inp["v"]),
                               O._to_np(inp["text_k"]), O._to_np(inp["text_v"]), rows=rows)
    e = rel_err(got, want)
    print(f"768p text rows ({len(rows)} rows): {e:.2e}")
    assert e <= 2e-3


@pytest.mark.parametrize("P", [2, 4])
def test_head_shards_through_the_library(P):
    """The head-sharded forward on one GPU: P head shards run one after another
    through vdn_hybrid_attn_operand (each with its heads' inputs), their
    operands are put together as the head -> token all-to-all would, and
    vdn_output_projection projects every token shard with the whole W.  Heads
    are independent up to the projection, so this equals the plain forward bit
    for bit, and the oracle within the output tolerance."""
    from softmax_attention_video_chunk_b200 import ulysses
    cfg = _edge_cfg(dict(T=11, N=96, d=128, H=4, n_text=24))
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0), gates="random")
    d = to_dev(inp)
    H = cfg.H
    x = torch.empty(cfg.B, cfg.L, 2, H, cfg.d, dtype=torch.float16, device="cuda")
    for r in range(P):
        hs = ulysses.head_slice(P, r, H)
        b_h, a_h, tk_h, tv_h = ulysses.head_inputs(d["beta"], d["alpha"], d["text_k"],
                                                    d["text_v"], hs)
        xr = vdn.hybrid_attn_operand(d["q"][:, :, hs].contiguous(), d["k"][:, :, hs].contiguous(),
                                     d["v"][:, :, hs].contiguous(), b_h, tk_h, tv_h,
                                     d["gates"][:, :, :, hs].contiguous(), cfg.T, alpha=a_h)
        x[:, :, :, hs] = xr
    # token-sharded projection: rank r projects tokens [r L/P, (r+1) L/P)
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"])
    Ls = cfg.L // P
    out = torch.cat([vdn.output_projection(x[:, r * Ls:(r + 1) * Ls].contiguous(), d["W_soft"],
                                           d["W_lin"], p) for r in range(P)], dim=1)
    plain = _fwd(d, cfg)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    e = rel_err(out.double().cpu(), want)
    print(f"head shards P={P}: {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_operand_then_projection_is_the_forward():
    """vdn_hybrid_attn_operand followed by vdn_output_projection is
    vdn_hybrid_attn_fwd, bit for bit (text keys in the Softmax, per-token
    write gates, random gates)."""
    cfg = _edge_cfg(dict(T=9, N=130, d=128, H=2, n_text=77))
    inp = make_inputs(cfg, gates="random", beta_per_token=True)
    d = to_dev(inp)
    kw = dict(text_softmax=True, beta_per_token=True)
    x = vdn.hybrid_attn_operand(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                d["gates"], cfg.T, **kw)
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], **kw)
    out = vdn.output_projection(x, d["W_soft"], d["W_lin"], p)
    plain = _fwd(d, cfg, **kw)
    torch.cuda.synchronize()
    assert torch.equal(out, plain)
    # the operand itself: x[..., 0] = g_s o_s, x[..., 1] = g_l RMS(o_l) (fp16)
    o_s, o_l = _branches(d, cfg, **kw)
    torch.cuda.synchronize()
    g = d["gates"].float()
    xs = (g[0] * o_s).to(torch.float16)
    rms = o_l.pow(2).mean(dim=-1, keepdim=True).add(1e-6).rsqrt()
    xl = (g[1] * o_l * rms).to(torch.float16)
    for got, ref in ((x[:, :, 0], xs), (x[:, :, 1], xl)):
        err = (got.float() - ref.float()).abs().max() / ref.float().pow(2).mean().sqrt()
        assert float(err) <= 4e-3, float(err)


@pytest.mark.parametrize("simt", [False, True])
def test_poisoned_workspace_is_never_read_before_written(simt):
    """Every byte of scratch the path reads is written first by the same call:
    a workspace filled with NaN bytes (0xFF) gives bit-identical, finite
    results to a zero-filled one (forward with text keys and per-token gates,
    the two branches, the boundary states and the text rows)."""
    cfg = _edge_cfg(dict(T=13, N=72, n_text=40))
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0), beta_per_token=True)
    d = to_dev(inp)
    tq = make_text_queries(cfg).cuda()
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], text_softmax=True,
                       beta_per_token=True, simt=simt)

    def run(fill):
        ws = vdn.alloc_workspace(p)
        ws.fill_(fill)
        out = _fwd(d, cfg, params=p, workspace=ws)
        ws.fill_(fill)
        o_s, o_l = vdn.hybrid_attn_branches(d["q"], d["k"], d["v"], d["beta"], d["text_k"],
                                            d["text_v"], cfg.T, alpha=d["alpha"], workspace=ws,
                                            params=p)
        ws.fill_(fill)
        F, G = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"], cfg.T,
                                       alpha=d["alpha"], workspace=ws, params=p)
        ws.fill_(fill)
        ot = vdn.text_query_attn(tq, d["k"], d["v"], d["text_k"], d["text_v"], cfg.T,
                                 workspace=ws, params=p)
        torch.cuda.synchronize()
        assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_OK"
        return [out, o_s, o_l, F, G, ot]

    clean, poisoned = run(0), run(255)
    for a, b in zip(clean, poisoned):
        assert torch.isfinite(b).all()
        assert torch.equal(a, b)


def test_wide_scores_rescale_path():
    """Scores spanning many octaves (q scaled up): the running-max rescale of
    the tensor-core kernel is exercised."""
    cfg = _edge_cfg(dict(T=12, N=96, d=64))
    inp = make_inputs(cfg)
    inp["q"] = (inp["q"].float() * 40.0).to(torch.bfloat16)
    d = to_dev(inp)
    o_s, _ = _branches(d, cfg, want_lin=False)
    torch.cuda.synchronize()
    v = O._to_np(inp["v"])
    ws_ = O.softmax_branch(O._to_np(inp["q"]), O._to_np(inp["k"]), v, cfg.T,
                           cfg.N, cfg.chunk, cfg.window_radius)
    # P is rounded once to fp16 (unit roundoff u = 2^-11) before P V, so
    # |o - o_exact| <= u * sum_j w_j |v_j| <= u * max|v| (weights w sum to 1);
    # FP32 accumulation adds far less.
    err = np.max(np.abs(o_s.double().cpu().numpy() - ws_))
    print(f"wide scores: max|err| {err:.3e}, bound {2.0 ** -11 * np.abs(v).max():.3e}")
    assert err <= 2.0 ** -11 * np.abs(v).max()


def test_out_bf16():
    cfg = _edge_cfg(dict(T=14, N=64))
    inp = make_inputs(cfg)
    d = to_dev(inp)
    out = _fwd(d, cfg, out_dtype="bf16")
    torch.cuda.synchronize()
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    # one bf16 rounding of the output on top of the fp32 result
    want_r = torch.from_numpy(want).to(torch.bfloat16).double().numpy()
    assert out.dtype == torch.bfloat16
    err = np.abs(out.double().cpu().numpy() - want_r)
    ulp = np.abs(want_r) * 2.0 ** -7
    assert np.all(err <= ulp + 2e-3 * np.sqrt(np.mean(want ** 2)))


def test_device_status_ok_and_range():
    cfg = _edge_cfg(dict(T=10, N=32))
    inp = make_inputs(cfg)
    d = to_dev(inp)
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"])
    ws = vdn.alloc_workspace(p)
    _fwd(d, cfg, params=p, workspace=ws)
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_OK"
    d["v"] = d["v"] * 0 + 1e5  # beyond the fp16 range of the V operand
    _fwd(d, cfg, params=p, workspace=ws)
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_ERR_RANGE"
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_OK"  # cleared


def test_bounded_wait_expires_into_status():
    """A wait that nothing satisfies ends at its limit with VDN_ERR_TIMEOUT in
    the status word (no hang, no fault), and the context stays usable: the
    same workspace then runs a forward to parity."""
    import time
    cfg = _edge_cfg(dict(T=10, N=32))
    inp = make_inputs(cfg)
    d = to_dev(inp)
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"])
    ws = vdn.alloc_workspace(p)
    assert vdn.STATUS[vdn.selftest_bounded_wait(ws, 50)] == "VDN_ERR_INVALID_ARG"
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    assert vdn.STATUS[vdn.selftest_bounded_wait(ws, 20000)] == "VDN_OK"
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_ERR_TIMEOUT"
    dt = time.perf_counter() - t0
    assert 0.015 <= dt < 1.0, dt  # expired at its 20 ms limit, ended well before 2x + slack
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_OK"  # cleared
    out = _fwd(d, cfg, params=p, workspace=ws)
    torch.cuda.synchronize()
    assert vdn.STATUS[vdn.device_status(p, ws)] == "VDN_OK"
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    assert rel_err(out.double().cpu().numpy(), want) <= TOL_OUT["bf16"]


# ----------------------------------------------------------------------------
# full-size workloads, sampled rows
# ----------------------------------------------------------------------------

def _sampled(cfg, rows, bsel, chunk=None, alpha_range=None, gates="const", **kw):
    inp = make_inputs(cfg, alpha_range=alpha_range, gates=gates)
    d = to_dev(inp)
    c = cfg.chunk if chunk is None else chunk
    out = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                              d["W_soft"], d["W_lin"], d["gates"], cfg.T, chunk=c,
                              alpha=d["alpha"], **kw)
    torch.cuda.synchronize()
    got = gpu_rows(out, rows, bsel)
    del d, out
    torch.cuda.empty_cache()
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, c, cfg.window_radius, rows=rows, bsel=bsel)
    return rel_err(got, want)


def test_768p_sampled():
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=3)
    e = _sampled(cfg, rows, None)
    print(f"768p sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_768p_random_gates_sampled():
    """The 768p workload with independent per-element gates g_s, g_l ~
    sigmoid(N(0, 1)): the fused epilogues of the Softmax and readout kernels
    read their own gate at the (token, head, channel) of each output."""
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 1, 7, 13, 14])
    e = _sampled(cfg, rows, None, gates="random")
    print(f"768p random gates sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_batched_random_gates_sampled():
    """Batched clips with random per-element gates: gate rows of batch items
    other than the first are indexed with the batch offset."""
    cfg = CONFIGS["batched_bf16"]
    rows = sample_rows(cfg, per_frame=2)
    e = _sampled(cfg, rows, [5, 15], gates="random")
    print(f"batched random gates sampled: {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_768p_channel_decay_sampled():
    """The 768p workload with a channel-wise decay gate alpha ~ U[0.9, 1]
    (every frame decays the state; the bridge decays across the window)."""
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 1, 7, 13, 14])
    e = _sampled(cfg, rows, None, alpha_range=(0.9, 1.0))
    print(f"768p decay sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_768p_text_keys_in_softmax_sampled():
    """The 768p workload with the 512 text tokens joining every video query's
    Softmax (one normaliser over the visible video keys and the text keys)."""
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 7, 14])
    inp = make_inputs(cfg)
    d = to_dev(inp)
    out = _fwd(d, cfg, text_softmax=True)
    torch.cuda.synchronize()
    got = gpu_rows(out, rows)
    del d, out
    torch.cuda.empty_cache()
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, rows=rows,
                                text_softmax=True)
    e = rel_err(got, want)
    print(f"768p text-softmax sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_768p_per_token_beta_sampled():
    """The 768p workload with one write gate per token, sigmoid(N(0,1))."""
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 7, 14])
    inp = make_inputs(cfg, beta_per_token=True)
    d = to_dev(inp)
    out = _fwd(d, cfg, beta_per_token=True)
    torch.cuda.synchronize()
    got = gpu_rows(out, rows)
    del d, out
    torch.cuda.empty_cache()
    want, _, _ = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, rows=rows,
                                beta_per_token=True)
    e = rel_err(got, want)
    print(f"768p per-token beta sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_long_clip_sampled():
    cfg = CONFIGS["long_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 1, 2, 29, 58, 59])
    e = _sampled(cfg, rows, None)
    print(f"long sampled ({len(rows)} rows): {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_batched_sampled():
    cfg = CONFIGS["batched_bf16"]
    rows = sample_rows(cfg, per_frame=3)
    e = _sampled(cfg, rows, [0, 15])
    print(f"batched sampled: {e:.2e}")
    assert e <= TOL_OUT["bf16"]


def test_span_clip_chunk5_and_dense():
    cfg = CONFIGS["span_bf16"]
    rows = sample_rows(cfg, per_frame=3)
    e = _sampled(cfg, rows, [0, 9])
    assert e <= TOL_OUT["bf16"]
    # one chunk spanning the clip: the Softmax branch is dense attention
    inp = make_inputs(cfg)
    d = to_dev(inp)
    o_s, _ = vdn.hybrid_attn_branches(d["q"], d["k"], d["v"], d["beta"], d["text_k"],
                                      d["text_v"], cfg.T, chunk=cfg.T, want_lin=False)
    torch.cuda.synchronize()
    got = gpu_rows(o_s, rows, [3])
    q = inp["q"][3:4].double()
    k = inp["k"][3:4].double()
    v = inp["v"][3:4].double()
    idx = torch.as_tensor(rows)
    s = torch.einsum("blhd,bmhd->bhlm", q[:, idx], k) / np.sqrt(cfg.d)
    dense = torch.einsum("bhlm,bmhd->blhd", torch.softmax(s, dim=-1), v).numpy()
    assert rel_err(got, dense) <= 2e-3


@pytest.mark.parametrize("beta_tok", [False, True])
@pytest.mark.parametrize("over", [dict(T=23, N=96, d=64, H=2), dict(T=12, N=136, d=128, H=2),
                                  dict(T=9, N=5, d=64, H=2)], ids=["d64", "d128", "N5"])
def test_boundary_states_tensor_core(over, beta_tok):
    """Chunk-boundary states of the bf16 path (tensor-core frame statistics +
    register Gauss-Jordan + chunk composition) against the oracle's literal
    frame-by-frame recurrence."""
    cfg = _edge_cfg(over)
    inp = make_inputs(cfg, alpha_range=(0.9, 1.0), beta_per_token=beta_tok)
    d = to_dev(inp)
    F, G = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"], cfg.T,
                                   alpha=d["alpha"], chunk=cfg.chunk, beta_per_token=beta_tok)
    torch.cuda.synchronize()
    Fo, Go = O.boundary_states(inp["k"], inp["v"], inp["beta"], inp["text_k"], inp["text_v"],
                               cfg.T, cfg.N, cfg.chunk, alpha=inp["alpha"],
                               beta_per_token=beta_tok)
    eF, eG = rel_err(F.double().cpu(), Fo), rel_err(G.double().cpu(), Go)
    print(f"states {over}: F {eF:.2e} G {eG:.2e}")
    assert eF <= 1e-4 and eG <= 1e-4


# (name, overrides, make_inputs kwargs, extra kwargs)
SCAN_CASES = [
    ("tiny_f32", None, {}, {}),
    ("d64", dict(T=23, N=96, d=64, H=2), dict(alpha_range=(0.9, 1.0)), {}),
    ("d128", dict(T=12, N=136, d=128, H=2), dict(alpha_range=(0.9, 1.0)), {}),
    ("T1", dict(T=1, N=40), {}, {}),
    ("T2", dict(T=2, N=24), {}, {}),
    ("T7_partial_chunk", dict(T=7, N=5), dict(alpha_range=(0.85, 1.0)), {}),
    ("chunk1_r0", dict(T=9, N=130, chunk=1, window_radius=0), {}, {}),
    ("c3_r2", dict(T=12, N=64, chunk=3, window_radius=2), {}, {}),
    ("text_full", dict(T=16, N=64), {}, dict(text_full=True)),
    ("beta_per_token_d128", dict(T=8, N=40, d=128, H=2, n_text=37),
     dict(beta_per_token=True), dict(beta_per_token=True)),
    ("frozen_d64", dict(T=14, N=72), None, dict(frozen_state=True)),
]


@pytest.mark.parametrize("scan", ["frames", "chunks"])
@pytest.mark.parametrize("name,over,mk,kw", SCAN_CASES, ids=[c[0] for c in SCAN_CASES])
def test_scan_paths_match_the_oracle(name, over, mk, kw, scan):
    """The two evaluations of the bidirectional scan (over frames, or chunk
    composition + chunk scan) give the oracle's chunk-boundary states and
    linear readout, on the tensor-core and FP32 frame kernels."""
    if over is None and name == "tiny_f32":
        cfg = CONFIGS["tiny_f32"]
    else:
        cfg = _edge_cfg(over)
    if kw.get("frozen_state"):
        inp = _frozen_inputs(cfg)
    else:
        inp = make_inputs(cfg, **mk)
    d = to_dev(inp)
    F, G = vdn.vda_boundary_states(d["k"], d["v"], d["beta"], d["text_k"], d["text_v"], cfg.T,
                                   alpha=d["alpha"], chunk=cfg.chunk,
                                   window_radius=cfg.window_radius, scan=scan, **kw)
    _, o_l = _branches(d, cfg, want_soft=False, scan=scan, **kw)
    torch.cuda.synchronize()
    okw = dict(text_full=kw.get("text_full", False), beta_per_token=kw.get("beta_per_token", False),
               frozen=kw.get("frozen_state", False))
    Fo, Go = O.boundary_states(inp["k"], inp["v"], inp["beta"], inp["text_k"], inp["text_v"],
                               cfg.T, cfg.N, cfg.chunk, cfg.window_radius, alpha=inp["alpha"],
                               **okw)
    _, _, wl = oracle_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, **okw)
    tol = 1e-5 if cfg.dtype == "f32" else 1e-4
    eF, eG = rel_err(F.double().cpu(), Fo), rel_err(G.double().cpu(), Go)
    eL = rel_err(o_l.double().cpu(), wl)
    print(f"scan={scan} {name}: F {eF:.2e} G {eG:.2e} o_lin {eL:.2e}")
    assert eF <= tol and eG <= tol and eL <= tol


def test_scan_paths_agree_on_the_768p_forward():
    """At 768p the shape picks the frame scan.  The linear readout (FP32, before
    any rounding) of the frame scan and of the chunk composition agree to FP32
    rounding; the outputs, which pass through one fp16 rounding of the gated
    operand (where a last-bit difference in o_lin can flip a rounding), agree
    within the output tolerance."""
    cfg = CONFIGS["768p_h4_bf16"]
    d = to_dev(make_inputs(cfg, alpha_range=(0.9, 1.0)))
    _, la = _branches(d, cfg, want_soft=False, scan="frames")
    _, lb = _branches(d, cfg, want_soft=False, scan="chunks")
    a = _fwd(d, cfg, scan="frames")
    b = _fwd(d, cfg, scan="chunks")
    torch.cuda.synchronize()
    e_lin = float((la - lb).abs().max()) / float(lb.pow(2).mean().sqrt())
    e_out = float((a - b).abs().max()) / float(b.float().pow(2).mean().sqrt())
    print(f"768p (4 heads) frames vs chunks: o_lin {e_lin:.2e}, out {e_out:.2e}")
    assert e_lin <= 1e-5
    assert e_out <= TOL_OUT["bf16"]
