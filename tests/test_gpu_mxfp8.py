"""MXFP8 projection mode (VDN_FLAG_PROJ_MXFP8) against the MXFP8 oracle."""
import numpy as np
import pytest
import torch

import softmax_attention_video_chunk_b200 as vdn
from oracle import mxfp8 as MX
from oracle import vdn_oracle as O
from synth import CONFIGS, make_inputs, sample_rows
from tests._parity import TOL_OUT, gpu_rows, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _decode(codes, scales, rows, cols):
    """(elements float64 [rows, cols], exponents [rows, cols/32]) from the
    library's codes and scale atoms."""
    el = codes.view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()
    s = scales.cpu().numpy()
    r = np.arange(rows)[:, None]
    j = np.arange(cols // 32)[None, :]
    idx = ((r // 128) * (cols // 128) + j // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + j % 4
    return el, s[idx].astype(np.float64) - 127


def test_quantizer_is_bit_exact():
    g = torch.Generator().manual_seed(21)
    rows, cols = 300, 384
    x = torch.randn(rows, cols, generator=g) * torch.exp(torch.randn(rows, 1, generator=g) * 3)
    x[5, 32:64] = 0                                   # all-zero block
    x[6, 0:32] = 1.99 * 2.0 ** 3                      # clips at 448 * scale
    x[7, 64:96] = torch.linspace(-1, 1, 32) * 1e-4    # small values (fp16 subnormal area)
    x[8, :] = torch.tensor([2.0 ** -9 * k for k in range(cols)]) % 0.75
    xh = x.to(torch.float16)
    codes, scales = vdn.mxfp8_quantize(xh.cuda(), rows_padded=384)
    torch.cuda.synchronize()
    el, e = _decode(codes, scales, rows, cols)
    want_el, want_e = MX.mxfp8_quantize(xh.double().numpy(), axis=-1)
    np.testing.assert_array_equal(e, want_e)
    np.testing.assert_array_equal(el, want_el)
    # padded rows carry the smallest scale
    _, e_pad = _decode(torch.zeros(384, cols, dtype=torch.uint8), scales, 384, cols)
    assert np.all(e_pad[rows:] == -127)


CASES = [
    ("d64_H3", dict(T=13, N=72, H=3, d=64), {}),          # D_out = 192: a ragged 256-column tile
    ("d128_H2", dict(T=9, N=130, H=2, d=128, n_text=40), dict(gates="random")),
    ("d64_H8_alpha", dict(T=20, N=64, H=8, d=64), dict(alpha_range=(0.9, 1.0), gates="random")),
]


def _cfg(over):
    return CONFIGS["small_bf16"].replace(seed=13).replace(**over)


def _oracle_mx_projection_of(x16, W_soft, W_lin):
    """The oracle's MXFP8 projection of a given fp16 operand x [..., 2, H, d]:
    quantise x along its row and [W_soft; W_lin] (fp16) along each column,
    multiply exactly."""
    x = x16.double().cpu().numpy()
    lead = x.shape[:-3]
    x = x.reshape(lead + (-1,))
    W = np.concatenate([O._to_np(W_soft), O._to_np(W_lin)], axis=0)
    return MX.mxfp8_dequantize(x, axis=-1) @ MX.mxfp8_dequantize(MX.to_fp16(W), axis=0)


@pytest.mark.parametrize("name,over,mk", CASES, ids=[c[0] for c in CASES])
def test_mxfp8_projection_of_the_library_operand(name, over, mk):
    """The block-scaled GEMM against the oracle on the same fp16 operand: the
    quantisation is exact on both sides, so only FP32 accumulation differs."""
    cfg = _cfg(over)
    d = to_dev(make_inputs(cfg, **mk))
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], proj_mxfp8=True)
    x = vdn.hybrid_attn_operand(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                d["gates"], cfg.T, alpha=d["alpha"], params=p)
    out = vdn.output_projection(x, d["W_soft"], d["W_lin"], p)
    torch.cuda.synchronize()
    want = _oracle_mx_projection_of(x, d["W_soft"], d["W_lin"])
    e = rel_err(out.double().cpu().numpy(), want)
    print(f"mxfp8 GEMM {name}: {e:.2e}")
    assert e <= 1e-5


@pytest.mark.parametrize("name,over,mk", CASES, ids=[c[0] for c in CASES])
def test_mxfp8_forward_within_the_formats_bounds(name, over, mk):
    """The whole forward in MXFP8 mode.  Against the oracle's MXFP8 forward the
    difference comes from elements whose value sits within the upstream
    difference (~2^-10 relative: fp16 P and fp16 x) of an E4M3 rounding
    boundary and so land on the neighbouring value: about 1% of the elements,
    one E4M3 step each, i.e. an RMS difference near sqrt(0.01) 2^-3.5 = 0.9% of
    the output RMS and a maximum of a few times that (bound: 6%).  Against the
    exact projection the format's own error (3-bit mantissas on both operands)
    is about 4% RMS (bound 6%) and up to about 25% at single outputs (bound
    35%)."""
    cfg = _cfg(over)
    inp = make_inputs(cfg, **mk)
    d = to_dev(inp)
    out = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                              d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"],
                              proj_mxfp8=True)
    plain = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"])
    torch.cuda.synchronize()
    exact, o_s, o_l = O.hybrid_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    g = O._to_np(inp["gates"])
    want = MX.output_projection_mxfp8(o_s, o_l, g[0], g[1], O._to_np(inp["W_soft"]),
                                      O._to_np(inp["W_lin"]))
    got = out.double().cpu().numpy()
    rms_w = np.sqrt(np.mean(want ** 2))
    e_mx_max = rel_err(got, want)
    e_mx_rms = np.sqrt(np.mean((got - want) ** 2)) / rms_w
    rms = np.sqrt(np.mean(exact ** 2))
    e_fmt_max = np.max(np.abs(got - exact)) / rms
    e_fmt_rms = np.sqrt(np.mean((got - exact) ** 2)) / rms
    print(f"mxfp8 {name}: vs MXFP8 oracle max {e_mx_max:.2e} rms {e_mx_rms:.2e}; vs exact "
          f"max {e_fmt_max:.3f} rms {e_fmt_rms:.3f}; default path vs exact "
          f"{rel_err(plain.double().cpu().numpy(), exact):.2e}")
    assert e_mx_rms <= 0.015 and e_mx_max <= 0.06
    assert e_fmt_rms <= 0.06 and e_fmt_max <= 0.35
    assert not torch.equal(out, plain)


@pytest.mark.parametrize("name,over,mk", CASES, ids=[c[0] for c in CASES])
def test_mxfp8_operand_projection_entry(name, over, mk):
    """vdn_output_projection with the flag is the MXFP8 half of the forward:
    the forward's Softmax and readout epilogues quantise their fp16 rows in
    registers, the entry quantises the fp16 operand with the stand-alone
    quantiser, and the two give the same codes and scales (bit-equal outputs),
    including the scale rows past B*L in the last 128-row group (d64_H3 has
    936 rows)."""
    cfg = _cfg(over)
    d = to_dev(make_inputs(cfg, **mk))
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], proj_mxfp8=True)
    x = vdn.hybrid_attn_operand(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                d["gates"], cfg.T, alpha=d["alpha"], params=p)
    out = vdn.output_projection(x, d["W_soft"], d["W_lin"], p)
    fwd = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                              d["W_soft"], d["W_lin"], d["gates"], cfg.T, alpha=d["alpha"],
                              params=p)
    torch.cuda.synchronize()
    assert torch.equal(out, fwd)


def test_mxfp8_768p_sampled():
    """768p: the MXFP8 projection of the library's operand on sampled rows
    against the oracle's MXFP8 projection of the same rows (FP32 accumulation
    over K = 6144 is the only difference)."""
    cfg = CONFIGS["768p_bf16"]
    rows = sample_rows(cfg, per_frame=2, chunks=[0, 7, 14])
    d = to_dev(make_inputs(cfg, gates="random"))
    p = vdn.params_for(d["q"], d["v"], d["text_k"], cfg.T, d["W_soft"], proj_mxfp8=True)
    out = vdn.hybrid_attn_fwd(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                              d["W_soft"], d["W_lin"], d["gates"], cfg.T, params=p)
    x = vdn.hybrid_attn_operand(d["q"], d["k"], d["v"], d["beta"], d["text_k"], d["text_v"],
                                d["gates"], cfg.T, params=p)
    torch.cuda.synchronize()
    idx = torch.as_tensor(rows, device="cuda")
    got = out[:, idx].double().cpu().numpy()
    want = _oracle_mx_projection_of(x[:, idx], d["W_soft"], d["W_lin"])
    e = rel_err(got, want)
    print(f"mxfp8 768p sampled ({len(rows)} rows): {e:.2e}")
    assert e <= 1e-5
