"""Shared helpers of the GPU parity tests (not collected as tests)."""
import numpy as np
import torch

from oracle import vdn_oracle as O

# Tolerances of the output, relative to the oracle output's RMS (max |err|):
# float32 inputs 1e-5, bf16 inputs with FP32 state 2e-3.
TOL_OUT = {"f32": 1e-5, "bf16": 2e-3}


def rel_err(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    rms = np.sqrt(np.mean(want * want))
    return float(np.max(np.abs(got - want)) / rms)


def to_dev(inp: dict, device="cuda") -> dict:
    return {k: (v.to(device).contiguous() if v is not None else None) for k, v in inp.items()}


def slice_batch(inp: dict, bsel) -> dict:
    """The same workload restricted to batch items ``bsel`` (for the oracle)."""
    out = {}
    for k, v in inp.items():
        if v is None:
            out[k] = None
        elif k in ("W_soft", "W_lin"):
            out[k] = v
        elif k == "gates":
            out[k] = v[:, bsel]
        else:
            out[k] = v[bsel]
    return out


def oracle_forward(inp: dict, T, N, chunk, radius, rows=None, bsel=None, **kw):
    src = slice_batch(inp, bsel) if bsel is not None else inp
    return O.hybrid_forward(src, T, N, chunk, radius, rows=rows, **kw)


def gpu_rows(x: torch.Tensor, rows, bsel=None) -> np.ndarray:
    """Select [b, rows] of a [B, L, ...] device tensor -> float64 numpy."""
    t = x if bsel is None else x[list(bsel)]
    idx = torch.as_tensor(np.asarray(rows), device=x.device)
    return t[:, idx].double().cpu().numpy()
