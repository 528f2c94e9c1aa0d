"""softmax_attention_video_chunk_b200 -- Python binding of libvdn.

Argument marshalling only: every step of the VDN hybrid attention forward
runs in the CUDA kernels of ``libvdn.so`` (sm_100a), reached through its C ABI
(``include/vdn.h``).  PyTorch supplies device memory and the stream.  There is
no fallback: if the library is missing or the call fails, this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvdn.so")

VDN_F32, VDN_BF16 = 0, 1
FLAG_TEXT_FULL, FLAG_SIMT, FLAG_TEXT_SOFTMAX, FLAG_BETA_PER_TOKEN = 1, 2, 4, 8
FLAG_FROZEN_STATE = 16
FLAG_SCAN_FRAMES, FLAG_SCAN_CHUNKS = 32, 64
FLAG_PROJ_MXFP8 = 128

STATUS = {
    0: "VDN_OK", 1: "VDN_ERR_INVALID_ARG", 2: "VDN_ERR_SHAPE", 3: "VDN_ERR_DTYPE",
    4: "VDN_ERR_ALIGNMENT", 5: "VDN_ERR_WORKSPACE", 6: "VDN_ERR_CUDA", 7: "VDN_ERR_TIMEOUT",
    8: "VDN_ERR_UNSUPPORTED", 9: "VDN_ERR_RANGE",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}


class VdnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({lib().vdn_status_string(code).decode()})")


N_STAGES = 5
STAGE_NAMES = ("vda_states", "convert", "softmax", "readout", "projection")


class VdnStageEvents(ctypes.Structure):
    _fields_ = [("events", ctypes.c_void_p * (N_STAGES + 1))]


class VdnParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int), ("N", ctypes.c_int),
        ("d_k", ctypes.c_int), ("d_v", ctypes.c_int), ("n_text", ctypes.c_int),
        ("D_out", ctypes.c_int), ("chunk", ctypes.c_int), ("window_radius", ctypes.c_int),
        ("dtype", ctypes.c_int), ("out_dtype", ctypes.c_int), ("softmax_scale", ctypes.c_float),
        ("rms_eps", ctypes.c_float), ("flags", ctypes.c_uint),
    ]


class VdnPrepParams(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("T", ctypes.c_int),
        ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int), ("d", ctypes.c_int),
        ("spatial_taps", ctypes.c_int), ("temporal_taps", ctypes.c_int),
        ("dtype", ctypes.c_int), ("l2_eps", ctypes.c_float),
    ]


PREP_WORKSPACE_BYTES = 256

_lib = None
_P = ctypes.c_void_p


def lib() -> ctypes.CDLL:
    """Load libvdn.so (built in-tree by ``__graft_entry__.build()`` or
    ``python -m softmax_attention_video_chunk_b200._build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m softmax_attention_video_chunk_b200._build`")
        L = ctypes.CDLL(LIB_PATH)
        PP = ctypes.POINTER(VdnParams)
        L.vdn_abi_version.restype = ctypes.c_int
        L.vdn_status_string.restype = ctypes.c_char_p
        L.vdn_status_string.argtypes = [ctypes.c_int]
        L.vdn_params_init.restype = ctypes.c_int
        L.vdn_params_init.argtypes = [PP] + [ctypes.c_int] * 7
        L.vdn_workspace_bytes.restype = ctypes.c_int
        L.vdn_workspace_bytes.argtypes = [PP, ctypes.POINTER(ctypes.c_size_t)]
        L.vdn_forward_launches.restype = ctypes.c_int
        L.vdn_forward_launches.argtypes = [PP, ctypes.POINTER(ctypes.c_int)]
        L.vdn_hybrid_attn_fwd.restype = ctypes.c_int
        L.vdn_hybrid_attn_fwd.argtypes = [PP] + [_P] * 12 + [ctypes.c_size_t, _P]
        L.vdn_hybrid_attn_fwd_staged.restype = ctypes.c_int
        L.vdn_hybrid_attn_fwd_staged.argtypes = ([PP] + [_P] * 12 + [ctypes.c_size_t, _P] +
                                                 [ctypes.POINTER(VdnStageEvents)])
        L.vdn_hybrid_attn_branches.restype = ctypes.c_int
        L.vdn_hybrid_attn_branches.argtypes = [PP] + [_P] * 10 + [ctypes.c_size_t, _P]
        L.vdn_vda_boundary_states.restype = ctypes.c_int
        L.vdn_vda_boundary_states.argtypes = [PP] + [_P] * 9 + [ctypes.c_size_t, _P]
        L.vdn_vda_boundary_states_noalloc.restype = ctypes.c_int
        L.vdn_vda_boundary_states_noalloc.argtypes = [PP] + [_P] * 8 + [_P]
        L.vdn_noalloc_device_status.restype = ctypes.c_int
        L.vdn_noalloc_device_status.argtypes = [_P]
        L.vdn_device_status.restype = ctypes.c_int
        L.vdn_device_status.argtypes = [PP, _P, _P]
        L.vdn_hybrid_attn_fwd_split.restype = ctypes.c_int
        L.vdn_hybrid_attn_fwd_split.argtypes = ([PP] + [_P] * 15 + [ctypes.c_size_t, _P] +
                                                [ctypes.POINTER(VdnStageEvents)])
        PPP = ctypes.POINTER(VdnPrepParams)
        L.vdn_prep_params_init.restype = ctypes.c_int
        L.vdn_prep_params_init.argtypes = [PPP] + [ctypes.c_int] * 7
        L.vdn_vda_prep.restype = ctypes.c_int
        L.vdn_vda_prep.argtypes = [PPP] + [_P] * 11 + [ctypes.c_size_t, _P]
        L.vdn_text_query_attn.restype = ctypes.c_int
        L.vdn_text_query_attn.argtypes = [PP] + [_P] * 7 + [ctypes.c_size_t, _P]
        L.vdn_selftest_bounded_wait.restype = ctypes.c_int
        L.vdn_selftest_bounded_wait.argtypes = [_P, ctypes.c_uint, _P]
        L.vdn_hybrid_attn_fwd_host.restype = ctypes.c_int
        L.vdn_hybrid_attn_fwd_host.argtypes = ([PP, _P, _P, _P, _P, ctypes.c_size_t, _P, _P, _P,
                                                ctypes.POINTER(ctypes.c_size_t),
                                                ctypes.POINTER(ctypes.c_size_t)])
        L.vdn_host_slot_release.restype = ctypes.c_int
        L.vdn_host_slot_release.argtypes = [_P]
        L.vdn_hybrid_attn_operand.restype = ctypes.c_int
        L.vdn_hybrid_attn_operand.argtypes = [PP] + [_P] * 10 + [ctypes.c_size_t, _P]
        L.vdn_output_projection.restype = ctypes.c_int
        L.vdn_output_projection.argtypes = [PP, ctypes.c_longlong] + [_P] * 5 + [ctypes.c_size_t, _P]
        L.vdn_mxfp8_quantize.restype = ctypes.c_int
        L.vdn_mxfp8_quantize.argtypes = [_P, ctypes.c_longlong, ctypes.c_longlong, ctypes.c_int,
                                         _P, _P, ctypes.c_size_t, _P]
        L.vdn_selftest_exp2.restype = ctypes.c_int
        L.vdn_selftest_exp2.argtypes = [_P, _P, ctypes.c_size_t, _P]
        _lib = L
    return _lib


def make_params(B, H, T, N, d, n_text, dtype="bf16", *, chunk=5, window_radius=1,
                D_out=None, out_dtype="f32", softmax_scale=0.0, rms_eps=1e-6,
                text_full=False, simt=False, text_softmax=False,
                beta_per_token=False, frozen_state=False, scan=None,
                proj_mxfp8=False) -> VdnParams:
    p = VdnParams()
    dt = {"f32": VDN_F32, "bf16": VDN_BF16}
    rc = lib().vdn_params_init(ctypes.byref(p), B, H, T, N, d, n_text, dt[dtype])
    p.chunk, p.window_radius = chunk, window_radius
    p.D_out = H * d if D_out is None else D_out
    p.out_dtype = dt[out_dtype]
    p.softmax_scale, p.rms_eps = softmax_scale, rms_eps
    p.flags = ((FLAG_TEXT_FULL if text_full else 0) | (FLAG_SIMT if simt else 0) |
               (FLAG_TEXT_SOFTMAX if text_softmax else 0) |
               (FLAG_BETA_PER_TOKEN if beta_per_token else 0) |
               (FLAG_FROZEN_STATE if frozen_state else 0) |
               {None: 0, "frames": FLAG_SCAN_FRAMES, "chunks": FLAG_SCAN_CHUNKS}[scan] |
               (FLAG_PROJ_MXFP8 if proj_mxfp8 else 0))
    size = ctypes.c_size_t(0)
    rc = lib().vdn_workspace_bytes(ctypes.byref(p), ctypes.byref(size))
    if rc != 0:
        raise VdnError(rc, "vdn_workspace_bytes")
    return p


def workspace_bytes(p: VdnParams) -> int:
    size = ctypes.c_size_t(0)
    rc = lib().vdn_workspace_bytes(ctypes.byref(p), ctypes.byref(size))
    if rc != 0:
        raise VdnError(rc, "vdn_workspace_bytes")
    return size.value


def forward_launches(p: VdnParams) -> int:
    """Kernel launches that one ``hybrid_attn_fwd`` call enqueues for ``p``."""
    n = ctypes.c_int(0)
    rc = lib().vdn_forward_launches(ctypes.byref(p), ctypes.byref(n))
    if rc != 0:
        raise VdnError(rc, "vdn_forward_launches")
    return n.value


# --------------------------------------------------------------------------
# torch-facing wrappers (marshalling only)
# --------------------------------------------------------------------------

def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_name(t) -> str:
    import torch
    if t.dtype == torch.bfloat16:
        return "bf16"
    if t.dtype == torch.float32:
        return "f32"
    raise ValueError(f"unsupported dtype {t.dtype}")


def params_for(q, v, text_k, T, W_soft=None, **kw) -> VdnParams:
    B, L, H, d = q.shape
    if L % T:
        raise ValueError("q.shape[1] must be T * N")
    n_text = 0 if text_k is None else text_k.shape[1]
    D_out = None if W_soft is None else W_soft.shape[1]
    return make_params(B, H, T, L // T, d, n_text, _dtype_name(q), D_out=D_out, **kw)


def alloc_workspace(p: VdnParams, device="cuda"):
    import torch
    return torch.empty(max(workspace_bytes(p), 256), dtype=torch.uint8, device=device)


def hybrid_attn_fwd(q, k, v, beta, text_k, text_v, W_soft, W_lin, gates, T, *, alpha=None,
                    out=None, workspace=None, stream=None, params=None, events=None, lin=None,
                    **kw):
    """out [B, L, D_out] = VDN hybrid attention forward (all steps in libvdn).

    ``events``: optional list of N_STAGES + 1 torch.cuda.Event(enable_timing=True)
    recorded at the stage boundaries (see vdn_hybrid_attn_fwd_staged).
    ``lin``: optional (q_lin, k_lin, v_lin), the linear branch's own inputs
    (vdn_hybrid_attn_fwd_split); by default both branches read q, k, v."""
    import torch
    p = params or params_for(q, v, text_k, T, W_soft, **kw)
    if out is None:
        odt = torch.float32 if p.out_dtype == VDN_F32 else torch.bfloat16
        out = torch.empty(q.shape[0], q.shape[1], p.D_out, dtype=odt, device=q.device)
    ws = alloc_workspace(p, q.device) if workspace is None else workspace
    ev = None
    if events is not None:
        if len(events) != N_STAGES + 1:
            raise ValueError(f"need {N_STAGES + 1} events")
        ev = VdnStageEvents()
        for i, e in enumerate(events):
            if not e.cuda_event:  # torch creates the CUDA event on first record
                e.record(torch.cuda.current_stream() if stream is None else stream)
            ev.events[i] = e.cuda_event
        ev = ctypes.byref(ev)
    if lin is None:
        rc = lib().vdn_hybrid_attn_fwd_staged(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                              _ptr(beta), _ptr(alpha), _ptr(text_k),
                                              _ptr(text_v), _ptr(W_soft), _ptr(W_lin),
                                              _ptr(gates), _ptr(out), _ptr(ws), ws.numel(),
                                              _stream(stream), ev)
    else:
        ql, kl, vl = lin
        rc = lib().vdn_hybrid_attn_fwd_split(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v),
                                             _ptr(ql), _ptr(kl), _ptr(vl), _ptr(beta),
                                             _ptr(alpha), _ptr(text_k), _ptr(text_v),
                                             _ptr(W_soft), _ptr(W_lin), _ptr(gates), _ptr(out),
                                             _ptr(ws), ws.numel(), _stream(stream), ev)
    if rc != 0:
        raise VdnError(rc, "vdn_hybrid_attn_fwd")
    return out


def hybrid_attn_operand(q, k, v, beta, text_k, text_v, gates, T, *, alpha=None, x=None,
                        workspace=None, stream=None, params=None, **kw):
    """x float16 [B, L, 2, H, d]: the gated branch outputs [g_s*o_s, g_l*RMS(o_l)],
    the operand of the output projections (vdn_hybrid_attn_operand)."""
    import torch
    p = params or params_for(q, v, text_k, T, **kw)
    B, L, H, d = q.shape
    if x is None:
        x = torch.empty(B, L, 2, H, d, dtype=torch.float16, device=q.device)
    ws = alloc_workspace(p, q.device) if workspace is None else workspace
    rc = lib().vdn_hybrid_attn_operand(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                       _ptr(alpha), _ptr(text_k), _ptr(text_v), _ptr(gates),
                                       _ptr(x), _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_hybrid_attn_operand")
    return x


def output_projection(x, W_soft, W_lin, params, *, out=None, workspace=None, stream=None):
    """out [..., D_out] = x[..., 0, :, :] W_soft + x[..., 1, :, :] W_lin for an
    operand x float16 [..., 2, H, d] (vdn_output_projection); ``params`` gives
    H, d, D_out and the dtypes."""
    import torch
    p = params
    lead = x.shape[:-3]
    rows = int(x.numel() // (2 * p.H * p.d_k))
    if out is None:
        odt = torch.float32 if p.out_dtype == VDN_F32 else torch.bfloat16
        out = torch.empty(*lead, p.D_out, dtype=odt, device=x.device)
    ws = alloc_workspace(p, x.device) if workspace is None else workspace
    rc = lib().vdn_output_projection(ctypes.byref(p), rows, _ptr(x), _ptr(W_soft), _ptr(W_lin),
                                     _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_output_projection")
    return out


def text_query_attn(text_q, k, v, text_k, text_v, T, *, workspace=None, stream=None,
                    params=None, **kw):
    """o_text float32 [B, n_text, H, d]: the text tokens as queries over every
    video and text key (vdn_text_query_attn)."""
    import torch
    kw["text_softmax"] = True  # workspace with the text tokens' V^T
    p = params or params_for(k, v, text_k, T, **kw)
    o = torch.empty(text_q.shape, dtype=torch.float32, device=text_q.device)
    ws = alloc_workspace(p, k.device) if workspace is None else workspace
    rc = lib().vdn_text_query_attn(ctypes.byref(p), _ptr(text_q), _ptr(k), _ptr(v), _ptr(text_k),
                                   _ptr(text_v), _ptr(o), _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_text_query_attn")
    return o


def make_prep_params(B, H, T, grid_h, grid_w, d, dtype="bf16", l2_eps=1e-6) -> VdnPrepParams:
    p = VdnPrepParams()
    rc = lib().vdn_prep_params_init(ctypes.byref(p), B, H, T, grid_h, grid_w, d,
                                    {"f32": VDN_F32, "bf16": VDN_BF16}[dtype])
    if rc != 0:
        raise VdnError(rc, "vdn_prep_params_init")
    p.l2_eps = l2_eps
    return p


def vda_prep(q, k, v, wk_s, wk_t, wv_s, wv_t, T, grid_h, grid_w, *, l2_eps=1e-6, out=None,
             workspace=None, stream=None, params=None):
    """(q_l, k_l, v_l) = VDA-Prep of the raw projections (see vdn_vda_prep):
    q_l = L2(q), k_l = L2(SiLU(conv(k))), v_l = SiLU(conv(v)).  Inputs
    [B, T*grid_h*grid_w, H, d]; filters float32 [H*d, 3, 3] and [H*d, 5].
    Pass q = None to skip Q, or k = v = None (and the filters) to skip K/V."""
    import torch
    x = k if k is not None else q
    B, L, H, d = x.shape
    p = params or make_prep_params(B, H, T, grid_h, grid_w, d, _dtype_name(x), l2_eps)
    if out is None:
        out = tuple(None if t is None else torch.empty_like(t) for t in (q, k, v))
    ws = (torch.empty(PREP_WORKSPACE_BYTES, dtype=torch.uint8, device=x.device)
          if workspace is None else workspace)
    rc = lib().vdn_vda_prep(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(wk_s), _ptr(wk_t),
                            _ptr(wv_s), _ptr(wv_t), _ptr(out[0]), _ptr(out[1]), _ptr(out[2]),
                            _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_vda_prep")
    return out


INPUT_NAMES = ("q", "k", "v", "beta", "alpha", "text_k", "text_v", "W_soft", "W_lin", "gates")
_HOST_FIELDS = ("q", "k", "v", "beta", "alpha", "text_k", "text_v", "W_o_soft", "W_o_lin",
                "gates")


class VdnHostInputs(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in _HOST_FIELDS]


class VdnHostSlot(ctypes.Structure):
    _fields_ = ([(n, ctypes.c_void_p) for n in _HOST_FIELDS] + [("out", ctypes.c_void_p)] +
                [("events", ctypes.c_void_p * 3), ("used", ctypes.c_int)])


def _host_ptr(t) -> Optional[int]:
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("host tensor expected")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


class HostSlot:
    """Device buffers of one end-to-end step (vdn_host_slot): inputs shaped
    like ``host_example`` and ``out``; the slot's events are released with
    the object (after the device is done with them)."""

    def __init__(self, host_example: dict, p: VdnParams, device):
        import torch
        self.bufs = {n: (None if host_example.get(n) is None else
                         torch.empty_like(host_example[n], device=device)) for n in INPUT_NAMES}
        odt = torch.float32 if p.out_dtype == VDN_F32 else torch.bfloat16
        self.out = torch.empty(p.B, p.T * p.N, p.D_out, dtype=odt, device=device)
        self.c = VdnHostSlot()
        for f, n in zip(_HOST_FIELDS, INPUT_NAMES):
            setattr(self.c, f, _ptr(self.bufs[n]))
        self.c.out = _ptr(self.out)

    def release(self):
        if self.c is not None:
            lib().vdn_host_slot_release(ctypes.byref(self.c))
            self.c = None

    def __del__(self):
        try:
            self.release()
        except Exception:
            pass


def _host_inputs(host: dict) -> VdnHostInputs:
    hi = VdnHostInputs()
    for f, n in zip(_HOST_FIELDS, INPUT_NAMES):
        setattr(hi, f, _host_ptr(host.get(n)))
    return hi


def host_fwd_step(p: VdnParams, host: dict, out_host, slot: HostSlot, workspace, s_in, s_cmp,
                  s_out):
    """One end-to-end step through vdn_hybrid_attn_fwd_host: uploads on
    ``s_in``, the forward on ``s_cmp``, the download into ``out_host`` on
    ``s_out`` (torch streams).  Returns (h2d_bytes, d2h_bytes)."""
    h2d, d2h = ctypes.c_size_t(0), ctypes.c_size_t(0)
    hi = _host_inputs(host)
    rc = lib().vdn_hybrid_attn_fwd_host(ctypes.byref(p), ctypes.byref(hi), _host_ptr(out_host),
                                        ctypes.byref(slot.c), _ptr(workspace), workspace.numel(),
                                        _stream(s_in), _stream(s_cmp), _stream(s_out),
                                        ctypes.byref(h2d), ctypes.byref(d2h))
    if rc != 0:
        raise VdnError(rc, "vdn_hybrid_attn_fwd_host")
    return h2d.value, d2h.value


def hybrid_attn_fwd_host(host: dict, T, *, slot=None, out_host=None, workspace=None,
                         stream=None, params=None, **kw):
    """End-to-end call on host (pinned) tensors through vdn_hybrid_attn_fwd_host:
    every input copied to the device, the forward, and ``out`` copied back into
    ``out_host``, all on one stream.  ``slot`` (a HostSlot) holds reusable
    device buffers.  Returns (out_host, h2d_bytes, d2h_bytes); out_host is
    complete after the stream synchronises."""
    import torch
    dev = torch.device("cuda", torch.cuda.current_device())
    s = torch.cuda.current_stream() if stream is None else stream
    if params is None:
        W = host["W_soft"]
        D_out = W.shape[1]
        B, L, H, d = host["q"].shape
        n_text = 0 if host.get("text_k") is None else host["text_k"].shape[1]
        params = make_params(B, H, T, L // T, d, n_text, _dtype_name(host["q"]), D_out=D_out,
                             **kw)
    p = params
    slot = HostSlot(host, p, dev) if slot is None else slot
    ws = alloc_workspace(p, dev) if workspace is None else workspace
    if out_host is None:
        odt = torch.float32 if p.out_dtype == VDN_F32 else torch.bfloat16
        out_host = torch.empty(p.B, p.T * p.N, p.D_out, dtype=odt, pin_memory=True)
    h2d, d2h = host_fwd_step(p, host, out_host, slot, ws, s, s, s)
    return out_host, h2d, d2h


def hybrid_attn_branches(q, k, v, beta, text_k, text_v, T, *, alpha=None, workspace=None,
                         stream=None, want_soft=True, want_lin=True, params=None, **kw):
    """(o_soft, o_lin) float32 [B, L, H, d]; o_lin before its RMS norm."""
    import torch
    p = params or params_for(q, v, text_k, T, **kw)
    o_s = torch.empty(q.shape, dtype=torch.float32, device=q.device) if want_soft else None
    o_l = torch.empty(q.shape, dtype=torch.float32, device=q.device) if want_lin else None
    ws = alloc_workspace(p, q.device) if workspace is None else workspace
    rc = lib().vdn_hybrid_attn_branches(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
                                        _ptr(alpha), _ptr(text_k), _ptr(text_v), _ptr(o_s),
                                        _ptr(o_l), _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_hybrid_attn_branches")
    return o_s, o_l


def vda_boundary_states(k, v, beta, text_k, text_v, T, *, alpha=None, workspace=None,
                        stream=None, params=None, **kw):
    """(F, G) float32 [B, H, n_chunks, d, d]: the forward / reverse state each
    query chunk reads before its decay bridge."""
    import torch
    p = params or params_for(k, v, text_k, T, **kw)
    nc = (p.T + p.chunk - 1) // p.chunk
    F = torch.empty(p.B, p.H, nc, p.d_k, p.d_v, dtype=torch.float32, device=k.device)
    G = torch.empty_like(F)
    ws = alloc_workspace(p, k.device) if workspace is None else workspace
    rc = lib().vdn_vda_boundary_states(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(beta),
                                       _ptr(alpha), _ptr(text_k), _ptr(text_v), _ptr(F),
                                       _ptr(G), _ptr(ws), ws.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_vda_boundary_states")
    return F, G


NOALLOC_SCRATCH_BYTES = 32 << 20


def vda_boundary_states_noalloc(k, v, beta, text_k, text_v, T, *, alpha=None, stream=None,
                                params=None, **kw):
    """Same result as vda_boundary_states, without any workspace: the library
    uses its own static device array (NOALLOC_SCRATCH_BYTES per GPU, shared by
    all calls; calls that overlap on the GPU race).  For callers that cannot
    allocate device memory.  Only the outputs F, G are allocated here, by the
    caller side (torch)."""
    import torch
    p = params or params_for(k, v, text_k, T, **kw)
    nc = (p.T + p.chunk - 1) // p.chunk
    F = torch.empty(p.B, p.H, nc, p.d_k, p.d_v, dtype=torch.float32, device=k.device)
    G = torch.empty_like(F)
    rc = lib().vdn_vda_boundary_states_noalloc(ctypes.byref(p), _ptr(k), _ptr(v), _ptr(beta),
                                               _ptr(alpha), _ptr(text_k), _ptr(text_v), _ptr(F),
                                               _ptr(G), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_vda_boundary_states_noalloc")
    return F, G


def noalloc_device_status(stream=None) -> int:
    """Synchronise and return (and clear) the device status word of the last
    vda_boundary_states_noalloc call on the current device."""
    return lib().vdn_noalloc_device_status(_stream(stream))


def device_status(p: Optional[VdnParams], workspace, stream=None) -> int:
    """Synchronise and return (and clear) the device status of the last call
    (``p`` may be None, e.g. for the VDA-Prep workspace)."""
    return lib().vdn_device_status(None if p is None else ctypes.byref(p), _ptr(workspace),
                                   _stream(stream))


def selftest_bounded_wait(workspace, limit_us: int, stream=None) -> int:
    """Enqueue the bounded-wait self-test (a wait that nothing satisfies)."""
    return lib().vdn_selftest_bounded_wait(_ptr(workspace), int(limit_us), _stream(stream))


def mxfp8_quantize(x, rows_padded=None, stream=None):
    """(codes uint8 [rows, cols], scales uint8 [atoms * 512]) of an fp16 device
    matrix x [rows, cols] (vdn_mxfp8_quantize; cols a multiple of 128)."""
    import torch
    if x.dtype != torch.float16 or x.dim() != 2:
        raise ValueError("x must be a 2-D float16 tensor")
    rows, cols = x.shape
    rp = rows if rows_padded is None else rows_padded
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=x.device)
    nbytes = ((rp + 127) // 128) * (cols // 128) * 512
    scales = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    rc = lib().vdn_mxfp8_quantize(_ptr(x), rows, rp, cols, _ptr(codes), _ptr(scales), nbytes,
                                  _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_mxfp8_quantize")
    return codes, scales


def selftest_exp2(x, stream=None):
    """2^x (float32 device tensor) through the Softmax kernel's FMA-pipe
    exponential (vdn_selftest_exp2)."""
    import torch
    if x.dtype != torch.float32:
        raise ValueError("x must be float32")
    y = torch.empty_like(x)
    rc = lib().vdn_selftest_exp2(_ptr(x), _ptr(y), x.numel(), _stream(stream))
    if rc != 0:
        raise VdnError(rc, "vdn_selftest_exp2")
    return y


def use_tc_params(p: VdnParams) -> bool:
    """True when the call runs the tensor-core kernels (bf16, d in {64, 128})."""
    return p.dtype == VDN_BF16 and p.d_k in (64, 128) and not (p.flags & FLAG_SIMT)


class HostPipeline:
    """End-to-end forwards on host (pinned) tensors with the copies overlapped.

    Each ``submit`` is one vdn_hybrid_attn_fwd_host call: host -> device copies
    of every input (copy stream), the forward (compute stream), and the
    device -> host copy of ``out`` (copy-back stream), ordered by the events of
    the step's slot.  Two slots of device buffers alternate, so step i+1's
    uploads and step i-1's download run while step i computes.  Host input and
    output tensors must stay untouched until ``synchronize`` (or until the slot
    is reused two steps later).
    """

    def __init__(self, host_example: dict, T, *, params=None, **kw):
        import torch
        self.T = T
        dev = torch.device("cuda", torch.cuda.current_device())
        self.dev = dev
        if params is None:
            q, W = host_example["q"], host_example["W_soft"]
            B, L, H, d = q.shape
            tk = host_example.get("text_k")
            params = make_params(B, H, T, L // T, d, 0 if tk is None else tk.shape[1],
                                 _dtype_name(q), D_out=W.shape[1], **kw)
        self.params = p = params
        self.slots = [HostSlot(host_example, p, dev) for _ in range(2)]
        self.ws = alloc_workspace(p, dev)
        self.s_h2d = torch.cuda.Stream(dev)
        self.s_cmp = torch.cuda.Stream(dev)
        self.s_d2h = torch.cuda.Stream(dev)
        self.step = 0

    def submit(self, host: dict, out_host):
        """Enqueue one forward; returns (h2d_bytes, d2h_bytes)."""
        slot = self.slots[self.step % 2]
        self.step += 1
        return host_fwd_step(self.params, host, out_host, slot, self.ws, self.s_h2d, self.s_cmp,
                             self.s_d2h)

    def inputs_read_event(self, i: int):
        """cudaEvent_t handle (int) recorded after the forward of slot i read
        its inputs (valid once the slot was used)."""
        return self.slots[i].c.events[1]

    def synchronize(self):
        for s in (self.s_h2d, self.s_cmp, self.s_d2h):
            s.synchronize()

    def close(self):
        self.synchronize()
        for sl in self.slots:
            sl.release()
