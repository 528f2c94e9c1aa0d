"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol the header declares, and validates its arguments before any
launch."""
import ctypes
import os
import re

import pytest

import softmax_attention_video_chunk_b200 as vdn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built_lib():
    from softmax_attention_video_chunk_b200 import _build
    if _build.needs_build():
        _build.build()
    return vdn.lib()


def _declared_symbols():
    src = open(os.path.join(ROOT, "include", "vdn.h")).read()
    return re.findall(r"VDN_API[^;{]*?\b(vdn_\w+)\s*\(", src)


def test_exports_every_declared_symbol():
    syms = _declared_symbols()
    assert len(syms) >= 8
    L = vdn.lib()
    for s in syms:
        assert hasattr(L, s), s


def test_abi_version_and_strings():
    L = vdn.lib()
    assert L.vdn_abi_version() == 1
    for code in range(10):
        assert L.vdn_status_string(code)
    assert b"UNKNOWN" in L.vdn_status_string(99)


def test_params_init_defaults():
    p = vdn.VdnParams()
    assert vdn.lib().vdn_params_init(ctypes.byref(p), 1, 24, 75, 1536, 128, 512, vdn.VDN_BF16) == 0
    assert (p.chunk, p.window_radius, p.D_out, p.out_dtype) == (5, 1, 24 * 128, vdn.VDN_F32)
    assert abs(p.rms_eps - 1e-6) < 1e-12 and p.softmax_scale == 0.0


@pytest.mark.parametrize("field,value,code", [
    ("B", 0, "VDN_ERR_SHAPE"), ("T", 0, "VDN_ERR_SHAPE"), ("N", 0, "VDN_ERR_SHAPE"),
    ("chunk", 0, "VDN_ERR_SHAPE"), ("window_radius", -1, "VDN_ERR_SHAPE"),
    ("n_text", -1, "VDN_ERR_SHAPE"), ("D_out", 12, "VDN_ERR_SHAPE"),
    ("d_v", 32, "VDN_ERR_UNSUPPORTED"), ("dtype", 7, "VDN_ERR_DTYPE"),
    ("out_dtype", 3, "VDN_ERR_DTYPE"), ("flags", 1 << 8, "VDN_ERR_INVALID_ARG"),
    ("softmax_scale", -1.0, "VDN_ERR_INVALID_ARG"), ("rms_eps", float("nan"), "VDN_ERR_INVALID_ARG"),
])
def test_param_validation(field, value, code):
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    setattr(p, field, value)
    size = ctypes.c_size_t(0)
    rc = vdn.lib().vdn_workspace_bytes(ctypes.byref(p), ctypes.byref(size))
    assert vdn.STATUS[rc] == code


def test_unsupported_head_dim():
    p = vdn.VdnParams()
    rc = vdn.lib().vdn_params_init(ctypes.byref(p), 1, 2, 15, 16, 48, 8, vdn.VDN_BF16)
    assert vdn.STATUS[rc] == "VDN_ERR_UNSUPPORTED"


def test_workspace_grows_with_problem():
    small = vdn.workspace_bytes(vdn.make_params(1, 2, 15, 16, 64, 8, "bf16"))
    big = vdn.workspace_bytes(vdn.make_params(1, 2, 30, 16, 64, 8, "bf16"))
    assert 0 < small < big
    # 768p-shaped workload: transitions, chunk maps, states, V^T, W^T, x
    p = vdn.make_params(1, 24, 75, 1536, 128, 512, "bf16")
    ws = vdn.workspace_bytes(p)
    assert 2.0e9 < ws < 4.0e9


def _call_fwd(p, ptrs, ws_ptr, ws_bytes):
    return vdn.lib().vdn_hybrid_attn_fwd(ctypes.byref(p), *ptrs, ws_ptr, ws_bytes, None)


def test_compute_entry_rejects_bad_arguments_before_launch():
    """Validation errors return before any CUDA call, so they are testable
    without a device (pointers are never dereferenced on this path)."""
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    need = vdn.workspace_bytes(p)
    good = [0x10000 + 0x1000 * i for i in range(11)]  # q k v beta alpha tk tv Ws Wl gates out
    good[4] = None  # alpha may be NULL
    ws = 0x7f0000000000
    # missing required pointer
    bad = list(good)
    bad[0] = None
    assert vdn.STATUS[_call_fwd(p, bad, ws, need)] == "VDN_ERR_INVALID_ARG"
    # misaligned pointer
    bad = list(good)
    bad[2] += 8
    assert vdn.STATUS[_call_fwd(p, bad, ws, need)] == "VDN_ERR_ALIGNMENT"
    # workspace too small / misaligned / missing
    assert vdn.STATUS[_call_fwd(p, good, ws, need - 1)] == "VDN_ERR_WORKSPACE"
    assert vdn.STATUS[_call_fwd(p, good, ws + 16, need)] == "VDN_ERR_ALIGNMENT"
    assert vdn.STATUS[_call_fwd(p, good, None, need)] == "VDN_ERR_WORKSPACE"
    # text pointers may be NULL only when n_text == 0
    bad = list(good)
    bad[5] = None
    assert vdn.STATUS[_call_fwd(p, bad, ws, need)] == "VDN_ERR_INVALID_ARG"


def test_branches_and_states_validate():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    need = vdn.workspace_bytes(p)
    L = vdn.lib()
    rc = L.vdn_hybrid_attn_branches(ctypes.byref(p), None, 0x1000, 0x2000, 0x3000, None, 0x4000,
                                    0x5000, 0x6000, 0x7000, 0x7f0000000000, need, None)
    assert vdn.STATUS[rc] == "VDN_ERR_INVALID_ARG"
    rc = L.vdn_vda_boundary_states(ctypes.byref(p), 0x1000, 0x2000, 0x3000, None, 0x4000, 0x5000,
                                   0x6008, None, 0x7f0000000000, need, None)
    assert vdn.STATUS[rc] == "VDN_ERR_ALIGNMENT"
    assert vdn.STATUS[L.vdn_device_status(ctypes.byref(p), None, None)] == "VDN_ERR_WORKSPACE"


def _prep_call(p, ptrs, ws=0x7000, ws_bytes=256):
    L = vdn.lib()
    return vdn.STATUS[L.vdn_vda_prep(ctypes.byref(p), *[ctypes.c_void_p(x) for x in ptrs],
                                     ctypes.c_void_p(ws), ws_bytes, None)]


def test_prep_params_defaults_and_validation():
    p = vdn.make_prep_params(1, 24, 75, 32, 48, 128, "bf16")
    assert (p.spatial_taps, p.temporal_taps) == (3, 5) and abs(p.l2_eps - 1e-6) < 1e-12
    L = vdn.lib()
    for field, value, code in [("d", 96, "VDN_ERR_UNSUPPORTED"), ("spatial_taps", 5, "VDN_ERR_UNSUPPORTED"),
                               ("temporal_taps", 3, "VDN_ERR_UNSUPPORTED"), ("grid_w", 0, "VDN_ERR_SHAPE"),
                               ("T", 0, "VDN_ERR_SHAPE"), ("dtype", 4, "VDN_ERR_DTYPE"),
                               ("l2_eps", -1.0, "VDN_ERR_INVALID_ARG"),
                               ("grid_h", 70000, "VDN_ERR_SHAPE"), ("H", 40000, "VDN_ERR_SHAPE")]:
        q = vdn.make_prep_params(1, 2, 4, 3, 5, 64, "bf16")
        setattr(q, field, value)
        ptrs = [0x1000 * (i + 1) for i in range(10)]
        assert _prep_call(q, ptrs) == code, field


def test_prep_rejects_bad_arguments_before_launch():
    p = vdn.make_prep_params(1, 2, 4, 3, 5, 64, "bf16")
    n = 4 * 15 * 2 * 64 * 2  # bytes of one tensor
    # q k v wk_s wk_t wv_s wv_t q_out k_out v_out
    base = [0x100000 * (i + 1) for i in range(10)]
    assert _prep_call(p, [0] * 10) == "VDN_ERR_INVALID_ARG"  # nothing to do
    bad = list(base)
    bad[1] = 0  # k missing while v present
    assert _prep_call(p, bad) == "VDN_ERR_INVALID_ARG"
    bad = list(base)
    bad[3] = 0x400008  # misaligned filter
    assert _prep_call(p, bad) == "VDN_ERR_ALIGNMENT"
    bad = list(base)
    bad[8] = base[2] + n // 2  # k_out overlaps v
    assert _prep_call(p, bad) == "VDN_ERR_INVALID_ARG"
    bad = list(base)
    bad[9] = bad[8]  # k_out == v_out
    assert _prep_call(p, bad) == "VDN_ERR_INVALID_ARG"
    assert _prep_call(p, [base[0]] + [0] * 9) == "VDN_ERR_INVALID_ARG"  # q without q_out
    assert _prep_call(p, base, ws=0) == "VDN_ERR_WORKSPACE"
    assert _prep_call(p, base, ws_bytes=255) == "VDN_ERR_WORKSPACE"
    assert _prep_call(p, base, ws=0x7010) == "VDN_ERR_ALIGNMENT"


def test_split_forward_requires_linear_inputs():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    L = vdn.lib()
    ptr = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(14)]
    ptr[3] = ctypes.c_void_p(0)  # q_lin missing
    rc = L.vdn_hybrid_attn_fwd_split(ctypes.byref(p), *ptr, ctypes.c_void_p(0x80000),
                                     1 << 40, None, None)
    assert vdn.STATUS[rc] == "VDN_ERR_INVALID_ARG"


def test_text_query_attn_validates_before_launch():
    L = vdn.lib()
    ptr = [ctypes.c_void_p(0x1000 * (i + 1)) for i in range(6)]  # text_q k v text_k text_v o_text
    p = vdn.make_params(1, 2, 15, 16, 64, 0, "bf16")  # no text tokens
    rc = L.vdn_text_query_attn(ctypes.byref(p), *ptr, ctypes.c_void_p(0x80000), 1 << 40, None)
    assert vdn.STATUS[rc] == "VDN_ERR_SHAPE"
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    bad = list(ptr)
    bad[0] = ctypes.c_void_p(0)  # text_q missing
    rc = L.vdn_text_query_attn(ctypes.byref(p), *bad, ctypes.c_void_p(0x80000), 1 << 40, None)
    assert vdn.STATUS[rc] == "VDN_ERR_INVALID_ARG"
    # the workspace must hold the text tokens' V^T (sized as with VDN_FLAG_TEXT_SOFTMAX)
    need = vdn.workspace_bytes(vdn.make_params(1, 2, 15, 16, 64, 8, "bf16", text_softmax=True))
    assert need > vdn.workspace_bytes(p)
    rc = L.vdn_text_query_attn(ctypes.byref(p), *ptr, ctypes.c_void_p(0x80000),
                               vdn.workspace_bytes(p), None)
    assert vdn.STATUS[rc] == "VDN_ERR_WORKSPACE"


def test_frozen_state_flag_is_accepted():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16", frozen_state=True)
    assert p.flags & vdn.FLAG_FROZEN_STATE
    assert vdn.workspace_bytes(p) == vdn.workspace_bytes(vdn.make_params(1, 2, 15, 16, 64, 8))


def test_host_entry_validates_before_any_copy():
    """vdn_hybrid_attn_fwd_host checks the host inputs, the slot's device
    buffers and the workspace before it enqueues anything."""
    L = vdn.lib()
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    need = vdn.workspace_bytes(p)
    ws = 0x7f0000000000
    hi = vdn.VdnHostInputs()
    slot = vdn.VdnHostSlot()
    for i, f in enumerate(vdn._HOST_FIELDS):
        setattr(hi, f, 0x100000 + 0x1000 * i)
        setattr(slot, f, 0x200000 + 0x1000 * i)
    hi.alpha = slot.alpha = None
    slot.out = 0x300000

    def call(host_in=hi, out=0x400000, sl=slot, w=ws, nbytes=need):
        h2d, d2h = ctypes.c_size_t(0), ctypes.c_size_t(0)
        return vdn.STATUS[L.vdn_hybrid_attn_fwd_host(
            ctypes.byref(p), None if host_in is None else ctypes.byref(host_in), out,
            None if sl is None else ctypes.byref(sl), w, nbytes, None, None, None,
            ctypes.byref(h2d), ctypes.byref(d2h))]

    assert call(host_in=None) == "VDN_ERR_INVALID_ARG"
    assert call(sl=None) == "VDN_ERR_INVALID_ARG"
    assert call(out=None) == "VDN_ERR_INVALID_ARG"
    assert call(nbytes=need - 1) == "VDN_ERR_WORKSPACE"
    assert call(w=ws + 64) == "VDN_ERR_ALIGNMENT"
    hi.alpha = 0x500000  # a host alpha without a device buffer for it
    assert call() == "VDN_ERR_INVALID_ARG"
    hi.alpha = None
    slot.gates = None  # a required device buffer missing
    assert call() == "VDN_ERR_INVALID_ARG"
    slot.gates = 0x200008  # misaligned
    assert call() == "VDN_ERR_ALIGNMENT"
    slot.gates = 0x209000
    slot.out = None
    assert call() == "VDN_ERR_INVALID_ARG"
    assert slot.used == 0 and all(e is None for e in slot.events)  # nothing was created
    assert L.vdn_host_slot_release(None) == 0


def test_scan_flags_are_exclusive():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    size = ctypes.c_size_t(0)
    for f in (vdn.FLAG_SCAN_FRAMES, vdn.FLAG_SCAN_CHUNKS):
        p.flags = f
        assert vdn.lib().vdn_workspace_bytes(ctypes.byref(p), ctypes.byref(size)) == 0
    p.flags = vdn.FLAG_SCAN_FRAMES | vdn.FLAG_SCAN_CHUNKS
    rc = vdn.lib().vdn_workspace_bytes(ctypes.byref(p), ctypes.byref(size))
    assert vdn.STATUS[rc] == "VDN_ERR_INVALID_ARG"


def test_operand_and_projection_validate_before_launch():
    L = vdn.lib()
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    need = vdn.workspace_bytes(p)
    ws = 0x7f0000000000
    ptr = [0x10000 + 0x1000 * i for i in range(10)]
    # q k v beta alpha tk tv gates x
    args = [ptr[0], ptr[1], ptr[2], ptr[3], None, ptr[4], ptr[5], ptr[6], ptr[7]]
    bad = list(args)
    bad[8] = None  # no operand buffer
    assert vdn.STATUS[L.vdn_hybrid_attn_operand(ctypes.byref(p), *bad, ws, need, None)] == \
        "VDN_ERR_INVALID_ARG"
    bad = list(args)
    bad[8] = ptr[7] + 8  # misaligned
    assert vdn.STATUS[L.vdn_hybrid_attn_operand(ctypes.byref(p), *bad, ws, need, None)] == \
        "VDN_ERR_ALIGNMENT"
    ps = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16", simt=True)
    assert vdn.STATUS[L.vdn_hybrid_attn_operand(ctypes.byref(ps), *args, ws, need, None)] == \
        "VDN_ERR_UNSUPPORTED"
    pf = vdn.make_params(1, 2, 15, 16, 64, 8, "f32")
    assert vdn.STATUS[L.vdn_output_projection(ctypes.byref(pf), 10, ptr[0], ptr[1], ptr[2],
                                              ptr[3], ws, vdn.workspace_bytes(pf), None)] == \
        "VDN_ERR_UNSUPPORTED"
    for rows, code in ((0, "VDN_ERR_SHAPE"), (-5, "VDN_ERR_SHAPE"), (1 << 31, "VDN_ERR_SHAPE")):
        assert vdn.STATUS[L.vdn_output_projection(ctypes.byref(p), rows, ptr[0], ptr[1], ptr[2],
                                                  ptr[3], ws, need, None)] == code
    assert vdn.STATUS[L.vdn_output_projection(ctypes.byref(p), 10, ptr[0], None, ptr[2],
                                              ptr[3], ws, need, None)] == "VDN_ERR_INVALID_ARG"


def test_mxfp8_quantize_validates():
    L = vdn.lib()
    x, c, s = 0x10000, 0x20000, 0x30000
    need = 1 * 2 * 512  # 100 rows padded to 128, 256 columns
    for rows, rp, cols, code in ((0, 0, 256, "VDN_ERR_SHAPE"), (100, 99, 256, "VDN_ERR_SHAPE"),
                                 (100, 128, 200, "VDN_ERR_SHAPE"), (100, 128, 64, "VDN_ERR_SHAPE")):
        assert vdn.STATUS[L.vdn_mxfp8_quantize(x, rows, rp, cols, c, s, need, None)] == code
    assert vdn.STATUS[L.vdn_mxfp8_quantize(x, 100, 128, 256, c, s, need - 1, None)] == \
        "VDN_ERR_WORKSPACE"
    assert vdn.STATUS[L.vdn_mxfp8_quantize(x + 8, 100, 128, 256, c, s, need, None)] == \
        "VDN_ERR_ALIGNMENT"


def test_mxfp8_projection_needs_the_tensor_core_path():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "f32", proj_mxfp8=True)
    need = vdn.workspace_bytes(p)
    ptrs = [0x10000 + 0x1000 * i for i in range(11)]
    ptrs[4] = None
    rc = vdn.lib().vdn_hybrid_attn_fwd(ctypes.byref(p), *ptrs, 0x7f0000000000, need, None)
    assert vdn.STATUS[rc] == "VDN_ERR_UNSUPPORTED"
    # the workspace grows by the quantised operands and their scales
    a = vdn.workspace_bytes(vdn.make_params(1, 2, 15, 16, 64, 8, "bf16"))
    b = vdn.workspace_bytes(vdn.make_params(1, 2, 15, 16, 64, 8, "bf16", proj_mxfp8=True))
    assert b > a


@pytest.mark.parametrize("shape,dtype,flags,expect", [
    # 768p: 24 heads, 75 frames: the direct frame scan (75 sequential products
    # in one wave against 10 waves of composition + 15 scan steps)
    ((1, 24, 75, 1536, 128, 512), "bf16", 0, 7),
    ((1, 24, 75, 1536, 128, 512), "bf16", vdn.FLAG_SCAN_CHUNKS, 8),
    ((1, 24, 75, 1536, 128, 512), "bf16", vdn.FLAG_SCAN_FRAMES, 7),
    ((1, 24, 75, 1536, 128, 512), "bf16", vdn.FLAG_PROJ_MXFP8, 8),
    # few heads, 15 frames: composition fits one wave, so chunks win (8 + 3 < 15)
    ((1, 2, 15, 16, 64, 8), "bf16", 0, 8),
    # one chunk: the frame scan (2 products) beats composition (8 + 1)
    ((1, 2, 2, 16, 64, 8), "bf16", 0, 7),
    # text keys in the Softmax: the text values get their own V^T conversion
    ((1, 24, 75, 1536, 128, 512), "bf16", vdn.FLAG_TEXT_SOFTMAX, 8),
    ((1, 24, 75, 1536, 128, 0), "bf16", vdn.FLAG_TEXT_SOFTMAX, 7),
    # CUDA-core path: states (2 or 3), Softmax, readout, RMS factors, projection
    ((1, 24, 75, 1536, 128, 512), "f32", 0, 6),
    ((1, 2, 15, 16, 64, 8), "bf16", vdn.FLAG_SIMT, 7),
])
def test_forward_launch_count(shape, dtype, flags, expect):
    p = vdn.make_params(*shape, dtype)
    p.flags |= flags
    assert vdn.forward_launches(p) == expect


def test_forward_launch_count_validates():
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "bf16")
    assert vdn.STATUS[vdn.lib().vdn_forward_launches(ctypes.byref(p), None)] == "VDN_ERR_INVALID_ARG"
    p.chunk = 0
    with pytest.raises(vdn.VdnError):
        vdn.forward_launches(p)
    p = vdn.make_params(1, 2, 15, 16, 64, 8, "f32")
    p.flags |= vdn.FLAG_PROJ_MXFP8
    with pytest.raises(vdn.VdnError):
        vdn.forward_launches(p)
