"""Plain, slow, float64 CPU oracle for the VDN hybrid attention forward.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or runs
this module; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may use it.  It shares no code with the CUDA library.

Source: "Video DeltaNet: A Video-Native Hybrid Attention for Livestream Video
Generation" (Xi et al.), method section.  The pages lost every displayed
equation, so each function states the reading it implements:

* Softmax branch -- the paragraph on the local window (chunk-aligned window, the
  two boundary anchors with four-way connectivity, anchor entries counted
  once).
* Linear branch -- the paragraph on bidirectional linear attention (forward and
  reverse regions outside the window, anchors excluded, decay bridge,
  text-aware initial state counted once) and the Video Delta Attention
  paragraphs (joint objective, normal equation, inverse in key space,
  Proposition 1).
* Output -- the paragraph on the two output gates (sigmoid gates, RMS norm of
  the linear readout, separate output projections that are added).

Readings where the pages are silent (all are listed with reasons in the
design notes):
  R1  S_t = (I + A_t)^-1 (Diag(alpha_t) S_{t-1} + W_t),
      A_t = sum_i beta_t k_i k_i^T,  W_t = sum_i beta_t k_i v_i^T,
      state d_k x d_v, readout q^T S.
  R2  chunk grid starts at frame 0; window = chunks c-r..c+r, shrunk (not
      shifted) at the clip ends; partial last chunk allowed.
  R3  anchor query frames (0 and T-1) have empty linear regions; they read
      the text state only.
  R4  frames excluded from a scan (anchors) still apply their decay.
  R5  each directional scan starts from 1/2 S_text (text counted once in the
      sum); ``text_full=True`` starts both from S_text instead.
  R6  the bridge decays from the window edge up to and including the query
      frame; alpha defaults to 1.
  R11 softmax scale 1/sqrt(d_k); RMS norm over d_v, eps 1e-6, no weight.

Layouts: q, k, v [B, L, H, d] with token index t*N + n; text_k/text_v
[B, n_text, H, d]; beta [B, H, 1+T] (index 0 = text) per frame, or with
``beta_per_token`` [B, H, n_text + L] (text tokens first); alpha [B, H, T, d_k]
or None; gates [2, B, L, H, d_v]; W_soft/W_lin [H*d_v, D_out]; out
[B, L, D_out].
"""
from __future__ import annotations

import numpy as np

F64 = np.float64


# ----------------------------------------------------------------------------
# Frame sets (Softmax window + anchors; linear regions)
# ----------------------------------------------------------------------------

def anchor_frames(T: int) -> set:
    """The two boundary anchors: the first and the last latent frame
    (the paragraph on the local window, boundary anchors)."""
    return {0, T - 1}


def window_frames(t_q: int, T: int, chunk: int, radius: int) -> list:
    """Frames of the chunk-aligned window of query frame t_q: its own chunk and
    ``radius`` chunks on each side, clipped to the clip (reading R2)."""
    c = t_q // chunk
    lo = max(0, (c - radius) * chunk)
    hi = min(T, (c + radius + 1) * chunk)
    return list(range(lo, hi))


def softmax_key_frames(t_q: int, T: int, chunk: int, radius: int) -> list:
    """Key frames visible to query frame t_q in the Softmax branch: an anchor
    query sees every frame; any other query sees its window plus both anchors,
    each frame once (method: an anchor frame that also lies in the window
    is not counted twice)."""
    A = anchor_frames(T)
    if t_q in A:
        return list(range(T))
    return sorted(set(window_frames(t_q, T, chunk, radius)) | A)


def forward_region(t_q: int, T: int, chunk: int, radius: int) -> list:
    """Frames summarised by the forward state of query frame t_q: all frames
    before its window, anchors excluded; empty for anchor queries (R3)."""
    A = anchor_frames(T)
    if t_q in A:
        return []
    lo = window_frames(t_q, T, chunk, radius)[0]
    return [t for t in range(0, lo) if t not in A]


def reverse_region(t_q: int, T: int, chunk: int, radius: int) -> list:
    """Frames summarised by the reverse state: all frames after the window,
    anchors excluded; empty for anchor queries (R3)."""
    A = anchor_frames(T)
    if t_q in A:
        return []
    hi = window_frames(t_q, T, chunk, radius)[-1] + 1
    return [t for t in range(hi, T) if t not in A]


def frame_mask(T: int, chunk: int, radius: int) -> np.ndarray:
    """[T, T] boolean: M[f_q, f_k] = key frame f_k visible to query frame f_q."""
    M = np.zeros((T, T), dtype=bool)
    for t in range(T):
        M[t, softmax_key_frames(t, T, chunk, radius)] = True
    return M


def token_mask(T: int, N: int, chunk: int, radius: int, rows=None) -> np.ndarray:
    """Explicit dense token mask [len(rows) or L, L] expanded from the frame
    mask (every token of a frame shares its frame's visibility)."""
    Mf = frame_mask(T, chunk, radius)
    L = T * N
    rows = np.arange(L) if rows is None else np.asarray(rows)
    fq = rows // N
    fk = np.arange(L) // N
    return Mf[fq][:, fk]


# ----------------------------------------------------------------------------
# Softmax branch
# ----------------------------------------------------------------------------

def softmax_branch(q, k, v, T, N, chunk=5, radius=1, scale=None, rows=None,
                   row_block=512, text_k=None, text_v=None):
    """Exact masked Softmax attention for every (b, h), float64.

    o_s[i] = sum_j softmax_j(scale * q_i . k_j  over visible j) v_j, computed
    densely against all L keys with the explicit mask (-inf outside), the row
    maximum subtracted before exp.  ``rows`` selects query tokens.

    With ``text_k`` / ``text_v`` ([B, n_text, H, d]) every video query also
    sees all text tokens, under the same normaliser (method: the text keeps
    its Softmax path; reading: one joint Softmax over the visible video keys
    and the text keys).
    Returns [B, R, H, d_v].
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    B, L, H, dk = q.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    with_text = text_k is not None and np.asarray(text_k).shape[1] > 0
    if with_text:
        k = np.concatenate([k, np.asarray(text_k, F64)], axis=1)
        v = np.concatenate([v, np.asarray(text_v, F64)], axis=1)
    rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), H, v.shape[-1]), F64)
    for r0 in range(0, len(rows), row_block):
        rr = rows[r0:r0 + row_block]
        mask = token_mask(T, N, chunk, radius, rr)  # [R, L]
        if with_text:
            mask = np.concatenate([mask, np.ones((len(rr), k.shape[1] - L), bool)], axis=1)
        for b in range(B):
            for h in range(H):
                s = scale * (q[b, rr, h, :] @ k[b, :, h, :].T)  # [R, L (+ n_text)]
                s = np.where(mask, s, -np.inf)
                s = s - s.max(axis=1, keepdims=True)
                p = np.exp(s)
                p /= p.sum(axis=1, keepdims=True)
                out[b, r0:r0 + len(rr), h, :] = p @ v[b, :, h, :]
    return out


def text_query_branch(text_q, k, v, text_k, text_v, scale=None, rows=None):
    """Softmax attention of the text tokens as queries: every text query sees
    every video key and every text key under one normaliser, with no mask
    (reading of the joint Softmax with text: text rows are dense over the
    clip).  text_q, text_k, text_v [B, n_text, H, d]; k, v [B, L, H, d].
    Returns [B, R, H, d_v] for the selected text rows."""
    tq = np.asarray(text_q, F64)
    kk = np.concatenate([np.asarray(k, F64), np.asarray(text_k, F64)], axis=1)
    vv = np.concatenate([np.asarray(v, F64), np.asarray(text_v, F64)], axis=1)
    B, nt, H, dk = tq.shape
    if scale is None:
        scale = 1.0 / np.sqrt(dk)
    rows = np.arange(nt) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), H, vv.shape[-1]), F64)
    for b in range(B):
        for h in range(H):
            s = scale * (tq[b, rows, h, :] @ kk[b, :, h, :].T)
            s = s - s.max(axis=1, keepdims=True)
            p = np.exp(s)
            p /= p.sum(axis=1, keepdims=True)
            out[b, :, h, :] = p @ vv[b, :, h, :]
    return out


# ----------------------------------------------------------------------------
# Video Delta Attention
# ----------------------------------------------------------------------------

def frame_stats(K, V, beta):
    """Frame statistics of one frame: A = sum_i beta_i k_i k_i^T (d_k x d_k)
    and W = sum_i beta_i k_i v_i^T (d_k x d_v); K [n, d_k], V [n, d_v]
    (Video Delta Attention, frame statistics).  ``beta`` is one write gate for
    the frame (reading R7) or one per token ([n])."""
    K = np.asarray(K, F64)
    V = np.asarray(V, F64)
    if np.ndim(beta) == 0:
        return beta * (K.T @ K), beta * (K.T @ V)
    bK = np.asarray(beta, F64)[:, None] * K
    return K.T @ bK, bK.T @ V


def vda_solve(A, W, S_prev, alpha=None):
    """VDA frame update from precomputed frame statistics (reading R1).

    The new state minimises 1/2 ||S - S~||^2 + 1/2 sum_i beta ||S^T k_i - v_i||^2
    with S~ = Diag(alpha) S_prev (the decayed inherited state); setting the
    gradient to zero gives the normal equation (I + A) S = S~ + W, solved in
    key-channel space.
    """
    dk = A.shape[0]
    S_tilde = decay(np.asarray(S_prev, F64), alpha)
    return np.linalg.solve(np.eye(dk) + A, S_tilde + W)


def frozen_solve(A, W, S_prev, alpha=None):
    """Frozen-state (SANA-WM) batched frame update from the same statistics,
    the comparison rule of the Video Delta Attention section: every token's
    correction is evaluated at the same decayed state S~ = Diag(alpha) S_prev,
    S = S~ + sum_i beta_i k_i (v_i - S~^T k_i)^T = (I - A) S~ + W.  (The
    pages also scale SANA-WM's keys by a frame-size factor whose symbol was
    lost; keys are taken as given, so a caller applies any such factor.)"""
    S_tilde = decay(np.asarray(S_prev, F64), alpha)
    return S_tilde - A @ S_tilde + W


def vda_update(S_prev, K, V, beta, alpha=None, frozen=False):
    """One Video Delta Attention frame update from the frame's keys K [n, d_k],
    values V [n, d_v] and write gate beta (``frozen``: the frozen-state rule
    instead)."""
    A, W = frame_stats(K, V, beta)
    return (frozen_solve if frozen else vda_solve)(A, W, S_prev, alpha)


def decay(S, alpha):
    """Decay-only step Diag(alpha) S (anchors inside a scan, the bridge)."""
    if alpha is None:
        return S
    return np.asarray(alpha, F64)[:, None] * S


def text_state(text_k, text_v, beta0, frozen=False):
    """S_text: the text tokens as one leading virtual frame, updated from the
    zero state (method, the text-aware initial state of both scans)."""
    text_k = np.asarray(text_k, F64)
    text_v = np.asarray(text_v, F64)
    S0 = np.zeros((text_k.shape[1], text_v.shape[1]), F64)
    return vda_update(S0, text_k, text_v, beta0, frozen=frozen)


def _frame_beta(beta_bh, t, N, n_text, per_token):
    """Write gate(s) of video frame t: beta[1 + t], or its N per-token gates."""
    if per_token:
        return beta_bh[n_text + t * N:n_text + (t + 1) * N]
    return beta_bh[1 + t]


def _text_beta(beta_bh, n_text, per_token):
    return beta_bh[:n_text] if per_token else beta_bh[0]


class _FrameStats:
    """Lazily computed frame statistics (A_t, W_t) of one (b, h): a cache of
    the plain definition, so that the literal per-query recurrence below does
    not recompute K_t^T K_t for every query."""

    def __init__(self, k_bh, v_bh, beta_bh, N, n_text=0, per_token=False):
        self.k, self.v, self.beta, self.N = k_bh, v_bh, beta_bh, N
        self.n_text, self.per_token = n_text, per_token
        self.cache = {}

    def __call__(self, t):
        if t not in self.cache:
            N = self.N
            self.cache[t] = frame_stats(self.k[t * N:(t + 1) * N], self.v[t * N:(t + 1) * N],
                                        _frame_beta(self.beta, t, N, self.n_text,
                                                    self.per_token))
        return self.cache[t]


def _scan_outside_window(stats, alpha_bh, init, T, lo, hi, frozen=False):
    """Forward state after frames [0, lo) and reverse state after frames
    [hi, T), each run frame by frame from ``init``; anchors decay only (R4)."""
    A = anchor_frames(T)
    solve = frozen_solve if frozen else vda_solve

    def al(t):
        return None if alpha_bh is None else alpha_bh[t]

    Sf = init.copy()
    for t in range(0, lo):
        Sf = decay(Sf, al(t)) if t in A else solve(*stats(t), Sf, al(t))
    Sr = init.copy()
    for t in range(T - 1, hi - 1, -1):
        Sr = decay(Sr, al(t)) if t in A else solve(*stats(t), Sr, al(t))
    return Sf, Sr


def linear_branch(q, k, v, beta, text_k, text_v, T, N, chunk=5, radius=1,
                  alpha=None, rows=None, text_full=False, beta_per_token=False,
                  frozen=False):
    """Linear (VDA) branch readout o_l = q^T S_f + q^T S_r for every (b, h)
    (method: the distant-context output adds the forward and reverse readouts).

    For each query chunk the two states are recomputed literally, frame by
    frame, from the text initial state: forward over every frame before the
    window, reverse over every frame after it (anchors decay only, R4).  Each
    query frame then bridges them with decay only across the window frames
    between the window edge and itself, inclusive (R6).  Anchor queries read
    1/2 S_text from each direction (R3).  The scan starts from 1/2 S_text
    (R5; ``text_full`` starts from S_text).  ``frozen``: every frame update
    (text frame included) follows the frozen-state rule (frozen_solve).
    Returns [B, R, H, d_v] (before RMS norm and gate).
    """
    q = np.asarray(q, F64)
    k = np.asarray(k, F64)
    v = np.asarray(v, F64)
    beta = np.asarray(beta, F64)
    text_k = np.asarray(text_k, F64)
    text_v = np.asarray(text_v, F64)
    B, L, H, dk = q.shape
    dv = v.shape[-1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    out = np.zeros((B, len(rows), H, dv), F64)
    frames = rows // N
    Aset = anchor_frames(T)
    nt = text_k.shape[1]
    for b in range(B):
        for h in range(H):
            S_text = text_state(text_k[b, :, h, :], text_v[b, :, h, :],
                                _text_beta(beta[b, h], nt, beta_per_token), frozen)
            init = S_text if text_full else 0.5 * S_text
            al = None if alpha is None else np.asarray(alpha, F64)[b, h]
            stats = _FrameStats(k[b, :, h, :], v[b, :, h, :], beta[b, h], N, nt, beta_per_token)
            per_chunk = {}
            for t_q in np.unique(frames):
                t_q = int(t_q)
                if t_q in Aset:
                    Sf, Sr = init, init
                else:
                    win = window_frames(t_q, T, chunk, radius)
                    lo, hi = win[0], win[-1] + 1
                    c = t_q // chunk
                    if c not in per_chunk:
                        per_chunk[c] = _scan_outside_window(stats, al, init, T, lo, hi,
                                                            frozen)
                    Sf, Sr = per_chunk[c]
                    for t in range(lo, t_q + 1):          # forward bridge
                        Sf = decay(Sf, None if al is None else al[t])
                    for t in range(hi - 1, t_q - 1, -1):  # reverse bridge
                        Sr = decay(Sr, None if al is None else al[t])
                sel = np.nonzero(frames == t_q)[0]
                qq = q[b, rows[sel], h, :]
                out[b, sel, h, :] = qq @ Sf + qq @ Sr
    return out


# ----------------------------------------------------------------------------
# Gated dual output projection
# ----------------------------------------------------------------------------

def rms_norm(o, eps=1e-6):
    """RMS normalisation over the value channels of each (token, head), no
    weight (R11)."""
    o = np.asarray(o, F64)
    return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)


def output_projection(o_s, o_l, g_s, g_l, W_soft, W_lin, eps=1e-6):
    """out = concat_h(g_s * o_s) W_soft + concat_h(g_l * RMS(o_l)) W_lin
    (separate output projections of the two gated branches, added)."""
    o_s = np.asarray(o_s, F64)
    B, R, H, dv = o_s.shape
    xs = (np.asarray(g_s, F64) * o_s).reshape(B, R, H * dv)
    xl = (np.asarray(g_l, F64) * rms_norm(o_l, eps)).reshape(B, R, H * dv)
    return xs @ np.asarray(W_soft, F64) + xl @ np.asarray(W_lin, F64)


def hybrid_forward(inp: dict, T, N, chunk=5, radius=1, scale=None, eps=1e-6,
                   rows=None, text_full=False, text_softmax=False, beta_per_token=False,
                   frozen=False):
    """The whole hybrid attention forward on the selected query rows.

    ``inp`` holds numpy (or torch CPU) arrays with the keys q, k, v, beta,
    alpha (or None), text_k, text_v, W_soft, W_lin, gates, and optionally
    q_lin, k_lin, v_lin: the linear branch's own inputs (its feature map of
    the projections); without them both branches read q, k, v.
    ``text_softmax``: video queries also attend all text tokens in the
    Softmax branch (one normaliser).
    Returns (out [B, R, D_out], o_s [B, R, H, d_v], o_l [B, R, H, d_v]).
    """
    a = {k: (None if v is None else np.asarray(_to_np(v), F64)) for k, v in inp.items()}
    L = a["q"].shape[1]
    rows = np.arange(L) if rows is None else np.asarray(rows)
    o_s = softmax_branch(a["q"], a["k"], a["v"], T, N, chunk, radius, scale, rows,
                         text_k=a["text_k"] if text_softmax else None,
                         text_v=a["text_v"] if text_softmax else None)
    ql = a["q_lin"] if a.get("q_lin") is not None else a["q"]
    kl = a["k_lin"] if a.get("k_lin") is not None else a["k"]
    vl = a["v_lin"] if a.get("v_lin") is not None else a["v"]
    o_l = linear_branch(ql, kl, vl, a["beta"], a["text_k"], a["text_v"],
                        T, N, chunk, radius, a.get("alpha"), rows, text_full, beta_per_token,
                        frozen)
    g = a["gates"]
    out = output_projection(o_s, o_l, g[0][:, rows], g[1][:, rows], a["W_soft"],
                            a["W_lin"], eps)
    return out, o_s, o_l


def boundary_states(k, v, beta, text_k, text_v, T, N, chunk=5, radius=1,
                    alpha=None, text_full=False, beta_per_token=False, frozen=False):
    """For every (b, h) and query chunk c, the forward and reverse states that
    a query of chunk c reads before its bridge: forward = after all frames
    before the window, reverse = after all frames after the window, each
    computed literally, frame by frame, for that chunk.
    Returns F, G with shape [B, H, n_chunks, d_k, d_v]."""
    k = np.asarray(_to_np(k), F64)
    v = np.asarray(_to_np(v), F64)
    beta = np.asarray(_to_np(beta), F64)
    text_k = np.asarray(_to_np(text_k), F64)
    text_v = np.asarray(_to_np(text_v), F64)
    B, L, H, dk = k.shape
    dv = v.shape[-1]
    nc = (T + chunk - 1) // chunk
    F = np.zeros((B, H, nc, dk, dv))
    G = np.zeros((B, H, nc, dk, dv))
    nt = text_k.shape[1]
    for b in range(B):
        for h in range(H):
            S_text = text_state(text_k[b, :, h, :], text_v[b, :, h, :],
                                _text_beta(beta[b, h], nt, beta_per_token), frozen)
            init = S_text if text_full else 0.5 * S_text
            al = None if alpha is None else np.asarray(_to_np(alpha), F64)[b, h]
            stats = _FrameStats(k[b, :, h, :], v[b, :, h, :], beta[b, h], N, nt, beta_per_token)
            for c in range(nc):
                lo = max(0, (c - radius) * chunk)
                hi = min(T, (c + radius + 1) * chunk)
                F[b, h, c], G[b, h, c] = _scan_outside_window(stats, al, init, T, lo, hi,
                                                              frozen)
    return F, G


def _to_np(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (CPU); bf16 has no numpy dtype
        import torch
        return x.detach().to(torch.float64).cpu().numpy()
    return np.asarray(x)
