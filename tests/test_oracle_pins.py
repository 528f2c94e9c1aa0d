"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a textbook
routine (token-level delta rule, least squares, dense softmax), a closed form,
an invariant stated on the pages, or brute-force enumeration on tiny inputs.
The pages print no worked numeric example (every displayed equation was lost
in extraction), so no printed values are available to pin.
"""
import itertools

import numpy as np
import pytest
import scipy.special

from oracle import vdn_oracle as O

rng_global = np.random.default_rng(0)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _delta_rule_token(S, k, v, beta_eff):
    """Textbook token-level delta rule (Gated DeltaNet form, without decay):
    read the prediction S^T k, write beta_eff * k (v - S^T k)^T."""
    pred = S.T @ k
    return S + beta_eff * np.outer(k, v - pred)


# --- Video Delta Attention frame update --------------------------------------

@pytest.mark.parametrize("seed", range(5))
def test_n1_reduces_to_token_delta_rule(seed):
    """With one token per frame, the VDA update equals the token-level delta
    rule with the effective write strength beta/(1 + beta ||k||^2)
    (Sherman-Morrison on (I + beta k k^T)^-1)."""
    rng = np.random.default_rng(seed)
    dk, dv = 6, 5
    S = rng.normal(size=(dk, dv))
    k = rng.normal(size=dk)          # not unit: exercises the ||k||^2 term
    v = rng.normal(size=dv)
    beta = rng.uniform(0.05, 3.0)
    alpha = rng.uniform(0.5, 1.0, size=dk)
    got = O.vda_update(S, k[None, :], v[None, :], beta, alpha)
    S_dec = alpha[:, None] * S
    want = _delta_rule_token(S_dec, k, v, beta / (1.0 + beta * k @ k))
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_joint_objective_least_squares(seed):
    """The frame update is the minimiser of 1/2||S - S~||^2 +
    1/2 sum_i beta ||S^T k_i - v_i||^2; solve the stacked least-squares system
    [I; sqrt(beta) K] S = [S~; sqrt(beta) V] with a generic routine."""
    rng = np.random.default_rng(100 + seed)
    dk, dv, n = 7, 4, 11
    S_prev = rng.normal(size=(dk, dv))
    K = _unit(rng.normal(size=(n, dk)))
    V = rng.normal(size=(n, dv))
    beta = rng.uniform(0.1, 2.0)
    alpha = rng.uniform(0.3, 1.0, size=dk)
    S_tilde = alpha[:, None] * S_prev
    Amat = np.vstack([np.eye(dk), np.sqrt(beta) * K])
    rhs = np.vstack([S_tilde, np.sqrt(beta) * V])
    want = np.linalg.lstsq(Amat, rhs, rcond=None)[0]
    got = O.vda_update(S_prev, K, V, beta, alpha)
    np.testing.assert_allclose(got, want, rtol=1e-10, atol=1e-10)
    # and the gradient of the objective vanishes there
    grad = (got - S_tilde) + beta * K.T @ (K @ got - V)
    assert np.abs(grad).max() < 1e-10


@pytest.mark.parametrize("seed", range(3))
def test_orthonormal_keys_decouple(seed):
    """With orthonormal keys (n <= d_k) the joint update equals independent
    token-level delta rules with beta/(1+beta), applied in any order."""
    rng = np.random.default_rng(200 + seed)
    dk, dv, n = 8, 3, 5
    Q, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    K = Q[:, :n].T
    V = rng.normal(size=(n, dv))
    S = rng.normal(size=(dk, dv))
    beta = rng.uniform(0.1, 2.0)
    got = O.vda_update(S, K, V, beta)
    for order in (range(n), reversed(range(n)), rng.permutation(n)):
        want = S.copy()
        for i in order:
            want = _delta_rule_token(want, K[i], V[i], beta / (1 + beta))
        np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-11)


def test_beta_zero_is_pure_decay():
    rng = np.random.default_rng(3)
    S = rng.normal(size=(6, 6))
    K = _unit(rng.normal(size=(9, 6)))
    V = rng.normal(size=(9, 6))
    alpha = rng.uniform(0, 1, size=6)
    np.testing.assert_allclose(O.vda_update(S, K, V, 0.0, alpha), alpha[:, None] * S,
                               rtol=0, atol=1e-14)


@pytest.mark.parametrize("seed", range(5))
def test_proposition1_non_expansive(seed):
    """Proposition 1: for alpha in [0,1] and beta >= 0 the inherited-state map
    is non-expansive in the spectral norm."""
    rng = np.random.default_rng(300 + seed)
    dk, dv, n = 10, 6, 30
    K = rng.normal(size=(n, dk))
    V = rng.normal(size=(n, dv))
    beta = rng.uniform(0, 5)
    alpha = rng.uniform(0, 1, size=dk)
    for _ in range(20):
        Sa = rng.normal(size=(dk, dv)) * rng.uniform(0.1, 10)
        Sb = rng.normal(size=(dk, dv)) * rng.uniform(0.1, 10)
        da = O.vda_update(Sa, K, V, beta, alpha) - O.vda_update(Sb, K, V, beta, alpha)
        assert np.linalg.norm(da, 2) <= np.linalg.norm(Sa - Sb, 2) * (1 + 1e-12)


def test_frozen_state_rule_differs_at_second_order():
    """The frozen-state batched rule S = (I - A) S~ + W (all corrections at the
    same decayed state) agrees with VDA to first order in beta; the gap
    shrinks ~4x when beta halves.  A sign error in the key-space inverse would
    make the gap first order (ratio ~2)."""
    rng = np.random.default_rng(7)
    dk, dv, n = 8, 5, 12
    K = _unit(rng.normal(size=(n, dk)))
    V = rng.normal(size=(n, dv))
    S = rng.normal(size=(dk, dv))

    def gap(beta):
        A, W = beta * K.T @ K, beta * K.T @ V
        frozen = (np.eye(dk) - A) @ S + W
        return np.linalg.norm(O.vda_update(S, K, V, beta) - frozen)

    r = gap(1e-3) / gap(5e-4)
    assert 3.8 < r < 4.2


def test_frozen_rule_is_the_sum_of_token_corrections_at_one_state():
    """The frozen-state rule, written as the pages define it: every token's
    correction beta_i k_i (v_i - S~^T k_i)^T is evaluated at the same decayed
    state S~ and all are added (explicit loop over tokens, per-token gates)."""
    rng = np.random.default_rng(11)
    dk, dv, n = 6, 4, 9
    K = rng.normal(size=(n, dk))
    V = rng.normal(size=(n, dv))
    S = rng.normal(size=(dk, dv))
    beta = rng.uniform(0.1, 0.9, size=n)
    alpha = rng.uniform(0.5, 1.0, size=dk)
    St = alpha[:, None] * S
    want = St.copy()
    for i in range(n):
        want += beta[i] * np.outer(K[i], V[i] - St.T @ K[i])
    got = O.vda_update(S, K, V, beta, alpha, frozen=True)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_frozen_rule_one_token_is_the_classic_delta_rule():
    """N = 1: S~ + beta k (v - S~^T k)^T, the one-token delta rule; VDA's
    (I + beta k k^T)^-1 (S~ + beta k v^T) differs from it."""
    rng = np.random.default_rng(12)
    k = rng.normal(size=5)
    v = rng.normal(size=3)
    S = rng.normal(size=(5, 3))
    want = S + 0.7 * np.outer(k, v - S.T @ k)
    got = O.vda_update(S, k[None], v[None], 0.7, frozen=True)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    assert np.linalg.norm(O.vda_update(S, k[None], v[None], 0.7) - want) > 1e-3


def test_frozen_transition_can_expand_where_vda_cannot():
    """Proposition 1 holds for VDA only: with beta ||k||^2 = 3 the frozen
    transition I - beta k k^T has an eigenvalue -2 (it amplifies the inherited
    state), while (I + beta k k^T)^-1 has spectral norm <= 1."""
    k = np.array([1.0, 0.0, 0.0])
    S0 = np.zeros((3, 2))
    dS = np.array([[1.0, 0.0], [0.0, 0.0], [0.0, 0.0]])
    v = np.zeros(2)

    def carried(frozen):
        return (O.vda_update(S0 + dS, k[None], v[None], 3.0, frozen=frozen) -
                O.vda_update(S0, k[None], v[None], 3.0, frozen=frozen))

    assert np.isclose(np.linalg.norm(carried(True)), 2.0)
    assert np.isclose(np.linalg.norm(carried(False)), 0.25)


def test_frozen_and_vda_agree_for_small_writes_in_the_forward():
    """Whole linear branch: the two rules agree to first order in beta and
    differ at beta of order 1."""
    import torch
    from synth import CONFIGS, make_inputs
    cfg = CONFIGS["tiny_f32"]
    inp = make_inputs(cfg)
    args = (inp["q"], inp["k"], inp["v"], None, inp["text_k"], inp["text_v"], cfg.T, cfg.N)
    rows = np.arange(0, cfg.L, 7)

    def run(beta, frozen):
        a = list(args)
        a[3] = torch.full((cfg.B, cfg.H, 1 + cfg.T), beta)
        return O.linear_branch(*a, rows=rows, frozen=frozen)

    def rel_gap(beta):
        ref = run(beta, False)
        return np.abs(run(beta, True) - ref).max() / np.abs(ref).max()

    # the output is O(beta) and the gap O(beta^2): the relative gap halves
    # with beta, and is large at beta of order 1
    r = rel_gap(2e-4) / rel_gap(1e-4)
    assert 1.9 < r < 2.1
    assert rel_gap(0.9) > 1e-2


def test_text_queries_dense_softmax_matches_library_attention():
    """Text rows: dense attention over [video keys; text keys], against
    torch's scaled_dot_product_attention on the concatenated keys."""
    import torch
    rng = np.random.default_rng(21)
    B, L, nt, H, d = 2, 37, 9, 3, 8
    tq, k, v = (rng.normal(size=(B, n, H, d)) for n in (nt, L, L))
    tk, tv = (rng.normal(size=(B, nt, H, d)) for _ in range(2))
    got = O.text_query_branch(tq, k, v, tk, tv)
    t = lambda x: torch.from_numpy(np.ascontiguousarray(np.swapaxes(x, 1, 2)))  # [B, H, n, d]
    want = torch.nn.functional.scaled_dot_product_attention(
        t(tq), torch.cat([t(k), t(tk)], 2), torch.cat([t(v), t(tv)], 2))
    np.testing.assert_allclose(got, np.swapaxes(want.numpy(), 1, 2), rtol=1e-10, atol=1e-12)


def test_text_queries_single_key_returns_its_value():
    rng = np.random.default_rng(22)
    tq = rng.normal(size=(1, 4, 1, 5))
    k, v = rng.normal(size=(1, 1, 1, 5)), rng.normal(size=(1, 1, 1, 5))
    empty = np.zeros((1, 0, 1, 5))
    # no text keys: the only key's value, for every text query
    kk = np.concatenate([k, empty], 1)
    out = O.text_query_branch(tq, kk, v, empty, empty)
    np.testing.assert_allclose(out, np.broadcast_to(v, out.shape), rtol=1e-14)


# --- Regions, mask ------------------------------------------------------------

def _brute_visible(tq, tk, T, C, r):
    """Pairwise statement of the pages' rule: keys in a chunk at most r chunks
    away, or the key frame is an anchor, or the query frame is an anchor."""
    anchors = (0, T - 1)
    near = abs(tq // C - tk // C) <= r
    return near or tk in anchors or tq in anchors


@pytest.mark.parametrize("T", list(range(1, 41)))
def test_regions_disjoint_and_cover(T):
    for C in range(1, 8):
        for r in (1, 2):
            M = O.frame_mask(T, C, r)
            for tq in range(T):
                S = set(O.softmax_key_frames(tq, T, C, r))
                Fw = set(O.forward_region(tq, T, C, r))
                Rv = set(O.reverse_region(tq, T, C, r))
                assert not (S & Fw) and not (S & Rv) and not (Fw & Rv)
                assert S | Fw | Rv == set(range(T))
                assert all(f < min(S - {0, T - 1}, default=T) for f in Fw)
                for tk in range(T):
                    assert M[tq, tk] == _brute_visible(tq, tk, T, C, r)


def test_token_mask_expands_frames():
    T, N, C = 7, 3, 2
    M = O.token_mask(T, N, C, 1)
    for i, j in itertools.product(range(T * N), repeat=2):
        assert M[i, j] == _brute_visible(i // N, j // N, T, C, 1)


def test_window_is_15_frames_inside_clip():
    """A query chunk away from the ends attends 3 chunks = 15 frames
    (method, local window: 15 frames wherever the clip does not cut it)."""
    T = 75
    assert len(O.window_frames(37, T, 5, 1)) == 15
    assert len(O.window_frames(2, T, 5, 1)) == 10       # shrunk at the start
    assert len(O.window_frames(73, T, 5, 1)) == 10      # and at the end
    # anchors counted once: chunk 0 already contains frame 0
    assert O.softmax_key_frames(2, T, 5, 1) == list(range(10)) + [74]


# --- Softmax branch -----------------------------------------------------------

def test_softmax_bruteforce_tiny():
    """Per-row enumeration with pure-Python loops over the visible keys."""
    rng = np.random.default_rng(11)
    B, T, N, H, d, C = 1, 7, 2, 2, 3, 2
    L = T * N
    q = rng.normal(size=(B, L, H, d)) * 2
    k = rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, d))
    got = O.softmax_branch(q, k, v, T, N, C, 1)
    sc = 1 / np.sqrt(d)
    for h in range(H):
        for i in range(L):
            vis = [j for j in range(L) if _brute_visible(i // N, j // N, T, C, 1)]
            w = [np.exp(sc * sum(q[0, i, h, c] * k[0, j, h, c] for c in range(d))) for j in vis]
            tot = sum(w)
            want = [sum(w[a] * v[0, j, h, c] for a, j in enumerate(vis)) / tot for c in range(d)]
            np.testing.assert_allclose(got[0, i, h], want, rtol=1e-12, atol=1e-13)


def test_window_spanning_clip_is_dense_softmax():
    """One chunk covering the clip: the mask is full, so the Softmax branch is
    dense attention (scipy.special.softmax)."""
    rng = np.random.default_rng(12)
    B, T, N, H, d = 2, 15, 4, 3, 8
    L = T * N
    q, k, v = (rng.normal(size=(B, L, H, d)) for _ in range(3))
    got = O.softmax_branch(q, k, v, T, N, chunk=T, radius=1)
    for b in range(B):
        for h in range(H):
            p = scipy.special.softmax(q[b, :, h] @ k[b, :, h].T / np.sqrt(d), axis=1)
            np.testing.assert_allclose(got[b, :, h], p @ v[b, :, h], rtol=1e-11, atol=1e-12)


# --- Linear branch --------------------------------------------------------------

def _tiny_linear_inputs(seed, B=1, T=17, N=3, H=2, d=4, nt=5):
    rng = np.random.default_rng(seed)
    L = T * N
    q = rng.normal(size=(B, L, H, d))
    k = _unit(rng.normal(size=(B, L, H, d)))
    v = rng.normal(size=(B, L, H, d))
    tk = _unit(rng.normal(size=(B, nt, H, d)))
    tv = rng.normal(size=(B, nt, H, d))
    beta = scipy.special.expit(rng.normal(size=(B, H, 1 + T)))
    alpha = rng.uniform(0.8, 1.0, size=(B, H, T, d))
    return q, k, v, tk, tv, beta, alpha


def test_text_counted_once():
    """With every video write off (beta_1..T = 0) and alpha = 1, each query
    reads exactly q^T S_text, whatever its frame (text counted once)."""
    q, k, v, tk, tv, beta, _ = _tiny_linear_inputs(21)
    T, N = 17, 3
    beta[:, :, 1:] = 0
    got = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1)
    for h in range(2):
        # S_text by least squares from the zero state
        n = tk.shape[1]
        Am = np.vstack([np.eye(4), np.sqrt(beta[0, h, 0]) * tk[0, :, h]])
        rhs = np.vstack([np.zeros((4, 4)), np.sqrt(beta[0, h, 0]) * tv[0, :, h]])
        S_text = np.linalg.lstsq(Am, rhs, rcond=None)[0]
        assert n == 5
        np.testing.assert_allclose(got[0, :, h], q[0, :, h] @ S_text, rtol=1e-11, atol=1e-12)


def test_pure_decay_closed_form():
    """No video writes, channel-wise decay: the forward readout carries
    prod_{j<=t} alpha_j and the reverse one prod_{j>=t} alpha_j (every frame
    between the text state and the query decays: frames outside the window,
    anchors, and the bridge across the window).  Anchor queries: q^T S_text."""
    q, k, v, tk, tv, beta, alpha = _tiny_linear_inputs(22)
    T, N, d = 17, 3, 4
    beta[:, :, 1:] = 0
    got = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1, alpha=alpha)
    for h in range(2):
        St = O.text_state(tk[0, :, h], tv[0, :, h], beta[0, h, 0])
        for i in range(T * N):
            t = i // N
            if t in (0, T - 1):
                want = q[0, i, h] @ St
            else:
                gf = np.prod(alpha[0, h, :t + 1], axis=0)
                gr = np.prod(alpha[0, h, t:], axis=0)
                want = q[0, i, h] @ (0.5 * gf[:, None] * St) + q[0, i, h] @ (0.5 * gr[:, None] * St)
            np.testing.assert_allclose(got[0, i, h], want, rtol=1e-11, atol=1e-12)


def test_time_reversal_equivariance():
    """Reversing the frame order (T a multiple of the chunk, so the chunk grid
    and the window are symmetric) swaps the forward and reverse scans: the
    linear readout of the reversed clip is the reversed readout."""
    T, N, H, d = 20, 3, 2, 4
    q, k, v, tk, tv, beta, alpha = _tiny_linear_inputs(23, T=T, N=N, H=H, d=d)

    def rev_tok(x):
        B, L = x.shape[:2]
        return x.reshape(B, T, N, *x.shape[2:])[:, ::-1].reshape(x.shape)

    beta_r = np.concatenate([beta[:, :, :1], beta[:, :, 1:][:, :, ::-1]], axis=2)
    alpha_r = alpha[:, :, ::-1]
    a = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1, alpha=alpha)
    b = O.linear_branch(rev_tok(q), rev_tok(k), rev_tok(v), beta_r, tk, tv, T, N, 5, 1,
                        alpha=alpha_r)
    np.testing.assert_allclose(rev_tok(b), a, rtol=1e-10, atol=1e-11)


def test_linear_regions_match_explicit_frame_sets():
    """The readout equals q^T (forward state over exactly forward_region) +
    q^T (reverse state over exactly reverse_region), built here by running the
    delta-rule update over those explicit frame lists (alpha = 1)."""
    T, N, H, d = 17, 3, 2, 4
    q, k, v, tk, tv, beta, _ = _tiny_linear_inputs(24, T=T, N=N, H=H, d=d)
    got = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1)
    for h in range(H):
        St = O.text_state(tk[0, :, h], tv[0, :, h], beta[0, h, 0])
        for tq in range(T):
            Sf = 0.5 * St
            for t in O.forward_region(tq, T, 5, 1):
                Sf = O.vda_update(Sf, k[0, t * N:(t + 1) * N, h], v[0, t * N:(t + 1) * N, h],
                                  beta[0, h, 1 + t])
            Sr = 0.5 * St
            for t in reversed(O.reverse_region(tq, T, 5, 1)):
                Sr = O.vda_update(Sr, k[0, t * N:(t + 1) * N, h], v[0, t * N:(t + 1) * N, h],
                                  beta[0, h, 1 + t])
            for n in range(N):
                i = tq * N + n
                np.testing.assert_allclose(got[0, i, h], q[0, i, h] @ Sf + q[0, i, h] @ Sr,
                                           rtol=1e-11, atol=1e-12)


def test_boundary_states_consistent_with_readout():
    T, N, H, d = 17, 3, 2, 4
    q, k, v, tk, tv, beta, _ = _tiny_linear_inputs(25, T=T, N=N, H=H, d=d)
    F, G = O.boundary_states(k, v, beta, tk, tv, T, N, 5, 1)
    got = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1)
    for h in range(H):
        for i in range(N, (T - 1) * N):
            c = (i // N) // 5
            np.testing.assert_allclose(got[0, i, h], q[0, i, h] @ (F[0, h, c] + G[0, h, c]),
                                       rtol=1e-11, atol=1e-12)


# --- Output -----------------------------------------------------------------------

def test_rms_norm_properties():
    rng = np.random.default_rng(31)
    o = rng.normal(size=(2, 5, 3, 16)) * 3
    y = O.rms_norm(o, eps=0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(O.rms_norm(7.5 * o, eps=0.0), y, rtol=1e-13)
    ye = O.rms_norm(o, eps=1e-6)
    ms = np.mean(o * o, axis=-1)
    np.testing.assert_allclose(np.mean(ye * ye, axis=-1), ms / (ms + 1e-6), rtol=1e-12)


def test_projection_head_blocks():
    """Head h's gated branch outputs only reach the output through rows
    h*d_v .. (h+1)*d_v of its own projection; zeroing a gate removes that
    branch."""
    rng = np.random.default_rng(32)
    B, R, H, dv, Do = 1, 4, 3, 5, 7
    os_, ol = rng.normal(size=(B, R, H, dv)), rng.normal(size=(B, R, H, dv))
    gs, gl = rng.uniform(size=(B, R, H, dv)), rng.uniform(size=(B, R, H, dv))
    Ws, Wl = rng.normal(size=(H * dv, Do)), rng.normal(size=(H * dv, Do))
    full = O.output_projection(os_, ol, gs, gl, Ws, Wl)
    no_lin = O.output_projection(os_, ol, gs, 0 * gl, Ws, Wl)
    no_soft = O.output_projection(os_, ol, 0 * gs, gl, Ws, Wl)
    np.testing.assert_allclose(full, no_lin + no_soft, rtol=1e-12, atol=1e-12)
    Ws2 = Ws.copy()
    Ws2[dv:2 * dv] = 0
    os2 = os_.copy()
    os2[:, :, 1] = 123.0
    np.testing.assert_allclose(O.output_projection(os2, ol, gs, 0 * gl, Ws2, Wl),
                               O.output_projection(os_, ol, gs, 0 * gl, Ws2, Wl), atol=1e-12)
    # a single head, single channel: out = g * o * W[row]
    one = O.output_projection(np.ones((1, 1, 1, 1)) * 2, np.zeros((1, 1, 1, 1)),
                              np.full((1, 1, 1, 1), 0.5), np.zeros((1, 1, 1, 1)),
                              np.array([[3.0, -1.0]]), np.zeros((1, 2)))
    np.testing.assert_allclose(one, [[[3.0, -1.0]]])


def test_softmax_with_text_keys_bruteforce():
    """Video queries with the text tokens visible: per-row enumeration over
    the visible video keys plus every text key, one normaliser."""
    rng = np.random.default_rng(13)
    B, T, N, H, d, C, nt = 1, 6, 2, 2, 3, 2, 3
    L = T * N
    q = rng.normal(size=(B, L, H, d))
    k = rng.normal(size=(B, L, H, d))
    v = rng.normal(size=(B, L, H, d))
    tk = rng.normal(size=(B, nt, H, d))
    tv = rng.normal(size=(B, nt, H, d))
    got = O.softmax_branch(q, k, v, T, N, C, 1, text_k=tk, text_v=tv)
    sc = 1 / np.sqrt(d)
    for h in range(H):
        for i in range(L):
            keys = [(k[0, j, h], v[0, j, h]) for j in range(L)
                    if _brute_visible(i // N, j // N, T, C, 1)]
            keys += [(tk[0, t, h], tv[0, t, h]) for t in range(nt)]
            w = [np.exp(sc * float(np.dot(q[0, i, h], kk))) for kk, _ in keys]
            want = sum(wi * vv for wi, (_, vv) in zip(w, keys)) / sum(w)
            np.testing.assert_allclose(got[0, i, h], want, rtol=1e-12, atol=1e-13)
    # without text keys the result is the plain window+anchor Softmax
    np.testing.assert_allclose(O.softmax_branch(q, k, v, T, N, C, 1, text_k=tk[:, :0],
                                                text_v=tv[:, :0]),
                               O.softmax_branch(q, k, v, T, N, C, 1), rtol=0, atol=0)


@pytest.mark.parametrize("seed", range(3))
def test_per_token_beta_least_squares(seed):
    """Per-token write gates: the update minimises
    1/2||S - S~||^2 + 1/2 sum_i beta_i ||S^T k_i - v_i||^2 (stacked rows sqrt(beta_i))."""
    rng = np.random.default_rng(400 + seed)
    dk, dv, n = 6, 5, 9
    S_prev = rng.normal(size=(dk, dv))
    K = _unit(rng.normal(size=(n, dk)))
    V = rng.normal(size=(n, dv))
    beta = rng.uniform(0.0, 2.0, size=n)
    alpha = rng.uniform(0.5, 1.0, size=dk)
    Amat = np.vstack([np.eye(dk), np.sqrt(beta)[:, None] * K])
    rhs = np.vstack([alpha[:, None] * S_prev, np.sqrt(beta)[:, None] * V])
    want = np.linalg.lstsq(Amat, rhs, rcond=None)[0]
    np.testing.assert_allclose(O.vda_update(S_prev, K, V, beta, alpha), want,
                               rtol=1e-10, atol=1e-10)


def test_per_token_beta_constant_equals_per_frame():
    q, k, v, tk, tv, beta, alpha = _tiny_linear_inputs(26)
    T, N, nt = 17, 3, 5
    per_tok = np.concatenate([np.repeat(beta[:, :, :1], nt, axis=2),
                              np.repeat(beta[:, :, 1:], N, axis=2)], axis=2)
    a = O.linear_branch(q, k, v, beta, tk, tv, T, N, 5, 1, alpha=alpha)
    b = O.linear_branch(q, k, v, per_tok, tk, tv, T, N, 5, 1, alpha=alpha, beta_per_token=True)
    np.testing.assert_allclose(b, a, rtol=1e-11, atol=1e-12)


# --- Gate routing of the whole forward ---------------------------------------

def _routing_case():
    from synth import CONFIGS, make_inputs
    cfg = CONFIGS["tiny_f32"].replace(T=7, N=6, H=2, d=32, n_text=5, seed=41)
    inp = make_inputs(cfg, gates="random")
    a = {k: (None if v is None else O._to_np(v)) for k, v in inp.items()}
    return cfg, inp, a


def _loop_projection(x, W):
    """out[b, r, :] = sum_h sum_c x[b, r, h, c] * W[h * d + c, :], written as
    explicit loops over heads and channels (no reshape)."""
    B, R, H, d = x.shape
    out = np.zeros((B, R, W.shape[1]))
    for b in range(B):
        for r in range(R):
            for h in range(H):
                for c in range(d):
                    out[b, r] += x[b, r, h, c] * W[h * d + c]
    return out


def _check_routing(fwd):
    """Raises AssertionError unless ``fwd`` (the oracle's hybrid_forward, or a
    variant of it) routes each gate to its own branch and projection."""
    cfg, inp, a = _routing_case()
    T, N = cfg.T, cfg.N
    o_s = O.softmax_branch(a["q"], a["k"], a["v"], T, N, cfg.chunk, cfg.window_radius)
    o_l = O.linear_branch(a["q"], a["k"], a["v"], a["beta"], a["text_k"], a["text_v"], T, N,
                          cfg.chunk, cfg.window_radius)
    g_s, g_l = a["gates"][0], a["gates"][1]
    assert np.std(g_s) > 0.05 and np.max(np.abs(g_s - g_l)) > 0.3  # two different gates
    soft_half = _loop_projection(g_s * o_s, a["W_soft"])
    ms = np.mean(o_l * o_l, axis=-1, keepdims=True)
    lin_half = _loop_projection(g_l * o_l / np.sqrt(ms + 1e-6), a["W_lin"])

    only_soft = dict(inp)
    only_soft["gates"] = inp["gates"].clone()
    only_soft["gates"][1] = 0
    out, _, _ = fwd(only_soft, T, N, cfg.chunk, cfg.window_radius)
    np.testing.assert_allclose(out, soft_half, rtol=1e-10, atol=1e-12)

    only_lin = dict(inp)
    only_lin["gates"] = inp["gates"].clone()
    only_lin["gates"][0] = 0
    out, _, _ = fwd(only_lin, T, N, cfg.chunk, cfg.window_radius)
    np.testing.assert_allclose(out, lin_half, rtol=1e-10, atol=1e-12)

    out, _, _ = fwd(inp, T, N, cfg.chunk, cfg.window_radius)
    np.testing.assert_allclose(out, soft_half + lin_half, rtol=1e-10, atol=1e-12)
    # the gates are not interchangeable: swapping them moves the output
    swapped = dict(inp)
    swapped["gates"] = inp["gates"].flip(0)
    out_sw, _, _ = fwd(swapped, T, N, cfg.chunk, cfg.window_radius)
    assert np.max(np.abs(out_sw - out)) > 1e-2 * np.sqrt(np.mean(out ** 2))


def test_forward_routes_each_gate_to_its_own_branch_and_projection():
    """The pages' output stage: the Softmax readout is gated by its own sigmoid
    gate and projected by its own matrix; the linear readout is RMS-normalised,
    gated by the second gate and projected by the second matrix; the two are
    added.  With g_l = 0 the forward is the Softmax half alone, with g_s = 0 the
    linear half alone (each rebuilt here with per-head, per-channel loops), and
    with both gates random the forward is their sum."""
    _check_routing(O.hybrid_forward)


@pytest.mark.parametrize("mistake", ["swap_gates", "swap_projections", "transpose_gate"])
def test_routing_pin_catches_planted_mistakes(monkeypatch, mistake):
    """The routing pin fails on an oracle with a planted mistake in its output
    stage (patched here, on the CPU): gates swapped between the branches,
    projections swapped, or the gate's head and channel axes transposed."""
    real = O.output_projection

    def planted(o_s, o_l, g_s, g_l, W_soft, W_lin, eps=1e-6):
        if mistake == "swap_gates":
            return real(o_s, o_l, g_l, g_s, W_soft, W_lin, eps)
        if mistake == "swap_projections":
            return real(o_s, o_l, g_s, g_l, W_lin, W_soft, eps)
        gs = np.asarray(g_s, np.float64)
        B, R, H, d = gs.shape
        gs = gs.reshape(B, R, H * d).reshape(B, R, d, H).swapaxes(-1, -2)
        return real(o_s, o_l, gs, g_l, W_soft, W_lin, eps)

    monkeypatch.setattr(O, "output_projection", planted)
    with pytest.raises(AssertionError):
        _check_routing(O.hybrid_forward)


def test_gate_rows_follow_the_sampled_query_rows():
    """Forward on a subset of query rows equals the same rows of the full
    forward, with random per-element gates (the gate rows follow the rows)."""
    cfg, inp, _ = _routing_case()
    full, _, _ = O.hybrid_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius)
    rows = np.array([0, 5, 6, 17, 23, cfg.T * cfg.N - 1])
    part, _, _ = O.hybrid_forward(inp, cfg.T, cfg.N, cfg.chunk, cfg.window_radius, rows=rows)
    np.testing.assert_allclose(part, full[:, rows], rtol=1e-12, atol=1e-13)


def test_random_gates_leave_every_other_draw_unchanged():
    from synth import CONFIGS, make_inputs
    cfg = CONFIGS["tiny_f32"]
    a, b = make_inputs(cfg), make_inputs(cfg, gates="random", alpha_range=(0.9, 1.0))
    for k in ("q", "k", "v", "text_k", "text_v", "beta", "W_soft", "W_lin"):
        assert np.array_equal(O._to_np(a[k]), O._to_np(b[k])), k
    g = O._to_np(b["gates"])
    assert g.shape == (2, cfg.B, cfg.L, cfg.H, cfg.d)
    assert 0 < g.min() and g.max() < 1 and abs(g.mean() - 0.5) < 0.05
