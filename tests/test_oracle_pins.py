"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here runs the CUDA library.  Each test checks the oracle against an
independent fact: the objective whose minimiser the closed form is, a
textbook least-squares routine, the per-token delta rule it reduces to with
one token per frame, a dense masked Softmax built by brute force, the
frame-pair counts of the mask derived by hand, and invariances.
"""

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle
from video_diffusion_hybrid_vda_b200 import synth


def _tiny(T=10, N=16, H=1, d=16, seed=0, with_fuse=False):
    s = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(s, dtype=torch.float32, seed=seed, with_fuse=with_fuse)
    return s, {kk: vv.numpy().astype(np.float64) for kk, vv in inp.items()}


# ---------------------------------------------------------------- objective

def _objective(S, S_bar, K, V, beta):
    """J(S) = ||S - S_bar||^2 + sum_i beta_i ||S k_i - v_i||^2 (token by token)."""
    J = np.sum((S - S_bar) ** 2)
    for i in range(K.shape[0]):
        r = S @ K[i] - V[i]
        J += beta[i] * (r @ r)
    return J


def _gradient(S, S_bar, K, V, beta):
    G = 2.0 * (S - S_bar)
    for i in range(K.shape[0]):
        G += 2.0 * beta[i] * np.outer(S @ K[i] - V[i], K[i])
    return G


@pytest.mark.parametrize("direction", ["fwd", "bwd"])
def test_scan_states_minimise_frame_objective(direction):
    """Every scan state zeroes the gradient of its frame's objective.

    The objective is evaluated from the raw tokens of the frame, so this
    pins prep (A, B), the closed-form solve and the decay/ordering of both
    scans at once.
    """
    s, x = _tiny(T=7, N=5, H=2, d=6, seed=3)
    o, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                 s.T, s.N, s.H, s.d)
    for h in range(s.H):
        for t in range(s.T):
            rows = slice(t * s.N, (t + 1) * s.N)
            cols = slice(h * s.d, (h + 1) * s.d)
            K, V, beta = x["k"][rows, cols], x["v"][rows, cols], x["beta"][rows, h]
            if direction == "fwd":
                S = S_fwd[t, h]
                prev = S_fwd[t - 1, h] if t > 0 else np.zeros((s.d, s.d))
            else:
                S = S_bwd[t, h]
                prev = S_bwd[t + 1, h] if t + 1 < s.T else np.zeros((s.d, s.d))
            S_bar = x["alpha"][t, h] * prev
            G = _gradient(S, S_bar, K, V, beta)
            assert np.abs(G).max() <= 1e-10 * (1.0 + np.abs(S).max())


def test_closed_form_is_strict_minimum():
    rng = np.random.default_rng(1)
    d, n = 8, 11
    K = rng.standard_normal((n, d))
    V = rng.standard_normal((n, d))
    beta = rng.uniform(0.05, 1.0, n)
    S_bar = rng.standard_normal((d, d))
    A = sum(beta[i] * np.outer(K[i], K[i]) for i in range(n))
    B = sum(beta[i] * np.outer(V[i], K[i]) for i in range(n))
    S = oracle.vda_frame_state(S_bar, A, B)
    J0 = _objective(S, S_bar, K, V, beta)
    for _ in range(20):
        E = rng.standard_normal((d, d))
        for eps in (1e-3, 1e-1, 1.0):
            assert _objective(S + eps * E, S_bar, K, V, beta) > J0


def test_closed_form_equals_weighted_ridge_lstsq():
    """S^T = argmin || [sqrt(b) K; I] X - [sqrt(b) V; S_bar^T] ||, by SVD lstsq."""
    rng = np.random.default_rng(2)
    for (n, d) in [(1, 4), (5, 8), (40, 16)]:
        K = rng.standard_normal((n, d))
        V = rng.standard_normal((n, d))
        beta = rng.uniform(0.0, 1.0, n)
        S_bar = rng.standard_normal((d, d))
        A = (K * beta[:, None]).T @ K
        B = V.T @ (K * beta[:, None])
        S = oracle.vda_frame_state(S_bar, A, B)
        sb = np.sqrt(beta)[:, None]
        lhs = np.vstack([sb * K, np.eye(d)])
        rhs = np.vstack([sb * V, S_bar.T])
        X, *_ = scipy.linalg.lstsq(lhs, rhs, lapack_driver="gelsd")
        assert np.abs(S - X.T).max() <= 1e-12 * (1 + np.abs(X).max())


def test_single_frame_is_ridge_regression():
    """T = 1: S = B (I + A)^-1 for both directions; the two states coincide."""
    s, x = _tiny(T=1, N=9, H=2, d=6, seed=5)
    o, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                 s.T, s.N, s.H, s.d)
    for h in range(s.H):
        c = slice(h * s.d, (h + 1) * s.d)
        sb = np.sqrt(x["beta"][:, h])[:, None]
        lhs = np.vstack([sb * x["k"][:, c], np.eye(s.d)])
        rhs = np.vstack([sb * x["v"][:, c], np.zeros((s.d, s.d))])
        X, *_ = scipy.linalg.lstsq(lhs, rhs)
        np.testing.assert_allclose(S_fwd[0, h], X.T, atol=1e-12)
        np.testing.assert_allclose(S_bwd[0, h], X.T, atol=1e-12)


# ------------------------------------------------------- non-expansiveness

@pytest.mark.parametrize("T,N,H,d", [(10, 16, 1, 16), (17, 16, 1, 16), (6, 40, 3, 8)])
def test_transition_is_non_expansive(T, N, H, d):
    """||M_t||_2 <= 1 with M_t = alpha_t (I + A_t)^-1 (10100.com, 方法概述 item 2)."""
    s = synth.Shape(T, N, H, d)
    x = {kk: vv.numpy().astype(np.float64)
         for kk, vv in synth.make_inputs(s, torch.float32, seed=7).items()}
    A, _ = oracle.vda_prep(x["k"], x["v"], x["beta"], T, N, H, d)
    for t in range(T):
        for h in range(H):
            M = oracle.transition_matrix(x["alpha"][t, h], A[t, h])
            sv = np.linalg.svd(M, compute_uv=False)
            assert sv.max() <= 1.0 + 1e-12
            # with beta > 0 and k != 0 the bound is strict along the keys
            assert sv.min() < x["alpha"][t, h]


@pytest.mark.parametrize("T,N,H,d", [(10, 16, 1, 16), (6, 40, 3, 8)])
def test_transition_is_what_the_scan_applies(T, N, H, d):
    """M_t is the map the scans apply to the inherited state (方法概述 item 2:
    the decayed old state is carried through (I + A_t)^-1).

    Two pins that tie transition_matrix to the recurrence, not only to its
    norm bound: (1) every forward and backward state obeys
    S_t = S_prev M_t + S_t^(0), where S_t^(0) is the frame's state from a zero
    inherited state; (2) two scans of one frame from different inherited
    states differ by exactly their difference times M_t.  Dropping alpha_t,
    inverting I + A_t the wrong way, or transposing M_t fails one of them
    (alpha_t < 1 and A_t is not a multiple of I in these inputs).
    """
    s = synth.Shape(T, N, H, d)
    x = {kk: vv.numpy().astype(np.float64)
         for kk, vv in synth.make_inputs(s, torch.float32, seed=11).items()}
    A, B = oracle.vda_prep(x["k"], x["v"], x["beta"], T, N, H, d)
    S_fwd, S_bwd = oracle.vda_scan(A, B, x["alpha"])
    zero = np.zeros((d, d))
    rng = np.random.default_rng(5)
    for h in range(H):
        for t in range(T):
            M = oracle.transition_matrix(x["alpha"][t, h], A[t, h])
            S0 = oracle.vda_frame_state(zero, A[t, h], B[t, h])
            prev_f = S_fwd[t - 1, h] if t > 0 else zero
            prev_b = S_bwd[t + 1, h] if t + 1 < T else zero
            np.testing.assert_allclose(S_fwd[t, h], prev_f @ M + S0, atol=1e-12)
            np.testing.assert_allclose(S_bwd[t, h], prev_b @ M + S0, atol=1e-12)
            # a non-symmetric perturbation of the inherited state, so that
            # M and M^T act differently on it
            X, Y = rng.standard_normal((d, d)), rng.standard_normal((d, d))
            a = x["alpha"][t, h]
            dS = (oracle.vda_frame_state(a * X, A[t, h], B[t, h])
                  - oracle.vda_frame_state(a * Y, A[t, h], B[t, h]))
            np.testing.assert_allclose(dS, (X - Y) @ M, atol=1e-12)


# ------------------------------------------------------ one token per frame

def _per_token_delta_rule(q, k, v, beta, alpha, T, H, d):
    """Classic gated delta rule, one token per step, both directions, summed.

    S <- alpha S;  S <- S + b' (v - S k) k^T  with  b' = beta / (1 + beta ||k||^2),
    read o_t = S_t q_t in each direction and add the two reads.
    """
    o = np.zeros((T, H * d))
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        for order in (range(T), range(T - 1, -1, -1)):
            S = [[0.0] * d for _ in range(d)]
            for t in order:
                kt, vt, qt = k[t, c], v[t, c], q[t, c]
                b = beta[t, h] / (1.0 + beta[t, h] * sum(kt[j] * kt[j] for j in range(d)))
                for a in range(d):
                    for j in range(d):
                        S[a][j] *= alpha[t, h]
                Sk = [sum(S[a][j] * kt[j] for j in range(d)) for a in range(d)]
                for a in range(d):
                    for j in range(d):
                        S[a][j] += b * (vt[a] - Sk[a]) * kt[j]
                for a in range(d):
                    o[t, h * d + a] += sum(S[a][j] * qt[j] for j in range(d))
    return o


def test_one_token_per_frame_is_per_token_delta_rule():
    s, x = _tiny(T=9, N=1, H=2, d=5, seed=11)
    # unnormalised keys make ||k|| != 1 so the Sherman-Morrison factor matters
    x["k"] = x["k"] * 1.7
    o, _, _ = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)
    ref = _per_token_delta_rule(x["q"], x["k"], x["v"], x["beta"], x["alpha"], s.T, s.H, s.d)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------- VDA invariances

def test_vda_linear_in_q():
    s, x = _tiny(T=6, N=4, H=2, d=4, seed=13)
    q2 = np.random.default_rng(0).standard_normal(x["q"].shape)
    f = lambda q: oracle.vda(q, x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)[0]
    np.testing.assert_allclose(f(x["q"] + 2.0 * q2), f(x["q"]) + 2.0 * f(q2), atol=1e-12)


def test_vda_unit_query_reads_state_column():
    """q = e_j at one token reads column j of S_fwd_t + S_bwd_t."""
    s, x = _tiny(T=5, N=3, H=2, d=4, seed=17)
    q = np.zeros_like(x["q"])
    r, h, j = 7, 1, 2                      # token 7 is in frame 2
    q[r, h * s.d + j] = 1.0
    o, S_fwd, S_bwd = oracle.vda(q, x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)
    t = r // s.N
    np.testing.assert_allclose(o[r, h * s.d:(h + 1) * s.d], (S_fwd[t, h] + S_bwd[t, h])[:, j],
                               atol=1e-14)
    assert np.abs(np.delete(o, r, axis=0)).max() == 0.0


def test_vda_frame_reversal_swaps_directions():
    """Reversing the frame order (tokens, beta, alpha) swaps the two scans."""
    s, x = _tiny(T=8, N=3, H=2, d=4, seed=19)
    rev_rows = np.concatenate([np.arange(t * s.N, (t + 1) * s.N) for t in range(s.T - 1, -1, -1)])
    o, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)
    o_r, R_fwd, R_bwd = oracle.vda(x["q"][rev_rows], x["k"][rev_rows], x["v"][rev_rows],
                                   x["beta"][rev_rows], x["alpha"][::-1], s.T, s.N, s.H, s.d)
    np.testing.assert_allclose(R_fwd, S_bwd[::-1], atol=1e-13)
    np.testing.assert_allclose(R_bwd, S_fwd[::-1], atol=1e-13)
    np.testing.assert_allclose(o_r, o[rev_rows], atol=1e-13)


def test_vda_readout_variant_differs_only_by_own_write():
    s, x = _tiny(T=5, N=2, H=1, d=3, seed=23)
    args = (x["q"], x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)
    o_sum, S_fwd, S_bwd = oracle.vda(*args)
    o_var, _, _ = oracle.vda(*args, combine="fwd_incl_bwd_excl")
    t = s.T - 1          # the last frame has no later backward state
    r = slice(t * s.N, (t + 1) * s.N)
    np.testing.assert_allclose(o_sum[r] - o_var[r], x["q"][r] @ S_bwd[t, 0].T, atol=1e-13)


# --------------------------------------------------------- window Softmax

def _dense_masked_attention(q, k, v, T, N, H, d):
    """Brute force: dense [L, L] scores, -inf outside the frame mask."""
    L = T * N
    allowed = np.zeros((L, L), dtype=bool)
    for tq in range(T):
        for tk in range(T):
            near = abs(tq // 5 - tk // 5) <= 1
            anchor = tq in (0, T - 1) or tk in (0, T - 1)
            if near or anchor:
                allowed[tq * N:(tq + 1) * N, tk * N:(tk + 1) * N] = True
    out = np.zeros((L, H * d))
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        s = q[:, c] @ k[:, c].T / np.sqrt(d)
        s = np.where(allowed, s, -np.inf)
        out[:, c] = scipy.special.softmax(s, axis=1) @ v[:, c]
    return out, allowed


@pytest.mark.parametrize("T", [10, 17, 23])
def test_window_attn_equals_dense_masked(T):
    s, x = _tiny(T=T, N=16, H=1, d=16, seed=0)
    o, lse = oracle.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    ref, allowed = _dense_masked_attention(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    np.testing.assert_allclose(o, ref, rtol=1e-12, atol=1e-12)
    if T == 10:
        assert allowed.all()          # 2 chunks: everything is within one chunk
    else:
        assert not allowed.all()
    sc = x["q"] @ x["k"].T / 4.0
    lse_ref = scipy.special.logsumexp(np.where(allowed, sc, -np.inf), axis=1)
    np.testing.assert_allclose(lse[0], lse_ref, rtol=1e-12)


@pytest.mark.parametrize("T,M", [(10, 5), (17, 9)])
def test_window_attn_with_context_keys_equals_dense_masked(T, M):
    """Context (text/audio) keys join the same softmax, visible to every query:
    brute force over [video keys; context keys] with an all-visible block."""
    s, x = _tiny(T=T, N=8, H=2, d=8, seed=41)
    rng = np.random.default_rng(T + M)
    ck = rng.standard_normal((M, s.D))
    cv = rng.standard_normal((M, s.D))
    o, lse = oracle.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d, ctx_k=ck, ctx_v=cv)
    _, allowed = _dense_masked_attention(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    full = np.hstack([allowed, np.ones((s.L, M), dtype=bool)])
    for h in range(s.H):
        c = slice(h * s.d, (h + 1) * s.d)
        K = np.vstack([x["k"][:, c], ck[:, c]])
        V = np.vstack([x["v"][:, c], cv[:, c]])
        sc = np.where(full, x["q"][:, c] @ K.T / np.sqrt(s.d), -np.inf)
        np.testing.assert_allclose(o[:, c], scipy.special.softmax(sc, axis=1) @ V, atol=1e-12)
        np.testing.assert_allclose(lse[h], scipy.special.logsumexp(sc, axis=1), rtol=1e-12)
    # no context keys: identical to the plain window attention
    o0, _ = oracle.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d,
                               ctx_k=ck[:0], ctx_v=cv[:0])
    o1, _ = oracle.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    np.testing.assert_array_equal(o0, o1)


def _closed_form_pair_count(T, cf=5):
    """Visible (query, key) frame pairs for chunk 5, +-1 chunk, both anchors.

    Anchor query frames see all T frames.  Another query frame in chunk c
    sees the frames of chunks c-1..c+1 (clipped to [0, T)) plus each anchor
    frame that lies outside that window.
    """
    total = len({0, T - 1}) * T
    nchunks = -(-T // cf)
    for c in range(nchunks):
        lo, hi = max(0, (c - 1) * cf), min(T, (c + 2) * cf)
        window = hi - lo
        extra = (0 if lo == 0 else 1) + (0 if hi == T else 1)
        members = [t for t in range(c * cf, min(T, (c + 1) * cf)) if t not in (0, T - 1)]
        total += len(members) * (window + extra)
    return total


def test_mask_pair_counts():
    assert oracle.mask_pair_count(102) == 1846 == _closed_form_pair_count(102)
    assert oracle.mask_pair_count(42) == 706 == _closed_form_pair_count(42)
    for T in range(1, 60):
        assert oracle.mask_pair_count(T) == _closed_form_pair_count(T)


def test_mask_density_near_pages_figures():
    """The article prints 42.08 % at 42 frames and 19.98 % at 102 (效率阶梯).

    Those figures likely count text/audio tokens too (not in this layer),
    so they pin the frame mask only to about 2.5 percentage points; the
    mask without anchors (32.5 % / 14.2 %) is ruled out by them.
    """
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "mask_density.txt")
    pages = {}
    with open(path, encoding="utf-8") as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                T, pct = line.split()[:2]
                pages[int(T)] = float(pct)
    for T, pct in pages.items():
        ours = 100.0 * oracle.mask_pair_count(T) / (T * T)
        assert abs(ours - pct) < 2.5, (T, ours, pct)
        no_anchor = 100.0 * oracle.mask_pair_count(T, anchors=0) / (T * T)
        assert abs(no_anchor - pct) > 5.0


# ------------------------------------------------------------------- fuse

def test_fuse_zero_gate_weights_give_half():
    s, x = _tiny(T=3, N=4, H=2, d=8, seed=29, with_fuse=True)
    L, D = s.L, s.D
    rng = np.random.default_rng(3)
    o_s, o_l = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    Z = np.zeros((D, D))
    y = oracle.hybrid_fuse(x["x"], o_s, o_l, Z, Z, x["gamma"], 1e-6, x["W_os"], x["W_ol"], s.H)
    n = oracle.rmsnorm_heads(o_l, s.H, s.d, x["gamma"], 1e-6)
    np.testing.assert_allclose(y, 0.5 * o_s @ x["W_os"].T + 0.5 * n @ x["W_ol"].T, atol=1e-12)


def test_rmsnorm_is_per_head():
    rng = np.random.default_rng(4)
    H, d, L = 3, 8, 5
    o = rng.standard_normal((L, H * d)) * np.repeat([0.1, 1.0, 30.0], d)
    n = oracle.rmsnorm_heads(o, H, d, np.ones(H * d), 0.0)
    rms = np.sqrt(np.mean(n.reshape(L, H, d) ** 2, axis=2))
    np.testing.assert_allclose(rms, 1.0, atol=1e-12)
    # a unit-RMS head block with gamma = 1 and eps = 0 is left unchanged
    np.testing.assert_allclose(oracle.rmsnorm_heads(n, H, d, np.ones(H * d), 0.0), n, atol=1e-12)
    g = np.arange(1, H * d + 1, dtype=np.float64)
    np.testing.assert_allclose(oracle.rmsnorm_heads(o, H, d, g, 0.0), n * g, atol=1e-12)


def test_fuse_gate_acts_before_projection():
    """Saturated gates select input channels of the projection, not outputs."""
    H, d = 2, 4
    D, L = H * d, 6
    rng = np.random.default_rng(5)
    x = np.ones((L, D))
    on = np.array([1, 0, 1, 1, 0, 0, 1, 0], dtype=bool)
    W_gs = np.zeros((D, D))
    W_gs[on, :] = 40.0
    W_gs[~on, :] = -40.0
    W_gl = -W_gs                                 # the complementary channels
    o_s, o_l = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    W_os, W_ol = rng.standard_normal((D, D)), rng.standard_normal((D, D))
    gamma = np.ones(D)
    y = oracle.hybrid_fuse(x, o_s, o_l, W_gs, W_gl, gamma, 1e-6, W_os, W_ol, H)
    n = oracle.rmsnorm_heads(o_l, H, d, gamma, 1e-6)
    ref = o_s[:, on] @ W_os[:, on].T + n[:, ~on] @ W_ol[:, ~on].T
    np.testing.assert_allclose(y, ref, atol=1e-9)


def test_fuse_fixed_softmax_gate():
    """With the Softmax gate pinned at 0.99 (the A1 stage of the recipe) and
    the linear gate closed, y = 0.99 o_s W_os^T."""
    H, d = 2, 4
    D, L = H * d, 5
    rng = np.random.default_rng(6)
    x = np.ones((L, D)) / D
    W_gs = np.full((D, D), np.log(0.99 / 0.01))   # x W^T = logit(0.99)
    W_gl = np.full((D, D), -1e4)
    o_s, o_l = rng.standard_normal((L, D)), rng.standard_normal((L, D))
    W_os, W_ol = rng.standard_normal((D, D)), rng.standard_normal((D, D))
    y = oracle.hybrid_fuse(x, o_s, o_l, W_gs, W_gl, np.ones(D), 1e-6, W_os, W_ol, H)
    np.testing.assert_allclose(y, 0.99 * o_s @ W_os.T, atol=1e-12)


def test_fuse_rows_match_full():
    s, x = _tiny(T=3, N=4, H=2, d=8, seed=31, with_fuse=True)
    rng = np.random.default_rng(7)
    o_s, o_l = rng.standard_normal((s.L, s.D)), rng.standard_normal((s.L, s.D))
    args = (x["x"], o_s, o_l, x["W_gs"], x["W_gl"], x["gamma"], 1e-6, x["W_os"], x["W_ol"], s.H)
    y = oracle.hybrid_fuse(*args)
    rows = [0, 5, 11]
    np.testing.assert_allclose(oracle.hybrid_fuse_rows(*args, rows), y[rows], atol=1e-14)
