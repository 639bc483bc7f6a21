"""Video Delta Attention (VDA), float64 CPU oracle.  TEST INFRASTRUCTURE ONLY.

Source: "Video DeltaNet" article on 10100.com, 方法概述 item 2 (frame-level
delta rule).  The state of latent frame t is the minimiser of a joint objective:
stay close to the decayed previous state S_bar_t, and fit every key-value
association of frame t at once.  With unit weights on both terms,

    J(S) = ||S - S_bar_t||_F^2 + sum_i beta_i ||S k_i - v_i||^2,

setting dJ/dS = 0 gives the closed form printed on the page,

    S_t = (S_bar_t + B_t) (I + A_t)^-1,
    A_t = sum_i beta_i k_i k_i^T,   B_t = sum_i beta_i v_i k_i^T,

with S_bar_t = alpha_t S_{t-1}.  The figure caption under 效率阶梯 says the
linear branch runs a forward and a backward scan over the frames.

Layout (frame-major, matching the CUDA library): a token row r = t*N + i;
q, k, v are [L, D] with head h in columns [h*d, (h+1)*d); beta is [L, H];
alpha is [T, H]; states are [T, H, d, d] with S[..., v_dim, k_dim].

Readings of the pages taken here:
* both scans include frame t's own write; the read-out sums the two
  directions' states: o_t = (S_fwd_t + S_bwd_t) q  (``combine="sum"``);
  ``combine="fwd_incl_bwd_excl"`` is kept for study only;
* the backward scan decays with the alpha_t of the frame being absorbed,
  i.e. the same recurrence run on the reversed frame sequence;
* no scale is applied to q in the read-out.
"""

import numpy as np


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def vda_prep(k, v, beta, T, N, H, d):
    """A_t,h = sum_i beta_i k_i k_i^T and B_t,h = sum_i beta_i v_i k_i^T.

    Sums run over the N spatial tokens of frame t (方法概述 item 2: A_t gathers
    key correlations, B_t gathers value-key writes).  Returns two float64
    arrays of shape [T, H, d, d]; B is indexed [v_dim, k_dim].
    """
    A = np.zeros((T, H, d, d))
    B = np.zeros((T, H, d, d))
    for t in range(T):
        rows = slice(t * N, (t + 1) * N)
        for h in range(H):
            cols = slice(h * d, (h + 1) * d)
            Kt = _f64(k[rows, cols])                # [N, d]
            Vt = _f64(v[rows, cols])                # [N, d]
            bK = _f64(beta[rows, h])[:, None] * Kt  # beta_i k_i
            A[t, h] = Kt.T @ bK                     # sum beta k k^T
            B[t, h] = Vt.T @ bK                     # sum beta v k^T
    return A, B


def vda_frame_state(S_bar, A, B):
    """One frame of the delta rule: S = (S_bar + B)(I + A)^-1.

    Solved as (I + A) S^T = (S_bar + B)^T (I + A is symmetric), without
    forming the inverse.
    """
    d = A.shape[-1]
    M = np.eye(d) + A
    return np.linalg.solve(M, (S_bar + B).T).T


def transition_matrix(alpha_t, A):
    """Inherited-state transition M_t = alpha_t (I + A_t)^-1.

    S_t = S_{t-1} M_t + B_t (I + A_t)^-1, so M_t is what an earlier frame's
    contribution is multiplied by at frame t.  The article (方法概述 item 2)
    states ||M_t||_2 <= 1.
    """
    d = A.shape[-1]
    return alpha_t * np.linalg.inv(np.eye(d) + A)


def vda_scan(A, B, alpha):
    """Forward and backward frame scans.

    Forward:  S_fwd_t = (alpha_t S_fwd_{t-1} + B_t)(I + A_t)^-1, S_fwd_{-1} = 0.
    Backward: S_bwd_t = (alpha_t S_bwd_{t+1} + B_t)(I + A_t)^-1, S_bwd_T = 0.
    Returns (S_fwd, S_bwd), each [T, H, d, d] float64.
    """
    A, B, alpha = _f64(A), _f64(B), _f64(alpha)
    T, H, d, _ = A.shape
    S_fwd = np.zeros((T, H, d, d))
    S_bwd = np.zeros((T, H, d, d))
    for h in range(H):
        S = np.zeros((d, d))
        for t in range(T):
            S = vda_frame_state(alpha[t, h] * S, A[t, h], B[t, h])
            S_fwd[t, h] = S
        S = np.zeros((d, d))
        for t in range(T - 1, -1, -1):
            S = vda_frame_state(alpha[t, h] * S, A[t, h], B[t, h])
            S_bwd[t, h] = S
    return S_fwd, S_bwd


def vda_readout(q, S_fwd, S_bwd, T, N, H, d, combine="sum", rows=None):
    """o[r, h] = (S_fwd_t + S_bwd_t) q_r for every token r of frame t.

    ``combine="fwd_incl_bwd_excl"`` reads S_fwd_t q + S_bwd_{t+1} q instead
    (study only).  ``rows`` restricts the output to the given token rows
    (the result then has len(rows) rows).
    """
    if combine not in ("sum", "fwd_incl_bwd_excl"):
        raise ValueError(combine)
    L = T * N
    rows = np.arange(L) if rows is None else np.asarray(rows, dtype=np.int64)
    out = np.zeros((len(rows), H * d))
    frames = rows // N
    for t in np.unique(frames):
        sel = np.nonzero(frames == t)[0]
        Qt = _f64(q[rows[sel]])                     # the tokens of frame t
        for h in range(H):
            if combine == "sum":
                S = S_fwd[t, h] + S_bwd[t, h]
            else:
                S = S_fwd[t, h] + (S_bwd[t + 1, h] if t + 1 < T else 0.0)
            # o_r = S q_r for each row r: rows of Q times S^T
            out[sel, h * d:(h + 1) * d] = Qt[:, h * d:(h + 1) * d] @ S.T
    return out


def vda(q, k, v, beta, alpha, T, N, H, d, combine="sum", rows=None):
    """Full VDA branch: prep, per-frame closed-form solve, both scans, read-out.

    Returns (o_vda [L or len(rows), H*d], S_fwd, S_bwd), float64.
    """
    A, B = vda_prep(k, v, beta, T, N, H, d)
    S_fwd, S_bwd = vda_scan(A, B, alpha)
    o = vda_readout(q, S_fwd, S_bwd, T, N, H, d, combine=combine, rows=rows)
    return o, S_fwd, S_bwd
