"""Gradients of Video Delta Attention, float64 CPU oracle.  TEST INFRASTRUCTURE ONLY.

The forward is the one in vda.py ("Video DeltaNet", 10100.com article,
方法概述 item 2): per head, A_t = sum beta k k^T, B_t = sum beta v k^T,
P_t = (I + A_t)^-1, S_fwd_t = (alpha_t S_fwd_{t-1} + B_t) P_t,
S_bwd_t = (alpha_t S_bwd_{t+1} + B_t) P_t, o_i = (S_fwd_t + S_bwd_t) q_i.
The article describes the staged alignment that trains this branch (方法概述
item 3); training needs these gradients.  Given dO = dLoss/do_vda:

  G_t      = sum_{i in t} dO_i q_i^T                  (dLoss/dS, each direction)
  dq_i     = (S_fwd_t + S_bwd_t)^T dO_i
  adjoint of the forward scan (reverse time):  D_fwd_t = (alpha_{t+1} D_fwd_{t+1} + G_t) P_t
  adjoint of the backward scan (forward time): D_bwd_t = (alpha_{t-1} D_bwd_{t-1} + G_t) P_t
  dB_t     = D_fwd_t + D_bwd_t
  dA_t     = -(S_fwd_t^T D_fwd_t + S_bwd_t^T D_bwd_t)
  dalpha_t = <D_fwd_t, S_fwd_{t-1}> + <D_bwd_t, S_bwd_{t+1}>
  dk_i     = beta_i ((dA_t + dA_t^T) k_i + dB_t^T v_i)
  dv_i     = beta_i dB_t k_i
  dbeta_i  = k_i^T dA_t k_i + v_i^T dB_t k_i

(D_t is dLoss with respect to the state before its (I + A_t)^-1 factor;
dA_t uses S_t = U_t P_t, dLoss/dP_t = U_t^T (dLoss/dS_t) and
dLoss/dA_t = -P_t (dLoss/dP_t) P_t.)  The test file pins these against
finite differences and against automatic differentiation of an independent
torch float64 forward.
"""

import numpy as np

from .vda import vda_prep, vda_scan


def vda_backward(q, k, v, beta, alpha, dO, T, N, H, d):
    """Returns (dq, dk, dv [L, H*d], dbeta [L, H], dalpha [T, H]) in float64."""
    q, k, v = (np.asarray(a, dtype=np.float64) for a in (q, k, v))
    beta, alpha, dO = (np.asarray(a, dtype=np.float64) for a in (beta, alpha, dO))
    A, B = vda_prep(k, v, beta, T, N, H, d)
    S_fwd, S_bwd = vda_scan(A, B, alpha)
    L = T * N
    dq, dk, dv = np.zeros((L, H * d)), np.zeros((L, H * d)), np.zeros((L, H * d))
    dbeta, dalpha = np.zeros((L, H)), np.zeros((T, H))
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        P = [np.linalg.inv(np.eye(d) + A[t, h]) for t in range(T)]
        G = [dO[t * N:(t + 1) * N, c].T @ q[t * N:(t + 1) * N, c] for t in range(T)]
        Df = [None] * T
        nxt = np.zeros((d, d))
        for t in range(T - 1, -1, -1):
            a_next = alpha[t + 1, h] if t + 1 < T else 0.0
            Df[t] = (a_next * nxt + G[t]) @ P[t]
            nxt = Df[t]
        Db = [None] * T
        prv = np.zeros((d, d))
        for t in range(T):
            a_prev = alpha[t - 1, h] if t > 0 else 0.0
            Db[t] = (a_prev * prv + G[t]) @ P[t]
            prv = Db[t]
        for t in range(T):
            rows = slice(t * N, (t + 1) * N)
            dB = Df[t] + Db[t]
            dA = -(S_fwd[t, h].T @ Df[t] + S_bwd[t, h].T @ Db[t])
            da = 0.0
            if t > 0:
                da += np.sum(Df[t] * S_fwd[t - 1, h])
            if t + 1 < T:
                da += np.sum(Db[t] * S_bwd[t + 1, h])
            dalpha[t, h] = da
            Kt, Vt, Qt, dOt = k[rows, c], v[rows, c], q[rows, c], dO[rows, c]
            b = beta[rows, h][:, None]
            dq[rows, c] = dOt @ (S_fwd[t, h] + S_bwd[t, h])
            dk[rows, c] = b * (Kt @ (dA + dA.T) + Vt @ dB)
            dv[rows, c] = b * (Kt @ dB.T)
            dbeta[rows, h] = np.einsum("ij,ij->i", Kt @ dA.T, Kt) + np.einsum("ij,ij->i", Kt @ dB.T, Vt)
    return dq, dk, dv, dbeta, dalpha
