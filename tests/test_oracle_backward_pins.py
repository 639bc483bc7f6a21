"""Pins of the VDA backward oracle: central finite differences of a scalar
loss, and automatic differentiation of an independent torch float64
forward (written here from the definition, sharing nothing with oracle/)."""

import numpy as np
import pytest
import torch

import oracle
from video_diffusion_hybrid_vda_b200 import synth


def _inputs(T, N, H, d, seed):
    s = synth.Shape(T, N, H, d)
    x = {k: v.numpy().astype(np.float64)
         for k, v in synth.make_inputs(s, dtype=torch.float32, seed=seed).items()}
    dO = np.random.default_rng(seed).standard_normal((s.L, s.D))
    return s, x, dO


def _torch_vda(q, k, v, beta, alpha, T, N, H, d):
    """Forward VDA in torch float64, from the definition."""
    outs = []
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        I = torch.eye(d, dtype=torch.float64)
        As, Bs = [], []
        for t in range(T):
            r = slice(t * N, (t + 1) * N)
            K, V, b = k[r, c], v[r, c], beta[r, h]
            As.append((K * b[:, None]).T @ K)
            Bs.append((V * b[:, None]).T @ K)
        fwd, bwd = [None] * T, [None] * T
        S = torch.zeros((d, d), dtype=torch.float64)
        for t in range(T):
            S = torch.linalg.solve(I + As[t], (alpha[t, h] * S + Bs[t]).T).T
            fwd[t] = S
        S = torch.zeros((d, d), dtype=torch.float64)
        for t in range(T - 1, -1, -1):
            S = torch.linalg.solve(I + As[t], (alpha[t, h] * S + Bs[t]).T).T
            bwd[t] = S
        o = torch.cat([q[t * N:(t + 1) * N, c] @ (fwd[t] + bwd[t]).T for t in range(T)])
        outs.append(o)
    return torch.cat(outs, dim=1)


@pytest.mark.parametrize("T,N,H,d", [(5, 3, 2, 4), (1, 4, 1, 3), (7, 1, 1, 5)])
def test_backward_matches_autograd_of_independent_forward(T, N, H, d):
    s, x, dO = _inputs(T, N, H, d, seed=T * 10 + N)
    tens = {n: torch.tensor(x[n], requires_grad=True) for n in ("q", "k", "v", "beta", "alpha")}
    o = _torch_vda(tens["q"], tens["k"], tens["v"], tens["beta"], tens["alpha"], T, N, H, d)
    (o * torch.tensor(dO)).sum().backward()
    got = oracle.vda_backward(x["q"], x["k"], x["v"], x["beta"], x["alpha"], dO, T, N, H, d)
    for g, n in zip(got, ("q", "k", "v", "beta", "alpha")):
        np.testing.assert_allclose(g, tens[n].grad.numpy(), rtol=1e-9, atol=1e-11, err_msg=n)


def test_backward_matches_finite_differences():
    T, N, H, d = 4, 3, 1, 3
    s, x, dO = _inputs(T, N, H, d, seed=5)

    def loss(xx):
        o, _, _ = oracle.vda(xx["q"], xx["k"], xx["v"], xx["beta"], xx["alpha"], T, N, H, d)
        return float(np.sum(o * dO))

    grads = dict(zip(("q", "k", "v", "beta", "alpha"),
                     oracle.vda_backward(x["q"], x["k"], x["v"], x["beta"], x["alpha"], dO,
                                         T, N, H, d)))
    rng = np.random.default_rng(0)
    eps = 1e-6
    for n in ("q", "k", "v", "beta", "alpha"):
        for _ in range(4):
            idx = tuple(rng.integers(0, dim) for dim in x[n].shape)
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[n][idx] += eps
            xm[n][idx] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            assert abs(fd - grads[n][idx]) <= 1e-6 * (1 + abs(fd)), (n, idx, fd, grads[n][idx])
