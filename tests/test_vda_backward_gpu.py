"""Parity of vdn_vda_backward (CUDA, through the C ABI) against the CPU
oracle's VDA gradients (float64, adjoint scans).

dq, dk, dv are bf16 outputs and dbeta is formed from bf16-rounded E and dB
operands of the tensor-core products: all four are held to the bf16 output
tolerance (2e-2 of each head's max).  dalpha is an fp32 inner product of
fp32 states and adjoint states: it is held to the state tolerance (1e-3).
"""

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import TOL_BF16, TOL_STATE, ensure_built, host, max_rel, per_head_max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _inputs(shape, seed):
    inp = synth.make_inputs(shape, dtype=torch.bfloat16, seed=seed, device="cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 7)
    inp["d_o"] = torch.randn((shape.L, shape.D), generator=g, device="cuda").to(torch.bfloat16)
    return inp


def _padded(t, pad, fill=float("nan")):
    big = torch.full((t.shape[0], t.shape[1] + pad), fill, dtype=t.dtype, device=t.device)
    big[:, :t.shape[1]] = t
    return big[:, :t.shape[1]]


def _run(vdn, shape, inp, **kw):
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    dq, dk, dv, dbeta, dalpha, ws = vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"],
                                                     inp["alpha"], inp["d_o"], T, N, H, d, **kw)
    assert vdn.get_device_status(ws) == 0
    return dq, dk, dv, dbeta, dalpha, ws


def _oracle(x, T, N, H, d):
    return oracle.vda_backward(x["q"], x["k"], x["v"], x["beta"], x["alpha"], x["d_o"],
                               T, N, H, d)


def _check(got, ref, H, d):
    names = ("dq", "dk", "dv")
    for g, r, n in zip(got[:3], ref[:3], names):
        assert per_head_max_rel(g, r, H, d) <= TOL_BF16, n
    for h in range(H):
        assert max_rel(got[3][:, h], ref[3][:, h]) <= TOL_BF16, ("dbeta", h)
        assert max_rel(got[4][:, h], ref[4][:, h]) <= TOL_STATE, ("dalpha", h)


SMALL = [
    (7, 200, 2, 128),   # ragged tails of the prep (32-row) and token (128-row) tiles
    (7, 200, 2, 64),
    (12, 96, 3, 128),   # N below one token tile
    (1, 130, 1, 128),   # single frame: no carried adjoint, dalpha = 0
    (5, 1, 3, 64),      # one token per frame
    (4, 1, 2, 128),
    (3, 4032, 1, 128),  # the full 48x84 frame, 32 token tiles per frame
    (17, 33, 2, 64),
    (9, 70, 2, 32),     # padded head dims
    (6, 50, 3, 16),
    (3, 40, 26, 128),   # many heads: the adjoint scan's 64-row blocks
]


@pytest.mark.parametrize("T,N,H,d", SMALL)
def test_vda_backward_parity_small(vdn, T, N, H, d):
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=T * 100 + N + d)
    got = [host(t) for t in _run(vdn, shape, inp)[:5]]
    ref = _oracle({k: host(v) for k, v in inp.items()}, T, N, H, d)
    _check(got, ref, H, d)
    if T == 1:
        assert np.all(got[4] == 0.0)


def test_vda_backward_adjoint_states(vdn):
    """The adjoint states in the workspace against the oracle's recurrences,
    and E = dA + dA^T symmetric."""
    T, N, H, d = 9, 150, 2, 128
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=11)
    ws = _run(vdn, shape, inp)[5]
    states, adj, E = (host(t) for t in vdn.vda_backward_debug_buffers(ws, T, N, H, d))
    x = {k: host(v).astype(np.float64) for k, v in inp.items()}
    A_ref, B_ref = oracle.vda_prep(x["k"], x["v"], x["beta"], T, N, H, d)
    Sf, Sb = oracle.vda_scan(A_ref, B_ref, x["alpha"])
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        P = [np.linalg.inv(np.eye(d) + A_ref[t, h]) for t in range(T)]
        G = [x["d_o"][t * N:(t + 1) * N, c].T @ x["q"][t * N:(t + 1) * N, c] for t in range(T)]
        Db = np.zeros((d, d))
        for t in range(T):
            Db = ((x["alpha"][t - 1, h] * Db if t else 0.0) + G[t]) @ P[t]
            assert max_rel(adj[0, t, h], Db) <= TOL_STATE, ("D_bwd", t, h)
        Df = np.zeros((d, d))
        for t in range(T - 1, -1, -1):
            Df = ((x["alpha"][t + 1, h] * Df if t + 1 < T else 0.0) + G[t]) @ P[t]
            assert max_rel(adj[1, t, h], Df) <= TOL_STATE, ("D_fwd", t, h)
        for t in range(T):
            assert max_rel(states[0, t, h], Sf[t, h]) <= TOL_STATE
            assert max_rel(states[1, t, h], Sb[t, h]) <= TOL_STATE
            np.testing.assert_array_equal(E[t, h], E[t, h].T)


def test_vda_backward_strided(vdn):
    """Row strides above H*d on every activation; columns past H*d of the
    outputs stay untouched."""
    T, N, H, d = 6, 140, 2, 64
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=5)
    strided = dict(inp)
    for name in ("q", "k", "v"):
        strided[name] = _padded(inp[name], 24)
    strided["d_o"] = _padded(inp["d_o"], 8)
    L, D = shape.L, shape.D
    outs = [_padded(torch.zeros((L, D), dtype=torch.bfloat16, device="cuda"), 40, 7.0)
            for _ in range(3)]
    got = _run(vdn, shape, strided, dq=outs[0], dk=outs[1], dv=outs[2])
    for o in outs:
        full = o.as_strided((L, D + 40), (D + 40, 1))
        assert torch.all(full[:, D:] == 7.0)
    ref = _oracle({k: host(v) for k, v in inp.items()}, T, N, H, d)
    _check([host(t) for t in got[:5]], ref, H, d)


def test_vda_backward_full_sampled_heads(vdn):
    """The full hybrid block's shape (102 x 4032 tokens, 24 heads of 128):
    heads 0 and 23 against the oracle on every token (heads are
    independent, so the oracle runs on each head's slice alone)."""
    T, N, H, d = 102, 4032, 24, 128
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=0)
    dq, dk, dv, dbeta, dalpha, ws = _run(vdn, shape, inp)
    for h in (0, 23):
        c = slice(h * d, (h + 1) * d)
        x = {n: host(inp[n][:, c]) for n in ("q", "k", "v", "d_o")}
        x["beta"] = host(inp["beta"][:, h:h + 1])
        x["alpha"] = host(inp["alpha"][:, h:h + 1])
        ref = _oracle(x, T, N, 1, d)
        got = [host(dq[:, c]), host(dk[:, c]), host(dv[:, c]), host(dbeta[:, h:h + 1]),
               host(dalpha[:, h:h + 1])]
        _check(got, ref, 1, d)
    del inp, dq, dk, dv, ws
    torch.cuda.empty_cache()


def test_vda_backward_rejects_bad_arguments(vdn):
    shape = synth.Shape(2, 16, 1, 128)
    inp = _inputs(shape, seed=1)
    with pytest.raises(vdn.VdnError):
        vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], inp["d_o"],
                         2, 16, 1, 96)
    with pytest.raises(vdn.VdnError):
        vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], inp["d_o"],
                         2, 16, 1, 128, ws=vdn.alloc_workspace(1024))


@pytest.mark.parametrize("T,N,H,d", [(7, 200, 2, 128), (9, 70, 2, 32)])
def test_vda_backward_reuses_a_forward_on_its_workspace(vdn, T, N, H, d):
    """A forward run on the gradient pass's workspace (states kept inside)
    hands P and the states over: the gradients equal those of the
    recomputing pass bit for bit."""
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=T + N)
    ref = _run(vdn, shape, inp)[:5]
    ws = vdn.alloc_workspace(vdn.vda_backward_workspace(T, N, H, d))
    o, _ = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H, d,
                        ws=ws)
    got = _run(vdn, shape, inp, ws=ws, reuse_forward=True)[:5]
    for g, r in zip(got, ref):
        assert torch.equal(g, r)

