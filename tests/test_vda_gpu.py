"""Parity of vdn_vda_scan (CUDA, through the C ABI) against the CPU oracle.

Small shapes are compared element by element on every intermediate
(A, B from prep; P from the solve; both scans' states; o_vda).  The
full-size shapes (42/102 latent frames x 4032 tokens) are compared on every
head's states (all frames) and sampled token rows; the scan sweep on one
head's states and sampled rows.
"""

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import (TOL_BF16, TOL_STATE, elementwise_rel, TOL_ELEMENTWISE, ensure_built, host, max_rel,
                               per_head_max_rel)
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu

# prep carries beta*k as a bf16 hi/lo pair (~2^-17 relative per term):
# A and B are compared at 1e-4 of their max; states and outputs at the layer
# tolerances.
TOL_PREP = 1e-4
TOL_SOLVE = 1e-4


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _inputs(shape, seed=0, ld_pad=0):
    inp = synth.make_inputs(shape, dtype=torch.bfloat16, seed=seed, device="cuda")
    if ld_pad:
        for name in ("q", "k", "v"):
            t = inp[name]
            big = torch.full((t.shape[0], t.shape[1] + ld_pad), float("nan"),
                             dtype=t.dtype, device=t.device)
            big[:, :t.shape[1]] = t
            inp[name] = big[:, :t.shape[1]]
    return inp


def _run(vdn, shape, inp, with_states=True):
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    states = torch.empty((2, T, H, d, d), dtype=torch.float32, device="cuda") if with_states else None
    o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H, d,
                         states=states)
    assert vdn.get_device_status(ws) == 0
    return o, states, ws


SMALL = [
    (7, 200, 2, 128),   # ragged prep tail (200 = 6*32 + 8) and read-out tail (200 = 128 + 72)
    (7, 200, 2, 64),
    (12, 96, 3, 128),   # N below one read-out tile
    (1, 130, 1, 128),   # single frame (ridge regression)
    (5, 1, 3, 64),      # one token per frame (per-token delta rule)
    (4, 1, 2, 128),
    (3, 4032, 1, 128),  # the full 48x84 frame, several tiles per frame
    (17, 33, 2, 64),
    (3, 40, 26, 128),   # 156 CTAs of 48-row blocks would not fit 148 SMs: 64-row blocks
    (3, 20, 40, 64),    # likewise at d = 64 (one 64-row block per state)
]


@pytest.mark.parametrize("T,N,H,d", SMALL)
def test_vda_parity_small(vdn, T, N, H, d, report_metric):
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=T * 1000 + N)
    o, states, ws = _run(vdn, shape, inp)
    x = {k: host(v) for k, v in inp.items()}
    A_ref, B_ref = oracle.vda_prep(x["k"], x["v"], x["beta"], T, N, H, d)
    A, B, P = (host(t) for t in vdn.vda_debug_buffers(ws, T, N, H, d))
    for t in range(T):
        for h in range(H):
            assert max_rel(A[t, h], A_ref[t, h]) <= TOL_PREP, ("A", t, h)
            assert max_rel(B[t, h], B_ref[t, h]) <= TOL_PREP, ("B", t, h)
            # solve checked on the GPU's own A and B
            A_sym = 0.5 * (A[t, h].astype(np.float64) + A[t, h].T.astype(np.float64))
            P_ref = np.linalg.inv(np.eye(d) + A_sym)
            assert max_rel(P[t, h], P_ref) <= TOL_SOLVE, ("P", t, h)
    S_fwd, S_bwd = oracle.vda_scan(A_ref, B_ref, x["alpha"])
    st = host(states)
    for t in range(T):
        for h in range(H):
            assert max_rel(st[0, t, h], S_fwd[t, h]) <= TOL_STATE, ("fwd", t, h)
            assert max_rel(st[1, t, h], S_bwd[t, h]) <= TOL_STATE, ("bwd", t, h)
    o_ref = oracle.vda_readout(x["q"], S_fwd, S_bwd, T, N, H, d)
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16
    err_el = elementwise_rel(host(o), o_ref)
    report_metric("o_vda_elementwise_rel", err_el)
    assert err_el <= TOL_ELEMENTWISE


def test_vda_strided_rows(vdn):
    """ld > H*d on the inputs and the output."""
    shape = synth.Shape(6, 150, 2, 64)
    inp = _inputs(shape, seed=5, ld_pad=40)
    out = torch.full((shape.L, shape.D + 24), float("nan"), dtype=torch.bfloat16, device="cuda")
    o_view = out[:, :shape.D]
    o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], *shape_args(shape),
                         out=o_view)
    assert vdn.get_device_status(ws) == 0
    assert torch.isnan(out[:, shape.D:].float()).all()        # padding untouched
    x = {k: host(v) for k, v in inp.items()}
    o_ref, _, _ = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], *shape_args(shape))
    assert per_head_max_rel(host(o_view), o_ref, shape.H, shape.d) <= TOL_BF16


def shape_args(s):
    return s.T, s.N, s.H, s.d


def _sampled_parity(vdn, shape, heads, n_rows=48, seed=0):
    T, N, H, d = shape_args(shape)
    inp = _inputs(shape, seed=seed)
    o, states, ws = _run(vdn, shape, inp)
    rng = np.random.default_rng(seed)
    # rows: frame starts and ends, the ragged last read-out tile, random
    rows = sorted(set([0, N - 1, N, T * N - 1, (T - 1) * N, (T - 1) * N + (N // 128) * 128] +
                      list(rng.integers(0, T * N, n_rows))))
    rows = np.array([r for r in rows if r < T * N])
    o_gpu = host(o[torch.as_tensor(rows, device="cuda")])
    st = states
    for h in heads:
        c = slice(h * d, (h + 1) * d)
        k = host(inp["k"][:, c])
        v = host(inp["v"][:, c])
        beta = host(inp["beta"][:, h:h + 1])
        alpha = host(inp["alpha"][:, h:h + 1])
        A_ref, B_ref = oracle.vda_prep(k, v, beta, T, N, 1, d)
        S_fwd, S_bwd = oracle.vda_scan(A_ref, B_ref, alpha)
        sf = host(st[0, :, h])
        sb = host(st[1, :, h])
        for t in range(T):
            assert max_rel(sf[t], S_fwd[t, 0]) <= TOL_STATE, ("fwd", t, h)
            assert max_rel(sb[t], S_bwd[t, 0]) <= TOL_STATE, ("bwd", t, h)
        q = host(inp["q"][torch.as_tensor(rows, device="cuda")][:, c])
        o_ref = np.zeros((len(rows), d))
        for j, r in enumerate(rows):
            t = r // N
            o_ref[j] = (S_fwd[t, 0] + S_bwd[t, 0]) @ q[j]
        assert max_rel(o_gpu[:, c], o_ref) <= TOL_BF16, ("o", h)
    del inp, o, states, ws
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [42, 102])
def test_vda_parity_full_layer_all_heads(vdn, T):
    _sampled_parity(vdn, synth.Shape(T, 4032, 24, 128), heads=range(24))


@pytest.mark.parametrize("shape", synth.sweep_shapes(), ids=lambda s: f"T{s.T}N{s.N}d{s.d}H{s.H}")
def test_vda_parity_scan_sweep_sampled(vdn, shape):
    # first, middle and last head: all frames' states and 48 sampled rows each
    _sampled_parity(vdn, shape, heads=[0, shape.H // 2, shape.H - 1], n_rows=48, seed=1)


def test_vda_timeout_path_reports_and_recovers(vdn):
    """A zero wait budget makes the pipelined kernels give up at their first
    unsatisfied wait: the call still returns, the status word says TIMEOUT,
    and the next call with the normal budget is correct."""
    shape = synth.Shape(6, 300, 2, 128)
    inp = _inputs(shape, seed=9)
    try:
        vdn.set_wait_budget_ns(0)
        o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                             *shape_args(shape))
        assert vdn.get_device_status(ws) == 6
    finally:
        vdn.set_wait_budget_ns(2_000_000_000)
    vdn.reset_device_status(ws)
    o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                         *shape_args(shape), ws=ws)
    assert vdn.get_device_status(ws) == 0
    x = {k: host(v) for k, v in inp.items()}
    o_ref, _, _ = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], *shape_args(shape))
    assert per_head_max_rel(host(o), o_ref, shape.H, shape.d) <= TOL_BF16


@pytest.mark.parametrize("solver", ["cholesky", "gauss-jordan"])
@pytest.mark.parametrize("T,N,H,d", [(7, 200, 2, 128), (17, 33, 2, 64), (3, 4032, 1, 128)])
def test_vda_solvers(vdn, solver, T, N, H, d):
    """Both solves: P against the GPU's own symmetrised A (inverted in
    float64 here), states and o_vda against the oracle."""
    shape = synth.Shape(T, N, H, d)
    inp = _inputs(shape, seed=T * 1000 + N + 1)
    try:
        vdn.set_vda_solver(vdn.SOLVER_GAUSS_JORDAN if solver == "gauss-jordan"
                           else vdn.SOLVER_CHOLESKY)
        o, states, ws = _run(vdn, shape, inp)
    finally:
        vdn.set_vda_solver(vdn.SOLVER_DEFAULT)
    x = {k: host(v) for k, v in inp.items()}
    A, B, P = (host(t) for t in vdn.vda_debug_buffers(ws, T, N, H, d))
    for t in range(T):
        for h in range(H):
            A_sym = 0.5 * (A[t, h].astype(np.float64) + A[t, h].T.astype(np.float64))
            P_ref = np.linalg.inv(np.eye(d) + A_sym)
            assert max_rel(P[t, h], P_ref) <= TOL_SOLVE, ("P", t, h)
    o_ref, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], T, N, H, d)
    st = host(states)
    for t in range(T):
        for h in range(H):
            assert max_rel(st[0, t, h], S_fwd[t, h]) <= TOL_STATE
            assert max_rel(st[1, t, h], S_bwd[t, h]) <= TOL_STATE
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16


def test_vda_solver_rejects_unknown(vdn):
    with pytest.raises(vdn.VdnError):
        vdn.set_vda_solver(7)


@pytest.mark.parametrize("solver", [0, 1])
@pytest.mark.parametrize("fault", ["nan", "indefinite"])
def test_vda_numeric_failure_reports_and_recovers(vdn, solver, fault):
    """Failures made on the host, none of which faults the GPU: a NaN in beta
    makes A_t NaN, and a beta of -50 on every token of one frame makes
    I + A_t indefinite (1 - 50 lambda_max < 0).  Either way some pivot of the
    solve is NaN or non-positive (Sylvester: an SPD-less symmetric matrix has
    a non-positive leading pivot, for Cholesky and for Gauss-Jordan without
    pivoting alike), the status word reads VDN_ERR_NUMERIC, and the next call
    on the same workspace after a reset is correct."""
    shape = synth.Shape(4, 40, 2, 64)
    inp = _inputs(shape, seed=21)
    bad = inp["beta"].clone()
    if fault == "nan":
        bad[45, 1] = float("nan")
    else:
        bad[2 * shape.N:3 * shape.N, 0] = -50.0
    try:
        vdn.set_vda_solver(solver)
        o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], bad, inp["alpha"],
                             *shape_args(shape))
        assert vdn.get_device_status(ws) == 5          # VDN_ERR_NUMERIC
        vdn.reset_device_status(ws)
        o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                             *shape_args(shape), ws=ws)
        assert vdn.get_device_status(ws) == 0
    finally:
        vdn.set_vda_solver(vdn.SOLVER_DEFAULT)
    x = {k: host(v) for k, v in inp.items()}
    o_ref, _, _ = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], *shape_args(shape))
    assert per_head_max_rel(host(o), o_ref, shape.H, shape.d) <= TOL_BF16
