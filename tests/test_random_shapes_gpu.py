"""Seeded random shapes through every entry point against the oracle:
frames, tokens per frame (ragged against every tile size), heads, head dims
(padded and native), mask parameters, row strides and context lengths."""

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import TOL_BF16, TOL_STATE, ensure_built, host, max_rel, per_head_max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu

SEEDS = list(range(12))


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _case(seed):
    rng = np.random.default_rng(1000 + seed)
    T = int(rng.integers(1, 24))
    N = int(rng.choice([1, 7, 33, 64, 100, 129, 250, 300]))
    H = int(rng.integers(1, 4))
    d = int(rng.choice([16, 32, 64, 128]))
    pad = int(rng.choice([0, 8, 24]))
    return synth.Shape(T, N, H, d), pad, rng


def _strided(t, pad):
    if pad == 0:
        return t
    big = torch.full((t.shape[0], t.shape[1] + pad), float("nan"), dtype=t.dtype, device=t.device)
    big[:, :t.shape[1]] = t
    return big[:, :t.shape[1]]


@pytest.mark.parametrize("seed", SEEDS)
def test_random_vda(vdn, seed):
    s, pad, _ = _case(seed)
    inp = synth.make_inputs(s, seed=seed, device="cuda")
    q, k, v = (_strided(inp[n], pad) for n in ("q", "k", "v"))
    states = torch.empty((2, s.T, s.H, s.d, s.d), device="cuda")
    o, ws = vdn.vda_scan(q, k, v, inp["beta"], inp["alpha"], s.T, s.N, s.H, s.d, states=states)
    assert vdn.get_device_status(ws) == 0
    x = {n: host(inp[n]) for n in ("q", "k", "v", "beta", "alpha")}
    o_ref, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"],
                                     s.T, s.N, s.H, s.d)
    st = host(states)
    for t in range(s.T):
        for h in range(s.H):
            assert max_rel(st[0, t, h], S_fwd[t, h]) <= TOL_STATE
            assert max_rel(st[1, t, h], S_bwd[t, h]) <= TOL_STATE
    assert per_head_max_rel(host(o), o_ref, s.H, s.d) <= TOL_BF16


@pytest.mark.parametrize("seed", SEEDS)
def test_random_window_attn(vdn, seed):
    s, pad, rng = _case(seed)
    cf = int(rng.integers(1, 7))
    wc = int(rng.integers(0, 3))
    an = int(rng.integers(0, 4))
    m_ctx = int(rng.choice([0, 0, 5, 140])) if s.d >= 64 else 0
    inp = synth.make_inputs(s, seed=seed + 50, device="cuda")
    q, k, v = (_strided(inp[n], pad) for n in ("q", "k", "v"))
    ck = cv = None
    if m_ctx:
        g = torch.Generator(device="cuda").manual_seed(seed)
        ck = torch.randn((m_ctx, s.D), generator=g, device="cuda").to(torch.bfloat16)
        cv = torch.randn((m_ctx, s.D), generator=g, device="cuda").to(torch.bfloat16)
    lse = torch.empty((s.H, s.L), device="cuda")
    o, ws = vdn.window_attn(q, k, v, s.T, s.N, s.H, s.d, cf, wc, an, lse=lse, ctx_k=ck, ctx_v=cv)
    assert vdn.get_device_status(ws) == 0
    x = {n: host(inp[n]) for n in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d, cf, wc, an,
                                        ctx_k=host(ck) if m_ctx else None,
                                        ctx_v=host(cv) if m_ctx else None)
    assert per_head_max_rel(host(o), o_ref, s.H, s.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("seed", SEEDS[:6])
def test_random_fuse(vdn, seed):
    s, _, rng = _case(seed)
    inp = synth.make_inputs(s, seed=seed + 90, device="cuda", with_fuse=True)
    g = torch.Generator(device="cuda").manual_seed(seed)
    o_s = torch.randn((s.L, s.D), generator=g, device="cuda").to(torch.bfloat16)
    o_l = torch.randn((s.L, s.D), generator=g, device="cuda").to(torch.bfloat16)
    y, ws = vdn.hybrid_fuse(inp["x"], o_s, o_l, inp["W_gs"], inp["W_gl"], inp["gamma"],
                            inp["W_os"], inp["W_ol"], s.H)
    assert vdn.get_device_status(ws) == 0
    ref = oracle.hybrid_fuse(host(inp["x"]), host(o_s), host(o_l), host(inp["W_gs"]),
                             host(inp["W_gl"]), host(inp["gamma"]), 1e-6, host(inp["W_os"]),
                             host(inp["W_ol"]), s.H)
    assert max_rel(host(y), ref) <= TOL_BF16
