"""Parity of vdn_window_attn (CUDA, through the C ABI) against the CPU oracle.

Small shapes: every output row and the log-sum-exp, over mask variants.
Full-size layers (42 and 102 latent frames x 4032 tokens x 24 heads): rows
sampled from anchor frames, chunk edges, the ragged last chunk and at
random, for several heads.
"""

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import elementwise_rel, TOL_ELEMENTWISE, TOL_BF16, ensure_built, host, max_rel, per_head_max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-3  # absolute, natural log (fp32 accumulation of bf16 products)


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _run(vdn, shape, inp, **kw):
    lse = torch.empty((shape.H, shape.L), dtype=torch.float32, device="cuda")
    o, ws = vdn.window_attn(inp["q"], inp["k"], inp["v"], shape.T, shape.N, shape.H, shape.d,
                            lse=lse, **kw)
    assert vdn.get_device_status(ws) == 0
    return o, lse


SMALL = [
    (10, 64, 2, 128),    # 2 chunks: every frame visible
    (17, 100, 2, 128),   # ragged last chunk, key tiles straddle frames
    (23, 130, 1, 64),
    (12, 256, 2, 128),   # tiles align with frames
    (7, 1, 1, 128),      # one token per frame
    (31, 40, 3, 64),
]


@pytest.mark.parametrize("T,N,H,d", SMALL)
def test_window_attn_parity_small(vdn, T, N, H, d, report_metric):
    shape = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(shape, seed=T * 100 + N, device="cuda")
    o, lse = _run(vdn, shape, inp)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], T, N, H, d)
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE
    err_el = elementwise_rel(host(o), o_ref)
    report_metric("o_s_elementwise_rel", err_el)
    assert err_el <= TOL_ELEMENTWISE


@pytest.mark.parametrize("cf,wc,anchors,scale", [
    (5, 1, 0, 0.0), (5, 1, 1, 0.0), (5, 1, 2, 0.0), (5, 0, 3, 0.0), (5, 2, 3, 0.0),
    (3, 1, 3, 0.0), (5, 1, 3, 0.2),
])
def test_window_attn_mask_variants(vdn, cf, wc, anchors, scale):
    shape = synth.Shape(26, 72, 2, 128)
    inp = synth.make_inputs(shape, seed=cf * 10 + wc + anchors, device="cuda")
    o, lse = _run(vdn, shape, inp, chunk_frames=cf, window_chunks=wc, anchors=anchors,
                  scale=scale)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], *shape_args(shape),
                                        chunk_frames=cf, window_chunks=wc, anchors=anchors,
                                        scale=scale)
    assert per_head_max_rel(host(o), o_ref, shape.H, shape.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE


def shape_args(s):
    return s.T, s.N, s.H, s.d


def test_window_attn_strided(vdn):
    shape = synth.Shape(11, 90, 2, 64)
    inp = synth.make_inputs(shape, seed=4, device="cuda")
    pad = {}
    for n in ("q", "k", "v"):
        big = torch.full((shape.L, shape.D + 16), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
        big[:, :shape.D] = inp[n]
        pad[n] = big[:, :shape.D]
    out = torch.full((shape.L, shape.D + 8), float("nan"), dtype=torch.bfloat16, device="cuda")
    o, ws = vdn.window_attn(pad["q"], pad["k"], pad["v"], *shape_args(shape), out=out[:, :shape.D])
    assert vdn.get_device_status(ws) == 0
    assert torch.isnan(out[:, shape.D:].float()).all()
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, _ = oracle.window_attn(x["q"], x["k"], x["v"], *shape_args(shape))
    assert per_head_max_rel(host(out[:, :shape.D]), o_ref, shape.H, shape.d) <= TOL_BF16


def _sample_rows(T, N, rng, n_random=24):
    rows = [0, N - 1, N, 5 * N - 1, 5 * N, 7 * N + N // 2, (T - 2) * N, (T - 1) * N - 1,
            (T - 1) * N, T * N - 1, (T // 2) * N + 255, (T // 2) * N + 256]
    rows += list(rng.integers(0, T * N, n_random))
    return np.array(sorted(set(r for r in rows if 0 <= r < T * N)))


@pytest.mark.parametrize("T", [42, 102])
def test_window_attn_full_layer_sampled(vdn, T):
    shape = synth.Shape(T, 4032, 24, 128)
    inp = synth.make_inputs(shape, seed=0, device="cuda")
    o, lse = _run(vdn, shape, inp)
    rows = _sample_rows(T, shape.N, np.random.default_rng(T))
    ridx = torch.as_tensor(rows, device="cuda")
    o_s = host(o[ridx])
    lse_s = host(lse[:, ridx])
    for h in (0, 13, 23):
        c = slice(h * 128, (h + 1) * 128)
        q = host(inp["q"][:, c])
        k = host(inp["k"][:, c])
        v = host(inp["v"][:, c])
        o_ref, lse_ref = oracle.window_attn_rows(q, k, v, T, shape.N, 1, 128, rows)
        assert max_rel(o_s[:, c], o_ref) <= TOL_BF16, h
        assert np.abs(lse_s[h] - lse_ref[0]).max() <= TOL_LSE, h
    del inp, o, lse
    torch.cuda.empty_cache()


def test_fma_pipe_exp2_error_bound(vdn):
    """The FMA-pipe exponential stays within 1e-4 relative of exact 2^x and of
    the MUFU ex2.approx over the range the Softmax feeds it (x <= 8), and
    clamps far-negative inputs to a tiny non-negative value."""
    xs = np.concatenate([np.linspace(-124.0, 8.0, 400001), np.arange(-40, 9, 0.5),
                         [0.0, -0.5, 0.5, -1e-7, 7.999]]).astype(np.float32)
    x = torch.as_tensor(xs, device="cuda")
    y_fma, y_mufu = vdn.selftest_exp2(x)
    torch.cuda.synchronize()
    ref = np.exp2(xs.astype(np.float64))
    yf, ym = host(y_fma).astype(np.float64), host(y_mufu).astype(np.float64)
    assert np.max(np.abs(yf / ref - 1.0)) <= 1e-4
    assert np.max(np.abs(yf / ym - 1.0)) <= 1e-4
    far = torch.tensor([-200.0, -1000.0, -float("inf")], device="cuda")
    yfar, _ = vdn.selftest_exp2(far)
    v = host(yfar)
    assert np.all(v >= 0) and np.all(v < 1e-37)


def _ctx(M, D, seed):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    ck = torch.randn((M, D), generator=g, device="cuda").to(torch.bfloat16)
    cv = torch.randn((M, D), generator=g, device="cuda").to(torch.bfloat16)
    return ck, cv


@pytest.mark.parametrize("T,N,H,d,M", [(10, 64, 2, 128, 1), (17, 100, 2, 128, 77),
                                       (12, 96, 1, 64, 300), (6, 40, 3, 128, 512)])
def test_window_attn_context_keys_small(vdn, T, N, H, d, M):
    """Text/audio context keys: every video query also attends to them."""
    shape = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(shape, seed=T + M, device="cuda")
    ck, cv = _ctx(M, shape.D, seed=M)
    o, lse = _run(vdn, shape, inp, ctx_k=ck, ctx_v=cv)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], T, N, H, d,
                                        ctx_k=host(ck), ctx_v=host(cv))
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE


def test_window_attn_context_keys_full_layer_sampled(vdn):
    """102 latent frames x 4032 tokens x 24 heads plus 512 text keys."""
    T, M = 102, 512
    shape = synth.Shape(T, 4032, 24, 128)
    inp = synth.make_inputs(shape, seed=3, device="cuda")
    ck, cv = _ctx(M, shape.D, seed=5)
    o, lse = _run(vdn, shape, inp, ctx_k=ck, ctx_v=cv)
    rows = _sample_rows(T, shape.N, np.random.default_rng(7), n_random=12)
    ridx = torch.as_tensor(rows, device="cuda")
    o_s, lse_s = host(o[ridx]), host(lse[:, ridx])
    for h in (2, 17):
        c = slice(h * 128, (h + 1) * 128)
        o_ref, lse_ref = oracle.window_attn_rows(
            host(inp["q"][:, c]), host(inp["k"][:, c]), host(inp["v"][:, c]), T, shape.N, 1, 128,
            rows, ctx_k=host(ck[:, c]), ctx_v=host(cv[:, c]))
        assert max_rel(o_s[:, c], o_ref) <= TOL_BF16, h
        assert np.abs(lse_s[h] - lse_ref[0]).max() <= TOL_LSE, h
    del inp, o, lse
    torch.cuda.empty_cache()


def test_window_attn_rescale_in_one_row_of_a_warp(vdn):
    """A context key aligned with one query row makes only that row's running
    max jump by far more than 2^8 at the last key tiles; the O rescale must
    stay correct for it and for its warp neighbours."""
    shape = synth.Shape(6, 64, 1, 128)
    inp = synth.make_inputs(shape, seed=11, device="cuda")
    ck, cv = _ctx(130, shape.D, seed=12)
    ck = (ck.float() * 0.05).to(torch.bfloat16)
    ck[0] = inp["q"][3]           # row 3 scores |q_3|^2 ~ 128 against this key
    ck[129] = inp["q"][40] * 2    # another row, in the ragged last context tile
    o, lse = _run(vdn, shape, inp, ctx_k=ck, ctx_v=cv)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], *shape_args(shape),
                                        ctx_k=host(ck), ctx_v=host(cv))
    assert per_head_max_rel(host(o), o_ref, shape.H, shape.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE


def test_window_attn_rescale_on_second_half_keys(vdn):
    """Keys 64..127 of a later tile carry a jump of the running max far above
    2^8 (one row at a time, in a full and in a ragged context tile): the
    rescale is decided only after the whole row of the tile is read."""
    shape = synth.Shape(6, 64, 1, 128)
    inp = synth.make_inputs(shape, seed=13, device="cuda")
    ck, cv = _ctx(250, shape.D, seed=14)
    ck = (ck.float() * 0.05).to(torch.bfloat16)
    ck[100] = inp["q"][5]          # column 100 of the first context tile
    ck[200] = inp["q"][50] * 2     # column 72 of the second (ragged, 122 keys)
    ck[250 - 1] = inp["q"][7] * 3  # the last key of the ragged tile
    o, lse = _run(vdn, shape, inp, ctx_k=ck, ctx_v=cv)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], *shape_args(shape),
                                        ctx_k=host(ck), ctx_v=host(cv))
    assert per_head_max_rel(host(o), o_ref, shape.H, shape.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE
