"""Parity of vdn_window_attn_mxfp8 (CUDA, through the C ABI) against the
MXFP8 window Softmax of the CPU oracle (operands quantized exactly as the
kernel's format defines them; the oracle is pinned in
test_oracle_mxfp8_pins.py).

Small shapes: every output row and the log-sum-exp, over mask variants and
key tiles that end inside and at the ends of frames.  Full-size layers (42
and 102 latent frames x 4032 tokens x 24 heads): sampled rows of anchor
frames, chunk edges and the last chunk, for several heads.  Tolerance: the
bf16 output's (2e-2, max-relative per head); the GPU forms P with the MUFU
exponential in fp32 and accumulates in fp32, so its only departures from the
oracle are the output's bf16 rounding and the rare element whose E4M3 code
or block scale sits on a rounding boundary.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import mxfp8 as omx
from tests.parity_util import TOL_BF16, ensure_built, host, per_head_max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu

TOL_LSE = 1e-3


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _run(vdn, s, inp, **kw):
    lse = torch.empty((s.H, s.L), dtype=torch.float32, device="cuda")
    o, ws = vdn.window_attn_mxfp8(inp["q"], inp["k"], inp["v"], s.T, s.N, s.H, s.d, lse=lse,
                                  **kw)
    assert vdn.get_device_status(ws) == 0
    return o, lse


SMALL = [
    (10, 64, 2),     # 2 chunks: every frame visible
    (17, 96, 2),     # one 96-key tile per frame
    (12, 256, 2),    # tiles straddle frames (256 = 2 x 96 + 64)
    (23, 160, 1),
    (7, 32, 1),      # one 32-token block per frame
]


@pytest.mark.parametrize("T,N,H", SMALL)
def test_window_mxfp8_parity_small(vdn, T, N, H, report_metric):
    s = synth.Shape(T, N, H, 128)
    inp = synth.make_inputs(s, seed=T * 100 + N + 7, device="cuda")
    o, lse = _run(vdn, s, inp)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = omx.window_attn_mxfp8(x["q"], x["k"], x["v"], T, N, H, 128)
    err = per_head_max_rel(host(o), o_ref, H, 128)
    report_metric("o_mx_max_rel", err)
    assert err <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE
    # what the format costs against the exact float64 Softmax (reported)
    o_exact, _ = oracle.window_attn(x["q"], x["k"], x["v"], T, N, H, 128)
    report_metric("o_mx_vs_exact_max_rel", per_head_max_rel(host(o), o_exact, H, 128))


@pytest.mark.parametrize("cf,wc,anchors,scale", [
    (5, 1, 0, 0.0), (5, 0, 3, 0.0), (3, 2, 1, 0.0), (5, 1, 3, 0.3),
])
def test_window_mxfp8_mask_variants(vdn, cf, wc, anchors, scale):
    s = synth.Shape(26, 64, 2, 128)
    inp = synth.make_inputs(s, seed=cf * 10 + wc + anchors, device="cuda")
    o, lse = _run(vdn, s, inp, chunk_frames=cf, window_chunks=wc, anchors=anchors, scale=scale)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, lse_ref = omx.window_attn_mxfp8(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d,
                                           chunk_frames=cf, window_chunks=wc, anchors=anchors,
                                           scale=scale)
    assert per_head_max_rel(host(o), o_ref, s.H, s.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE


def test_window_mxfp8_rescale_on_a_large_score_jump(vdn):
    """Queries whose scores jump by far more than 2^8 (log2 units) at a later
    key tile: the integer running maximum moves and O is rescaled by an exact
    power of two; the result still equals the oracle, which takes the row's
    global maximum."""
    s = synth.Shape(12, 64, 1, 128)
    inp = synth.make_inputs(s, seed=5, device="cuda")
    k = inp["k"].clone()
    k[10 * s.N: 11 * s.N] *= 40.0      # frame 10: much larger scores for every query
    inp["k"] = k
    o, lse = _run(vdn, s, inp)
    x = {kk: host(v) for kk, v in inp.items() if kk in ("q", "k", "v")}
    o_ref, lse_ref = omx.window_attn_mxfp8(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    assert per_head_max_rel(host(o), o_ref, s.H, s.d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= TOL_LSE * max(1.0, np.abs(lse_ref).max())


@pytest.mark.parametrize("T", [42, 102])
def test_window_mxfp8_full_layer_sampled_rows(vdn, T):
    s = synth.Shape(T, 4032, 24, 128)
    inp = synth.make_inputs(s, seed=0, device="cuda")
    o, lse = _run(vdn, s, inp)
    rng = np.random.default_rng(T)
    N = s.N
    frames = [0, 1, 4, 5, T // 2, T - 3, T - 2, T - 1]
    rows = sorted(set([f * N for f in frames] + [f * N + N - 1 for f in frames] +
                      list(rng.integers(0, s.L, 16))))
    rows_t = torch.as_tensor(rows, device="cuda")
    heads = [0, 11, 23]
    cols = np.concatenate([np.arange(h * 128, (h + 1) * 128) for h in heads])
    cols_t = torch.as_tensor(cols, device="cuda")
    q = host(inp["q"][:, cols_t])
    k = host(inp["k"][:, cols_t])
    v = host(inp["v"][:, cols_t])
    del inp
    o_ref, lse_ref = omx.window_attn_mxfp8_rows(q, k, v, T, N, len(heads), 128, rows)
    o_gpu = host(o[rows_t][:, cols_t])
    assert per_head_max_rel(o_gpu, o_ref, len(heads), 128) <= TOL_BF16
    lse_gpu = host(lse[torch.as_tensor(heads, device="cuda")][:, rows_t])
    assert np.abs(lse_gpu - lse_ref).max() <= TOL_LSE
    del o, lse
    torch.cuda.empty_cache()


def test_window_mxfp8_refuses_unsupported_shapes(vdn):
    for T, N, d in ((4, 40, 128), (4, 64, 64)):
        s = synth.Shape(T, N, 1, d)
        t = torch.zeros((s.L, s.D), dtype=torch.bfloat16, device="cuda")
        with pytest.raises(vdn.VdnError) as e:
            vdn.window_attn_mxfp8(t, t, t, T, N, 1, d, ws=vdn.alloc_workspace(1 << 20))
        assert e.value.code == 2        # VDN_ERR_UNSUPPORTED


def test_hybrid_layer_all_mxfp8(vdn):
    """HybridLayer(softmax="mxfp8", projections="mxfp8"): the Softmax branch
    against the oracle's MXFP8 window Softmax, y against the oracle's MXFP8
    fuse on the layer's own branch outputs, and the host-copy path
    (forward_many) giving the same y."""
    s = synth.Shape(12, 96, 2, 128)
    inp = synth.make_inputs(s, seed=8, device="cuda", with_fuse=True)
    layer = vdn.HybridLayer(s.T, s.N, s.H, s.d, inp["W_gs"], inp["W_gl"], inp["W_os"],
                            inp["W_ol"], inp["gamma"], projections="mxfp8", softmax="mxfp8")
    acts = [inp[k] for k in ("q", "k", "v", "beta", "alpha", "x")]
    y = layer.forward(*acts).clone()
    assert layer.status() == 0
    x = {k: host(inp[k]) for k in ("q", "k", "v")}
    o_ref, _ = omx.window_attn_mxfp8(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    assert per_head_max_rel(host(layer.o_s), o_ref, s.H, s.d) <= TOL_BF16
    y_ref = omx.hybrid_fuse_mxfp8(host(inp["x"]), host(layer.o_s), host(layer.o_vda),
                                  host(inp["W_gs"]), host(inp["W_gl"]), host(inp["gamma"]), 1e-6,
                                  host(inp["W_os"]), host(inp["W_ol"]), s.H)
    assert np.abs(host(y) - y_ref).max() / np.abs(y_ref).max() <= TOL_BF16
    hosts = [[t.cpu().pin_memory() for t in acts]]
    outs = [torch.empty((s.L, s.D), dtype=torch.bfloat16).pin_memory()]
    layer.forward_many(hosts, outs)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], y.cpu())


def test_window_mxfp8_strided_rows_and_output(vdn):
    """Row strides larger than H*d on the inputs and on the output: the
    quantizers read through ld, the kernel writes through ld_o and leaves the
    padding columns untouched."""
    s = synth.Shape(13, 64, 2, 128)
    inp = synth.make_inputs(s, seed=77, device="cuda")
    pad = 64
    big = {}
    for n in ("q", "k", "v"):
        t = torch.full((s.L, s.D + pad), float("nan"), dtype=torch.bfloat16, device="cuda")
        t[:, :s.D] = inp[n]
        big[n] = t[:, :s.D]
    out = torch.full((s.L, s.D + pad), 3.0, dtype=torch.bfloat16, device="cuda")
    o, ws = vdn.window_attn_mxfp8(big["q"], big["k"], big["v"], s.T, s.N, s.H, s.d,
                                  out=out[:, :s.D])
    assert vdn.get_device_status(ws) == 0
    assert torch.all(out[:, s.D:] == 3.0)
    x = {k: host(v) for k, v in inp.items() if k in ("q", "k", "v")}
    o_ref, _ = omx.window_attn_mxfp8(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
    assert per_head_max_rel(host(out[:, :s.D]), o_ref, s.H, s.d) <= TOL_BF16


def test_window_mxfp8_72_frames_sampled_rows(vdn):
    """The sweep's middle length (72 frames x 1024 tokens, 32-aligned) on
    sampled rows of two heads."""
    s = synth.Shape(72, 1024, 4, 128)
    inp = synth.make_inputs(s, seed=72, device="cuda")
    o, lse = _run(vdn, s, inp)
    N, T = s.N, s.T
    rng = np.random.default_rng(72)
    rows = sorted(set([0, N - 1, 5 * N, 5 * N - 1, (T - 1) * N, T * N - 1, (T // 2) * N + 3] +
                      list(rng.integers(0, s.L, 12))))
    heads = [1, 3]
    cols = np.concatenate([np.arange(h * 128, (h + 1) * 128) for h in heads])
    cols_t = torch.as_tensor(cols, device="cuda")
    rows_t = torch.as_tensor(rows, device="cuda")
    x = {k: host(inp[k][:, cols_t]) for k in ("q", "k", "v")}
    o_ref, lse_ref = omx.window_attn_mxfp8_rows(x["q"], x["k"], x["v"], T, N, 2, 128, rows)
    assert per_head_max_rel(host(o[rows_t][:, cols_t]), o_ref, 2, 128) <= TOL_BF16
    lse_gpu = host(lse[torch.as_tensor(heads, device="cuda")][:, rows_t])
    assert np.abs(lse_gpu - lse_ref).max() <= TOL_LSE
