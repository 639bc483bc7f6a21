"""The tiny oracle configuration on the GPU: 1 head x 16, hidden 16, 10 (two
full chunks) and 17 (ragged chunk) latent frames of 4x4 tokens, plus a
2-head x 32 case.  Small heads run on zero-padded 64-wide copies inside the
library; every entry point and the chained layer are compared with the
oracle."""

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


CASES = [(10, 16, 1, 16), (17, 16, 1, 16), (12, 24, 2, 32)]


@pytest.mark.parametrize("T,N,H,d", CASES)
def test_tiny_vda(vdn, T, N, H, d):
    s = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(s, seed=0, device="cuda")
    states = torch.empty((2, T, H, d, d), device="cuda")
    o, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H, d,
                         states=states)
    assert vdn.get_device_status(ws) == 0
    x = {k: host(v) for k, v in inp.items()}
    o_ref, S_fwd, S_bwd = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], T, N, H, d)
    st = host(states)
    for t in range(T):
        for h in range(H):
            assert max_rel(st[0, t, h], S_fwd[t, h]) <= TOL_STATE
            assert max_rel(st[1, t, h], S_bwd[t, h]) <= TOL_STATE
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16


@pytest.mark.parametrize("T,N,H,d", CASES)
def test_tiny_window_attn(vdn, T, N, H, d):
    s = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(s, seed=1, device="cuda")
    lse = torch.empty((H, s.L), device="cuda")
    o, ws = vdn.window_attn(inp["q"], inp["k"], inp["v"], T, N, H, d, lse=lse)
    assert vdn.get_device_status(ws) == 0
    x = {k: host(v) for k, v in inp.items()}
    o_ref, lse_ref = oracle.window_attn(x["q"], x["k"], x["v"], T, N, H, d)
    assert per_head_max_rel(host(o), o_ref, H, d) <= TOL_BF16
    assert np.abs(host(lse) - lse_ref).max() <= 1e-3


@pytest.mark.parametrize("T,N,H,d", CASES)
def test_tiny_layer(vdn, T, N, H, d):
    """The whole hybrid layer (both branches and the fuse) at hidden H*d."""
    s = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(s, seed=2, device="cuda", with_fuse=True)
    layer = vdn.HybridLayer(T, N, H, d, inp["W_gs"], inp["W_gl"], inp["W_os"], inp["W_ol"],
                            inp["gamma"])
    y = layer.forward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], inp["x"])
    assert layer.status() == 0
    x = {k: host(v) for k, v in inp.items()}
    o_s, _ = oracle.window_attn(x["q"], x["k"], x["v"], T, N, H, d)
    o_l, _, _ = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], T, N, H, d)
    y_ref = oracle.hybrid_fuse(x["x"], o_s, o_l, x["W_gs"], x["W_gl"], x["gamma"], 1e-6,
                               x["W_os"], x["W_ol"], H)
    assert max_rel(host(y), y_ref) <= TOL_BF16
    # the fuse alone, on the layer's own branch outputs
    y2, ws = vdn.hybrid_fuse(inp["x"], layer.o_s, layer.o_vda, inp["W_gs"], inp["W_gl"],
                             inp["gamma"], inp["W_os"], inp["W_ol"], H)
    assert vdn.get_device_status(ws) == 0
    y2_ref = oracle.hybrid_fuse(x["x"], host(layer.o_s), host(layer.o_vda), x["W_gs"], x["W_gl"],
                                x["gamma"], 1e-6, x["W_os"], x["W_ol"], H)
    assert max_rel(host(y2), y2_ref) <= TOL_BF16


@pytest.mark.parametrize("T,N,H,d,nvid", [
    (12, 96, 2, 128, 3),   # two head groups, three videos
    (7, 100, 3, 128, 1),   # one video: head-group fill and row-block drain on it; ragged rows
    (5, 64, 5, 128, 2),    # H = 5: a single head group
    (9, 128, 4, 128, 2),   # four head groups
    (7, 100, 4, 64, 2),    # head dim 64
])
def test_forward_many_pipelined_host_path(vdn, T, N, H, d, nvid):
    """HybridLayer.forward_many (pinned host in/out, copies overlapping the
    compute; the first video's inputs arriving by head groups, the last
    video's fuse and read-back in row blocks) gives y bit-identical to
    forward() on device tensors."""
    s = synth.Shape(T, N, H, d)
    vids = [synth.make_inputs(s, seed=20 + i, device="cuda", with_fuse=True)
            for i in range(nvid)]
    w = vids[0]
    layer = vdn.HybridLayer(s.T, s.N, s.H, s.d, w["W_gs"], w["W_gl"], w["W_os"], w["W_ol"],
                            w["gamma"])
    names = ("q", "k", "v", "beta", "alpha", "x")
    refs = []
    for v in vids:
        refs.append(layer.forward(*[v[n] for n in names]).clone())
    batches = [[v[n].to("cpu").pin_memory() for n in names] for v in vids]
    outs = [torch.empty((s.L, s.D), dtype=torch.bfloat16).pin_memory() for _ in vids]
    layer.forward_many(batches, outs)
    torch.cuda.synchronize()
    assert layer.status() == 0
    for o, r in zip(outs, refs):
        assert torch.equal(o, r.cpu())


def test_forward_many_after_the_grouping_changes(vdn):
    """Changing the fill and drain granularity between forward_many calls
    (the per-group beta/alpha buffers are rebuilt for the new grouping)
    keeps y bit-identical to forward()."""
    s = synth.Shape(7, 100, 4, 128)
    v = synth.make_inputs(s, seed=31, device="cuda", with_fuse=True)
    layer = vdn.HybridLayer(s.T, s.N, s.H, s.d, v["W_gs"], v["W_gl"], v["W_os"], v["W_ol"],
                            v["gamma"])
    names = ("q", "k", "v", "beta", "alpha", "x")
    ref = layer.forward(*[v[n] for n in names]).clone().cpu()
    batch = [[v[n].to("cpu").pin_memory() for n in names]]
    for fg, db in ((4, 4), (2, 3), (1, 1), (4, 8)):
        layer.FILL_GROUPS, layer.DRAIN_BLOCKS = fg, db
        out = [torch.empty((s.L, s.D), dtype=torch.bfloat16).pin_memory()]
        layer.forward_many(batch, out)
        torch.cuda.synchronize()
        assert layer.status() == 0
        assert torch.equal(out[0], ref), (fg, db)
