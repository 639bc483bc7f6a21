"""Parity of vdn_hybrid_fuse (CUDA, through the C ABI) against the CPU oracle:
gates, per-head RMSNorm and the two summed output projections."""

import numpy as np
import pytest
import torch

import oracle
from tests.parity_util import TOL_BF16, elementwise_rel, TOL_ELEMENTWISE, ensure_built, host, max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _inputs(T, N, H, d, seed):
    shape = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(shape, seed=seed, device="cuda", with_fuse=True)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    # branch outputs with a per-head scale spread, as the RMSNorm sees them
    inp["o_s"] = torch.randn((shape.L, shape.D), generator=g, device="cuda").to(torch.bfloat16)
    scale = torch.linspace(0.1, 3.0, shape.D, device="cuda")
    inp["o_vda"] = (torch.randn((shape.L, shape.D), generator=g, device="cuda") * scale).to(
        torch.bfloat16)
    inp["gamma"] = (1.0 + 0.1 * torch.randn(shape.D, generator=g, device="cuda")).contiguous()
    return shape, inp


def _fuse(vdn, shape, inp, eps=1e-6):
    y, ws = vdn.hybrid_fuse(inp["x"], inp["o_s"], inp["o_vda"], inp["W_gs"], inp["W_gl"],
                            inp["gamma"], inp["W_os"], inp["W_ol"], shape.H, eps=eps)
    assert vdn.get_device_status(ws) == 0
    return y


def _ref_rows(shape, inp, rows, eps=1e-6):
    r = torch.as_tensor(rows, device="cuda")
    return oracle.hybrid_fuse_rows(host(inp["x"][r]), host(inp["o_s"][r]), host(inp["o_vda"][r]),
                                   host(inp["W_gs"]), host(inp["W_gl"]), host(inp["gamma"]), eps,
                                   host(inp["W_os"]), host(inp["W_ol"]), shape.H,
                                   np.arange(len(rows)))


@pytest.mark.parametrize("T,N,H,d", [(3, 100, 2, 128), (5, 200, 8, 64), (2, 640, 4, 128),
                                     (1, 7, 4, 64)])
def test_fuse_parity_small(vdn, T, N, H, d, report_metric):
    shape, inp = _inputs(T, N, H, d, seed=T + N)
    y = _fuse(vdn, shape, inp)
    ref = _ref_rows(shape, inp, np.arange(shape.L))
    assert max_rel(host(y), ref) <= TOL_BF16
    err_el = elementwise_rel(host(y), ref)
    report_metric("y_elementwise_rel", err_el)
    assert err_el <= TOL_ELEMENTWISE


def test_fuse_zero_gate_weights(vdn):
    """W_gs = W_gl = 0 gives both gates 0.5."""
    shape, inp = _inputs(2, 256, 2, 128, seed=3)
    inp["W_gs"].zero_()
    inp["W_gl"].zero_()
    y = _fuse(vdn, shape, inp)
    n = oracle.rmsnorm_heads(host(inp["o_vda"]), shape.H, shape.d, host(inp["gamma"]), 1e-6)
    ref = 0.5 * host(inp["o_s"]).astype(np.float64) @ host(inp["W_os"]).T.astype(np.float64) + \
        0.5 * n @ host(inp["W_ol"]).T.astype(np.float64)
    assert max_rel(host(y), ref) <= TOL_BF16


def test_fuse_full_block_sampled(vdn):
    """The full hybrid block's fuse at 102 x 4032 tokens, hidden 3072 (sampled rows)."""
    shape, inp = _inputs(102, 4032, 24, 128, seed=0)
    y = _fuse(vdn, shape, inp)
    rng = np.random.default_rng(0)
    rows = np.array(sorted(set([0, 127, 128, shape.L - 1, shape.L - 128] +
                               list(rng.integers(0, shape.L, 40)))))
    ref = _ref_rows(shape, inp, rows)
    got = host(y[torch.as_tensor(rows, device="cuda")])
    assert max_rel(got, ref) <= TOL_BF16
    del inp, y
    torch.cuda.empty_cache()


@pytest.mark.parametrize("G", [2, 4, 8])
def test_fuse_head_shards_sum_to_full(vdn, G):
    """Row-parallel fuse: the fp32 partials of G head shards, summed (the
    all-reduce of a head-parallel run, done here on one GPU), give y."""
    shape, inp = _inputs(2, 1000, 8, 128, seed=40 + G)
    y_full = _fuse(vdn, shape, inp)
    Hl = shape.H // G
    acc = torch.zeros((shape.L, shape.D), dtype=torch.float32, device="cuda")
    for r in range(G):
        c = slice(r * Hl * 128, (r + 1) * Hl * 128)
        part, ws = vdn.hybrid_fuse_shard(inp["x"], inp["o_s"][:, c].contiguous(),
                                         inp["o_vda"][:, c].contiguous(), inp["W_gs"],
                                         inp["W_gl"], inp["gamma"], inp["W_os"], inp["W_ol"],
                                         128, r * Hl)
        assert vdn.get_device_status(ws) == 0
        acc += part
    ref = _ref_rows(shape, inp, np.arange(shape.L))
    assert max_rel(host(acc), ref) <= TOL_BF16
    assert max_rel(host(acc), host(y_full)) <= TOL_BF16


@pytest.mark.parametrize("G", [2, 4, 8])
def test_fuse_shards_reduce_scatter_into_owners(vdn, G):
    """The output GEMM fused with the reduce-scatter: G shards (each a
    separate launch, as G ranks would run them) add their partials into G
    owner buffers; the owners' row blocks, stacked, equal the full fuse.
    No launch waits on another, so they may share one GPU."""
    shape, inp = _inputs(2, 1000, 8, 128, seed=50 + G)
    y_full = _fuse(vdn, shape, inp)
    Hl = shape.H // G
    R = -(-shape.L // G)
    owners = [torch.zeros((min(R, shape.L - o * R), shape.D), dtype=torch.float32, device="cuda")
              for o in range(G)]
    for r in range(G):
        c = slice(r * Hl * 128, (r + 1) * Hl * 128)
        ws = vdn.hybrid_fuse_shard_rs(inp["x"], inp["o_s"][:, c].contiguous(),
                                      inp["o_vda"][:, c].contiguous(), inp["W_gs"], inp["W_gl"],
                                      inp["gamma"], inp["W_os"], inp["W_ol"], 128, r * Hl,
                                      owners)
        assert vdn.get_device_status(ws) == 0
    y = torch.cat(owners, dim=0)
    ref = _ref_rows(shape, inp, np.arange(shape.L))
    assert max_rel(host(y), ref) <= TOL_BF16
    assert max_rel(host(y), host(y_full)) <= TOL_BF16

