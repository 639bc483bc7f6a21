"""Parity of the MXFP8 projections (CUDA, through the C ABI) against the
MXFP8 oracle: the quantizer's codes and scale bytes bit for bit; the
block-scaled GEMM (fp32 output) against the float64 product of the same
dequantized operands; the fuse with MXFP8 projections against the oracle's
MXFP8 fuse.

Tolerances: the GEMM accumulates in fp32 over K <= 6144 terms, 1e-5 of the
output's max.  The fuse writes bf16 (2e-2, the bf16 output tolerance); its
gated inputs Z are formed in fp32 on the GPU and in float64 by the oracle
before both quantize them, so an element next to a rounding boundary may
take the neighbouring E4M3 code on one side, which moves an output by far
less than the bf16 bound.
"""

import numpy as np
import pytest
import torch

import oracle
from oracle import mxfp8 as omx
from tests.parity_util import TOL_BF16, ensure_built, host, max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _wide_range(R, K, seed):
    """bf16 rows whose magnitudes span many binades, with zero blocks and
    tiny values."""
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    x = torch.randn((R, K), generator=g, device="cuda")
    x *= torch.exp2(torch.randint(-30, 30, (R, 1), generator=g, device="cuda").float())
    x[::7, 32:64] = 0.0
    x[min(3, R - 1), :] *= 1e-30
    return x.to(torch.bfloat16)


@pytest.mark.parametrize("R,K", [(300, 512), (128, 128), (1, 256), (777, 1024)])
def test_quantize_bit_exact(vdn, R, K):
    x = _wide_range(R, K, seed=R + K)
    q, sf = vdn.mxfp8_quantize(x)
    codes, scales = omx.mx_quantize(host(x).astype(np.float64))
    np.testing.assert_array_equal(q.cpu().numpy(), codes)
    np.testing.assert_array_equal(sf.cpu().numpy()[:vdn.mxfp8_scale_bytes(R, K)],
                                  omx.sf_tiled(scales))


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (300, 256, 512), (1000, 384, 1024),
                                   (77, 96, 256)])
def test_gemm_fp32_against_dequantized_product(vdn, M, N, K):
    a = _wide_range(M, K, seed=M) if M != 1000 else \
        torch.randn((M, K), device="cuda").to(torch.bfloat16)
    b = torch.randn((N, K), device="cuda").to(torch.bfloat16)
    aq, bq = vdn.mxfp8_quantize(a), vdn.mxfp8_quantize(b)
    c, ws = vdn.gemm_mxfp8(aq, bq, out_f32=True)
    assert vdn.get_device_status(ws) == 0
    ref = omx.gemm_mx(*omx.mx_quantize(host(a).astype(np.float64)),
                      *omx.mx_quantize(host(b).astype(np.float64)))
    for i in range(M):  # per row: rows differ by up to 2^60 in scale
        assert max_rel(host(c[i]), ref[i]) <= 1e-5, i


def test_gemm_bf16_output(vdn):
    a = torch.randn((256, 512), device="cuda").to(torch.bfloat16)
    b = torch.randn((128, 512), device="cuda").to(torch.bfloat16)
    c, _ = vdn.gemm_mxfp8(vdn.mxfp8_quantize(a), vdn.mxfp8_quantize(b))
    ref = omx.gemm_mx(*omx.mx_quantize(host(a).astype(np.float64)),
                      *omx.mx_quantize(host(b).astype(np.float64)))
    assert max_rel(host(c), ref) <= TOL_BF16


def _fuse_inputs(T, N, H, d, seed):
    shape = synth.Shape(T, N, H, d)
    inp = synth.make_inputs(shape, seed=seed, device="cuda", with_fuse=True)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed + 1)
    inp["o_s"] = torch.randn((shape.L, shape.D), generator=g, device="cuda").to(torch.bfloat16)
    inp["o_vda"] = (torch.randn((shape.L, shape.D), generator=g, device="cuda") *
                    torch.linspace(0.1, 3.0, shape.D, device="cuda")).to(torch.bfloat16)
    inp["gamma"] = (1.0 + 0.1 * torch.randn(shape.D, generator=g, device="cuda")).contiguous()
    return shape, inp


def _oracle_rows(inp, rows, H):
    r = torch.as_tensor(rows, device="cuda")
    return omx.hybrid_fuse_mxfp8(host(inp["x"][r]), host(inp["o_s"][r]), host(inp["o_vda"][r]),
                                 host(inp["W_gs"]), host(inp["W_gl"]), host(inp["gamma"]), 1e-6,
                                 host(inp["W_os"]), host(inp["W_ol"]), H)


@pytest.mark.parametrize("T,N,H,d", [(2, 100, 2, 128), (3, 70, 4, 64), (1, 300, 8, 32)])
def test_fuse_mxfp8_small(vdn, T, N, H, d):
    shape, inp = _fuse_inputs(T, N, H, d, seed=T * N)
    wg, wo = vdn.mxfp8_fuse_weights(inp["W_gs"], inp["W_gl"], inp["W_os"], inp["W_ol"])
    y, ws = vdn.hybrid_fuse_mxfp8(inp["x"], inp["o_s"], inp["o_vda"], wg, inp["gamma"], wo, H)
    assert vdn.get_device_status(ws) == 0
    ref = _oracle_rows(inp, np.arange(shape.L), H)
    assert max_rel(host(y), ref) <= TOL_BF16
    # what the format costs against the unquantized fuse (reported bound,
    # a property of MXFP8 rather than of the kernels)
    exact = oracle.hybrid_fuse_rows(host(inp["x"]), host(inp["o_s"]), host(inp["o_vda"]),
                                    host(inp["W_gs"]), host(inp["W_gl"]), host(inp["gamma"]), 1e-6,
                                    host(inp["W_os"]), host(inp["W_ol"]), H, np.arange(shape.L))
    assert max_rel(ref, exact) <= 0.10


def test_fuse_mxfp8_full_block_sampled(vdn):
    """102 x 4032 tokens, hidden 3072 (24 heads of 128): sampled rows."""
    shape, inp = _fuse_inputs(102, 4032, 24, 128, seed=0)
    wg, wo = vdn.mxfp8_fuse_weights(inp["W_gs"], inp["W_gl"], inp["W_os"], inp["W_ol"])
    y, ws = vdn.hybrid_fuse_mxfp8(inp["x"], inp["o_s"], inp["o_vda"], wg, inp["gamma"], wo, 24)
    assert vdn.get_device_status(ws) == 0
    rng = np.random.default_rng(0)
    rows = np.array(sorted(set([0, 127, 128, shape.L - 1] + list(rng.integers(0, shape.L, 24)))))
    ref = _oracle_rows(inp, rows, 24)
    assert max_rel(host(y[torch.as_tensor(rows, device="cuda")]), ref) <= TOL_BF16
    del inp, y, ws
    torch.cuda.empty_cache()


def test_hybrid_layer_with_mxfp8_projections(vdn):
    """HybridLayer(projections="mxfp8"): y against the oracle's MXFP8 fuse
    on the layer's own branch outputs, and the host-copy path (forward_many)
    giving the same y."""
    shape = synth.Shape(12, 96, 2, 128)
    inp = synth.make_inputs(shape, seed=4, device="cuda", with_fuse=True)
    layer = vdn.HybridLayer(shape.T, shape.N, shape.H, shape.d, inp["W_gs"], inp["W_gl"],
                            inp["W_os"], inp["W_ol"], inp["gamma"], projections="mxfp8")
    acts = [inp[k] for k in ("q", "k", "v", "beta", "alpha", "x")]
    y = layer.forward(*acts).clone()
    assert layer.status() == 0
    ref = omx.hybrid_fuse_mxfp8(host(inp["x"]), host(layer.o_s), host(layer.o_vda),
                                host(inp["W_gs"]), host(inp["W_gl"]), host(inp["gamma"]), 1e-6,
                                host(inp["W_os"]), host(inp["W_ol"]), shape.H)
    assert max_rel(host(y), ref) <= TOL_BF16
    hosts = [[t.cpu().pin_memory() for t in acts]]
    outs = [torch.empty((shape.L, shape.D), dtype=torch.bfloat16).pin_memory()]
    layer.forward_many(hosts, outs)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], y.cpu())
