"""Seeded synthetic inputs for the hybrid attention layer.

This module draws random tensors and nothing else: it holds none of the
layer's arithmetic, so both the CUDA library's tests and the CPU oracle's
tests can take their inputs from it.

Value laws (the workload described for 42-102 latent frames of 1344x768
video, 16x spatial compression -> 48x84 = 4032 tokens per frame):

* q, k, v ~ N(0, 1); every key is L2-normalised per token and per head;
* beta = sigmoid(N(0, 1)), one write strength per token and head, [L, H];
* alpha ~ U(0.9, 1.0), one decay per frame and head, [T, H];
* x ~ N(0, 1) (block input for the gates);
* W_gs, W_gl, W_os, W_ol ~ N(0, 0.02^2), [D, D], y = z W^T convention;
* gamma = 1, [D].

Draw order from one generator seeded with ``seed``: q, k, v, beta, alpha,
x, W_gs, W_gl, W_os, W_ol.  Large shapes are drawn in fp32 on the target
device and cast to the storage dtype; the oracle reads back the cast bytes.
"""

from dataclasses import dataclass

import torch


@dataclass(frozen=True)
class Shape:
    T: int          # latent frames
    N: int          # tokens per frame
    H: int          # heads
    d: int          # head dim (dk == dv)

    @property
    def L(self):
        return self.T * self.N

    @property
    def D(self):
        return self.H * self.d


# Named workloads (sizes only).
PRESETS = {
    "tiny": Shape(10, 16, 1, 16),            # 2 chunks of 5, 4x4 grid
    "tiny17": Shape(17, 16, 1, 16),          # ragged last chunk, mask < 100 %
    "layer42": Shape(42, 4032, 24, 128),     # 42 latent frames, 48x84 grid
    "layer102": Shape(102, 4032, 24, 128),   # 102 latent frames, 48x84 grid
}


def sweep_shapes():
    """VDA scan-only sweep: T x N x d x H."""
    out = []
    for T in (42, 72, 102):
        for N in (1008, 4032):
            for d in (64, 128):
                for H in (24, 48):
                    out.append(Shape(T, N, H, d))
    return out


def _randn(gen, shape, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32)


def make_inputs(shape, dtype=torch.bfloat16, seed=0, device="cpu", with_fuse=False):
    """Draw the layer's inputs for ``shape``.

    Returns a dict with q, k, v [L, D] (``dtype``), beta [L, H] fp32,
    alpha [T, H] fp32 and, when ``with_fuse``, x [L, D] (``dtype``),
    W_gs, W_gl, W_os, W_ol [D, D] (``dtype``) and gamma [D] fp32.
    """
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    L, D = shape.L, shape.D
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    out = {}
    out["q"] = _randn(gen, (L, D), device).to(dtype)
    k = _randn(gen, (L, H, d), device)
    k = k / k.norm(dim=2, keepdim=True)
    out["k"] = k.reshape(L, D).to(dtype)
    del k
    out["v"] = _randn(gen, (L, D), device).to(dtype)
    out["beta"] = torch.sigmoid(_randn(gen, (L, H), device)).contiguous()
    out["alpha"] = (0.9 + 0.1 * torch.rand((T, H), generator=gen, device=device,
                                           dtype=torch.float32)).contiguous()
    if with_fuse:
        out["x"] = _randn(gen, (L, D), device).to(dtype)
        for name in ("W_gs", "W_gl", "W_os", "W_ol"):
            out[name] = (0.02 * _randn(gen, (D, D), device)).to(dtype)
        out["gamma"] = torch.ones(D, device=device, dtype=torch.float32)
    return out


def to_host_f32(t):
    """Widen a (possibly bf16) tensor to an fp32 numpy array on the host."""
    return t.detach().to("cpu", torch.float32).numpy()
