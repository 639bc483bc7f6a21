"""Branch calibration and output projections, float64 CPU oracle.  TEST INFRASTRUCTURE ONLY.

Source: "Video DeltaNet" article on 10100.com, 方法概述 item 3 (branch calibration):
the Softmax branch gets a content-dependent sigmoid gate; the linear branch
is RMS-normalised and then passes its own sigmoid output gate; each branch
has its own output projection and the two projections are added.  The
Korean summary on hotpaper.ai (기술적 접근법) repeats that RMS normalisation
and learnable gates calibrate the two paths.

Readings of the pages taken here:
* gates are elementwise over the hidden size D, computed from the block
  input x ("content-dependent"), without bias: g = sigmoid(x W^T);
* a gate multiplies its branch output before that branch's projection;
* RMSNorm acts per token and per head over the head's d channels,
  n = o / sqrt(mean(o^2) + eps) * gamma, gamma of length D;
* weights follow the y = z W^T convention with W[out, in].
"""

import numpy as np


def sigmoid(z):
    # exp(-z) overflows to inf for z below about -709; 1 / (1 + inf) = 0 is
    # then the exact float64 result, so the overflow is not reported
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-z))


def rmsnorm_heads(o, H, d, gamma, eps):
    """Per-token, per-head RMSNorm over d channels, scaled by gamma [H*d]."""
    o = np.asarray(o, dtype=np.float64)
    oh = o.reshape(o.shape[0], H, d)
    rms = np.sqrt(np.mean(oh * oh, axis=2, keepdims=True) + eps)
    return (oh / rms).reshape(o.shape[0], H * d) * np.asarray(gamma, dtype=np.float64)


def fuse_gates(x, W_gs, W_gl):
    """g_s = sigmoid(x W_gs^T), g_l = sigmoid(x W_gl^T)."""
    x = np.asarray(x, dtype=np.float64)
    g_s = sigmoid(x @ np.asarray(W_gs, dtype=np.float64).T)
    g_l = sigmoid(x @ np.asarray(W_gl, dtype=np.float64).T)
    return g_s, g_l


def hybrid_fuse_rows(x, o_s, o_vda, W_gs, W_gl, gamma, eps, W_os, W_ol, H, rows):
    """y for the given token rows: (g_s*o_s) W_os^T + (g_l*RMSNorm(o_vda)) W_ol^T."""
    rows = np.asarray(rows, dtype=np.int64)
    D = np.asarray(W_os).shape[0]
    d = D // H
    xr = np.asarray(x[rows], dtype=np.float64)
    g_s, g_l = fuse_gates(xr, W_gs, W_gl)
    zs = g_s * np.asarray(o_s[rows], dtype=np.float64)
    zl = g_l * rmsnorm_heads(o_vda[rows], H, d, gamma, eps)
    return zs @ np.asarray(W_os, dtype=np.float64).T + zl @ np.asarray(W_ol, dtype=np.float64).T


def hybrid_fuse(x, o_s, o_vda, W_gs, W_gl, gamma, eps, W_os, W_ol, H):
    """y for every token row."""
    return hybrid_fuse_rows(x, o_s, o_vda, W_gs, W_gl, gamma, eps, W_os, W_ol, H,
                            np.arange(np.asarray(x).shape[0]))
