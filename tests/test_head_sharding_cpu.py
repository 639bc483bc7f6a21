"""Head-parallel orchestration of one video (HeadShardedLayer) on two gloo
ranks on CPU.  The four compute calls are replaced by float64 stand-ins built
from the oracle (test-only injection), so this checks the host logic: which
head columns and beta/alpha slices each rank takes, the row-parallel fuse
partials, and the all-reduce that sums them into y."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

T, N, H, d = 7, 6, 4, 8


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _inputs():
    g = torch.Generator().manual_seed(3)
    L, D = T * N, H * d
    t = {n: torch.randn((L, D), generator=g, dtype=torch.float64) for n in ("q", "k", "v", "x")}
    t["k"] = (t["k"].view(L, H, d) / t["k"].view(L, H, d).norm(dim=2, keepdim=True)).view(L, D)
    t["beta"] = torch.sigmoid(torch.randn((L, H), generator=g, dtype=torch.float64))
    t["alpha"] = 0.9 + 0.1 * torch.rand((T, H), generator=g, dtype=torch.float64)
    for n in ("W_gs", "W_gl", "W_os", "W_ol"):
        t[n] = 0.1 * torch.randn((D, D), generator=g, dtype=torch.float64)
    t["gamma"] = 1.0 + 0.1 * torch.randn(D, generator=g, dtype=torch.float64)
    return t


def _fake_ops():
    import oracle

    def window_attn(q, k, v, T_, N_, Hl, d_, out):
        o, _ = oracle.window_attn(q.numpy(), k.numpy(), v.numpy(), T_, N_, Hl, d_)
        out.copy_(torch.from_numpy(o))

    def vda_scan(q, k, v, beta, alpha, T_, N_, Hl, d_, out):
        o, _, _ = oracle.vda(q.numpy(), k.numpy(), v.numpy(), beta.numpy(), alpha.numpy(),
                             T_, N_, Hl, d_)
        out.copy_(torch.from_numpy(o))

    def fuse_shard(x, o_s, o_vda, W_gs, W_gl, gamma, W_os, W_ol, d_, head0, eps, out):
        Dl = o_s.shape[1]
        c = slice(head0 * d_, head0 * d_ + Dl)
        g_s, g_l = oracle.fuse_gates(x.numpy(), W_gs.numpy()[c], W_gl.numpy()[c])
        n = oracle.rmsnorm_heads(o_vda.numpy(), Dl // d_, d_, gamma.numpy()[c], eps)
        y = (g_s * o_s.numpy()) @ W_os.numpy()[:, c].T + (g_l * n) @ W_ol.numpy()[:, c].T
        out.copy_(torch.from_numpy(y))

    return {"window_attn": window_attn, "vda_scan": vda_scan, "fuse_shard": fuse_shard}


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        from video_diffusion_hybrid_vda_b200.vdn import HeadShardedLayer
        t = _inputs()
        layer = HeadShardedLayer(T, N, H, d, t["W_gs"], t["W_gl"], t["W_os"], t["W_ol"],
                                 t["gamma"], device="cpu", ops=_fake_ops(),
                                 act_dtype=torch.float64, acc_dtype=torch.float64)
        y = layer.forward(t["q"], t["k"], t["v"], t["beta"], t["alpha"], t["x"])
        out[rank] = (layer.head0, layer.Hl, y.numpy().copy())
    finally:
        dist.destroy_process_group()


def test_two_rank_head_sharded_layer_equals_full_layer():
    import oracle
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    t = {k: v.numpy() for k, v in _inputs().items()}
    o_s, _ = oracle.window_attn(t["q"], t["k"], t["v"], T, N, H, d)
    o_l, _, _ = oracle.vda(t["q"], t["k"], t["v"], t["beta"], t["alpha"], T, N, H, d)
    y_ref = oracle.hybrid_fuse(t["x"], o_s, o_l, t["W_gs"], t["W_gl"], t["gamma"], 1e-6,
                               t["W_os"], t["W_ol"], H)
    assert [out[r][0] for r in range(world)] == [0, 2]
    for r in range(world):
        np.testing.assert_allclose(out[r][2], y_ref, rtol=1e-10, atol=1e-10)
