"""Multi-GPU orchestration of one video on gloo ranks on CPU, for both
layouts a caller may hold:

* HeadShardedLayer (every rank holds the full activations): which head
  columns and beta/alpha slices each rank takes, the row-parallel fuse
  partials, the reduce-scatter that sums them into row blocks of y, and the
  all-gather of the blocks;
* SeqShardedLayer (every rank holds a block of token rows): the all-to-alls
  that bring all rows of a rank's heads to it and the branch outputs back,
  and the fuse on the row block.

The compute calls are replaced by float64 stand-ins built from the oracle
(test-only injection), so these check the host logic against the full
oracle layer."""

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

    def fuse(x, o_s, o_vda, W_gs, W_gl, gamma, W_os, W_ol, H_, eps, out):
        y = oracle.hybrid_fuse(x.numpy(), o_s.numpy(), o_vda.numpy(), W_gs.numpy(), W_gl.numpy(),
                               gamma.numpy(), eps, W_os.numpy(), W_ol.numpy(), H_)
        out.copy_(torch.from_numpy(y))

    return {"window_attn": window_attn, "vda_scan": vda_scan, "fuse_shard": fuse_shard,
            "fuse": fuse}


def _worker(rank, world, port, out):
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        from video_diffusion_hybrid_vda_b200.vdn import HeadShardedLayer
        t = _inputs()
        res = {}
        for mode in ("full", "rows"):
            layer = HeadShardedLayer(T, N, H, d, t["W_gs"], t["W_gl"], t["W_os"], t["W_ol"],
                                     t["gamma"], device="cpu", ops=_fake_ops(),
                                     act_dtype=torch.float64, acc_dtype=torch.float64,
                                     output=mode)
            y = layer.forward(t["q"], t["k"], t["v"], t["beta"], t["alpha"], t["x"])
            res[mode] = (layer.head0, layer.Hl, layer.rows, y.numpy().copy())
        out[rank] = res
    finally:
        dist.destroy_process_group()


def _run_ranks(target, world, *args):
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=target, args=(r, world, port, out) + args) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
        assert p.exitcode == 0
    return out


def _oracle_layer(t, T_, N_, H_, d_):
    import oracle
    t = {k: v.numpy() for k, v in t.items()}
    o_s, _ = oracle.window_attn(t["q"], t["k"], t["v"], T_, N_, H_, d_)
    o_l, _, _ = oracle.vda(t["q"], t["k"], t["v"], t["beta"], t["alpha"], T_, N_, H_, d_)
    return oracle.hybrid_fuse(t["x"], o_s, o_l, t["W_gs"], t["W_gl"], t["gamma"], 1e-6,
                              t["W_os"], t["W_ol"], H_)


def test_two_rank_head_sharded_layer_equals_full_layer():
    world = 2
    out = _run_ranks(_worker, world)
    y_ref = _oracle_layer(_inputs(), T, N, H, d)
    assert [out[r]["full"][0] for r in range(world)] == [0, 2]
    blocks = []
    for r in range(world):
        np.testing.assert_allclose(out[r]["full"][3], y_ref, rtol=1e-10, atol=1e-10)
        rows, y_rows = out[r]["rows"][2], out[r]["rows"][3]
        np.testing.assert_allclose(y_rows, y_ref[rows], rtol=1e-10, atol=1e-10)
        blocks.append((rows.start, rows.stop))
    # the row blocks tile [0, L) in rank order
    assert blocks[0][0] == 0 and blocks[-1][1] == T * N
    assert all(blocks[i][1] == blocks[i + 1][0] for i in range(world - 1))


# sequence-sharded caller: 17 frames (the mask masks), 68 rows over 2 or 4 ranks
TS, NS = 17, 4


def _seq_inputs():
    g = torch.Generator().manual_seed(5)
    L, D = TS * NS, H * d
    t = {n: torch.randn((L, D), generator=g, dtype=torch.float64) for n in ("q", "k", "v", "x")}
    t["k"] = (t["k"].view(L, H, d) / t["k"].view(L, H, d).norm(dim=2, keepdim=True)).view(L, D)
    t["beta"] = torch.sigmoid(torch.randn((L, H), generator=g, dtype=torch.float64))
    t["alpha"] = 0.9 + 0.1 * torch.rand((TS, H), generator=g, dtype=torch.float64)
    for n in ("W_gs", "W_gl", "W_os", "W_ol"):
        t[n] = 0.1 * torch.randn((D, D), generator=g, dtype=torch.float64)
    t["gamma"] = 1.0 + 0.1 * torch.randn(D, generator=g, dtype=torch.float64)
    return t


def _seq_worker(rank, world, port, out):
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        from video_diffusion_hybrid_vda_b200.vdn import SeqShardedLayer
        t = _seq_inputs()
        layer = SeqShardedLayer(TS, NS, H, d, t["W_gs"], t["W_gl"], t["W_os"], t["W_ol"],
                                t["gamma"], device="cpu", ops=_fake_ops(),
                                act_dtype=torch.float64, acc_dtype=torch.float64)
        r = layer.rows
        # the caller holds only its rows (and the whole alpha)
        y = layer.forward(*[t[n][r].clone() for n in ("q", "k", "v", "beta")], t["alpha"],
                          t["x"][r].clone())
        out[rank] = (r, layer.head0, y.numpy().copy())
    finally:
        dist.destroy_process_group()


def test_sequence_sharded_layer_equals_full_layer():
    y_ref = _oracle_layer(_seq_inputs(), TS, NS, H, d)
    for world in (2, 4):
        out = _run_ranks(_seq_worker, world)
        R = TS * NS // world
        for r in range(world):
            rows, head0, y = out[r]
            assert (rows.start, rows.stop, head0) == (r * R, (r + 1) * R, r * H // world)
            np.testing.assert_allclose(y, y_ref[rows], rtol=1e-10, atol=1e-10)
