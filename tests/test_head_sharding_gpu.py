"""HeadShardedLayer with its real CUDA calls in a one-rank NCCL group: the
sharded path (head-column views with row stride D, beta/alpha slices, the
shard fuse in fp32 and the all-reduce) must reproduce HybridLayer.  Runs with
more ranks need more GPUs than a single-GPU run provides; the multi-rank
host logic is covered on CPU (test_head_sharding_cpu.py)."""

import socket

import pytest
import torch
import torch.distributed as dist

from tests.parity_util import TOL_BF16, ensure_built, host, max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_one_rank_head_sharded_layer_matches_layer():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            init_method=f"tcp://127.0.0.1:{_free_port()}",
                            device_id=torch.device("cuda", 0))
    try:
        s = synth.Shape(12, 200, 2, 128)
        inp = synth.make_inputs(s, seed=31, device="cuda", with_fuse=True)
        w = [inp[n] for n in ("W_gs", "W_gl", "W_os", "W_ol")]
        names = ("q", "k", "v", "beta", "alpha", "x")
        ref = vdn.HybridLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"]).forward(
            *[inp[n] for n in names]).clone()
        layer = vdn.HeadShardedLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"])
        y = layer.forward(*[inp[n] for n in names])
        torch.cuda.synchronize()
        assert max_rel(host(y), host(ref)) <= TOL_BF16
    finally:
        dist.destroy_process_group()


def test_one_rank_sharded_layers_with_row_output_match_layer():
    """HeadShardedLayer with row-block output and SeqShardedLayer (all-to-alls
    of a one-rank group) with their real CUDA calls reproduce HybridLayer."""
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            init_method=f"tcp://127.0.0.1:{_free_port()}",
                            device_id=torch.device("cuda", 0))
    try:
        s = synth.Shape(17, 96, 2, 128)
        inp = synth.make_inputs(s, seed=37, device="cuda", with_fuse=True)
        w = [inp[n] for n in ("W_gs", "W_gl", "W_os", "W_ol")]
        names = ("q", "k", "v", "beta", "alpha", "x")
        ref = vdn.HybridLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"]).forward(
            *[inp[n] for n in names]).clone()
        y_rows = vdn.HeadShardedLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"],
                                      output="rows").forward(*[inp[n] for n in names])
        y_seq = vdn.SeqShardedLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"]).forward(
            *[inp[n] for n in names])
        torch.cuda.synchronize()
        assert max_rel(host(y_rows), host(ref)) <= TOL_BF16
        assert max_rel(host(y_seq), host(ref)) <= TOL_BF16
    finally:
        dist.destroy_process_group()


def _fused_rs_worker(rank, world, port, out):
    """One rank of the fused GEMM + reduce-scatter path: its own process and
    CUDA context (both on device 0 here), a gloo group for the host-side
    meetings and the handle exchange, CUDA IPC mappings of the other rank's
    row block."""
    import torch.distributed as dist_
    dist_.init_process_group("gloo", rank=rank, world_size=world,
                             init_method=f"tcp://127.0.0.1:{port}")
    try:
        ensure_built()
        from video_diffusion_hybrid_vda_b200 import vdn
        torch.cuda.set_device(0)
        s = synth.Shape(17, 96, 4, 128)
        inp = synth.make_inputs(s, seed=41, device="cuda", with_fuse=True)
        w = [inp[n] for n in ("W_gs", "W_gl", "W_os", "W_ol")]
        names = ("q", "k", "v", "beta", "alpha", "x")
        ref = vdn.HybridLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"]).forward(
            *[inp[n] for n in names]).clone()
        layer = vdn.HeadShardedLayer(s.T, s.N, s.H, s.d, *w, inp["gamma"], output="rows",
                                     collective="fused")
        errs = []
        for _ in range(2):                              # the blocks are re-zeroed per call
            y = layer.forward(*[inp[n] for n in names])
            torch.cuda.synchronize()
            errs.append(max_rel(host(y), host(ref[layer.rows])))
        layer.close()                                   # peer mappings released on both ranks
        out[rank] = (layer.rows.start, layer.rows.stop, errs)
    finally:
        dist_.destroy_process_group()


def test_fused_reduce_scatter_two_processes_match_layer():
    """HeadShardedLayer(collective="fused") on two ranks, each its own
    process: the output GEMM of every rank adds its rows of y straight into
    the owning rank's block through CUDA IPC peer mappings; each rank's
    block equals HybridLayer's rows.  The two processes share one GPU; no
    kernel waits on the other rank (the ranks meet on the host)."""
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    procs = [ctx.Process(target=_fused_rs_worker, args=(r, world, port, out))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    L = 17 * 96
    blocks = sorted((out[r][0], out[r][1]) for r in range(world))
    assert blocks[0][0] == 0 and blocks[-1][1] == L and blocks[0][1] == blocks[1][0]
    for r in range(world):
        for e in out[r][2]:
            assert e <= TOL_BF16
