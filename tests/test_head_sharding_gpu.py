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
