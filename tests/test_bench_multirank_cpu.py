"""The bench's multi-rank plumbing on CPU: two gloo ranks on 127.0.0.1.

Every rank times its own video; the job time is the max over ranks and the
value is all ranks' tokens over that time (weak scaling)."""

import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            init_method=f"tcp://127.0.0.1:{port}")
    try:
        import bench
        vals = bench.max_over_ranks([100.0 + 7 * rank, 50.0 - rank, float(rank)],
                                    torch.device("cpu"), world)
        out[rank] = vals
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert out[r] == [107.0, 50.0, 1.0]


def test_weak_scaling_value():
    import bench
    assert bench.weak_scaling_value(1, 411264, 1000.0) == pytest.approx(411264.0)
    assert bench.weak_scaling_value(8, 411264, 500.0) == pytest.approx(8 * 411264 * 2.0)
    assert bench.max_over_ranks([1.0, 2.0], torch.device("cpu"), 1) == [1.0, 2.0]


def test_bench_work_model_pair_count_matches_oracle():
    """The bench's own frame-pair count (its work model for the roofline)
    equals the oracle's mask for the layer shapes and the mask variants."""
    import bench
    import oracle
    for T in (1, 2, 3, 10, 17, 42, 72, 102):
        for cf, wc, anchors in ((5, 1, 3), (5, 0, 0), (3, 2, 1), (5, 1, 2)):
            assert bench.mask_pair_count(T, cf, wc, anchors) == \
                oracle.mask_pair_count(T, chunk_frames=cf, window_chunks=wc, anchors=anchors)
