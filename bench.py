"""Benchmark of the Video DeltaNet hybrid attention layer on B200.

One step = one pass of the whole layer (window-and-anchor Softmax, Video
Delta Attention prep/solve/scan/read-out, gated fuse with both output
projections) over one video's synthetic inputs at 102 latent frames x 4032
tokens (48x84), 24 heads x 128, bf16, seeded.  Inputs live in HBM when the
timed region starts; each activation (2.5 GB) is larger than L2, so no L2
flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload layer102|layer42|small]
                    [--part all|layer|vda_backward|fuse_mxfp8|window_mxfp8|layer_mxfp8|
                            scan_sweep]
                    [--parallel videos|heads|seq] [--collective reduce_scatter|fused]
                    [--solver gauss-jordan|cholesky]

The line also carries rows timed on their own, not part of the step:
``vda_backward``, the VDA gradient pass (dq, dk, dv, dbeta, dalpha from
dL/do_vda, forward recomputed inside, and on a saved forward);
``vda_by_solver``, the VDA branch with each solve of (I + A_t)^-1
(Gauss-Jordan, the default, and Cholesky); ``fuse_mxfp8``, the fuse with
both projection GEMMs in MXFP8 (x quantized inside the timed call, weights
quantized beforehand), against the FP8 peak and beside the bf16 fuse's
output; ``window_mxfp8``, the window Softmax with both products in MXFP8
(q, k, v quantized inside the timed call), against its FP8 tensor and MUFU
bounds and beside the bf16 window Softmax's output; and ``layer_mxfp8``,
the whole layer pass with both MXFP8 modes, beside the bf16 layer's y.
``--part vda_backward`` / ``fuse_mxfp8`` / ``window_mxfp8`` /
``layer_mxfp8`` time only that row (for launch lists and captures).
``--part scan_sweep`` times the VDA branch alone at every point of the
scan-only sweep (T 42/72/102 x N 1008/4032 x d 64/128 x H 24/48), each
against its roofline.

With N > 1 (torchrun) every rank runs its own video (independent problems,
no collective on the data path): weak scaling, time = max over ranks.
``--parallel heads`` instead splits one video over the ranks by heads
(every rank holds the full activations; the row-parallel fuse ends in a
reduce-scatter of y, NCCL's or the fused GEMM + reduce-scatter kernel's
with ``--collective fused``), and ``--parallel seq`` by token rows, with
the attention branches run head-parallel between two all-to-alls (both
strong scaling; on one GPU a one-rank group).
``--impl reference`` times the float64 CPU oracle instead, on a bounded
sample of the same workload, extrapolated by work.
"""

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from video_diffusion_hybrid_vda_b200 import synth  # noqa: E402

WORKLOADS = {
    "layer102": synth.Shape(102, 4032, 24, 128),
    "layer42": synth.Shape(42, 4032, 24, 128),
    "small": synth.Shape(12, 4032, 24, 128),   # for ncu captures: ~2 GB on the device
}
METRIC = "VDN hybrid attn layer ms & tokens/s at 102 latent frames; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# FP32 (non-tensor) peak from unit counts and clocks: 148 SMs x 128 FMA/clk x
# 2 FLOP x 1.965 GHz (clocks.max.sm)
FP32_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
# MUFU exponentials from unit counts and clocks: 148 SMs x 16 per clock x 1.965 GHz
MUFU_EXP_PER_S = 148 * 16 * 1.965e9
KERNEL_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "window_attn_traffic.json")


def mask_pair_count(T, cf=5, wc=1, anchors=3):
    """Visible (query frame, key frame) pairs of the window-and-anchor mask."""
    n = 0
    for tq in range(T):
        for tk in range(T):
            if (anchors & 1 and 0 in (tq, tk)) or (anchors & 2 and T - 1 in (tq, tk)) or \
                    abs(tq // cf - tk // cf) <= wc:
                n += 1
    return n


WINDOW_SOURCES = ("window_attn.cu", "window_sched.cuh", "ptx.cuh", "common.cuh", "repack.cuh",
                  "exp2_fma.cuh")


def window_source_hash():
    """sha256 over the sources the window Softmax kernel is built from (a
    stored DRAM-traffic figure is used only while these are unchanged)."""
    import hashlib
    h = hashlib.sha256()
    for name in WINDOW_SOURCES:
        with open(os.path.join(ROOT, "video_diffusion_hybrid_vda_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def work_model(s):
    """Algorithmic work of one layer pass (unmasked pairs only)."""
    pairs = mask_pair_count(s.T) * s.N * s.N          # token pairs per head
    softmax_flop = pairs * s.H * 4 * s.d                # QK^T and PV
    proj_flop = 4 * 2 * s.L * s.D * s.D                 # gate GEMMs + output GEMMs
    # VDA HBM bytes: prep reads k, v (bf16) and beta; read-out reads q, writes o
    vda_bytes = 2 * s.L * s.D * 2 + s.L * s.H * 4 + 2 * s.L * s.D * 2
    # FP32 ALU work in FLOP (an FMA is 2, as in the FP32 peak) per (frame,
    # head): the SPD inverse, d^3 FMA (Gauss-Jordan: d pivots x d^2 updates;
    # Cholesky: factor, W = L^-1 and P = W^T W, d^3 / 3 each), and both
    # scans' (alpha S + B) P, a d^3-FMA product each
    vda_alu_flop = s.T * s.H * (2 * s.d ** 3 + 4 * s.d ** 3)
    # VDA gradient pass: reads q, k, v, dO (bf16) and beta, writes dq, dk, dv
    # (bf16) and dbeta; FP32 ALU: the forward's solve and scans again, the
    # two adjoint scans (2 d^3 each) and the combine (two d^3 products, 4 d^3);
    # on a saved forward (P and states kept) only the last two
    vda_bwd_bytes = 7 * s.L * s.D * 2 + 2 * s.L * s.H * 4
    vda_bwd_saved_alu_flop = s.T * s.H * (4 * s.d ** 3 + 4 * s.d ** 3)
    vda_bwd_alu_flop = vda_alu_flop + vda_bwd_saved_alu_flop
    return dict(pairs=pairs, heads=s.H, softmax_flop=softmax_flop, proj_flop=proj_flop,
                vda_bytes=vda_bytes, vda_alu_flop=vda_alu_flop, vda_bwd_bytes=vda_bwd_bytes,
                vda_bwd_alu_flop=vda_bwd_alu_flop, vda_bwd_saved_alu_flop=vda_bwd_saved_alu_flop)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def clocks_start():
    fd, path = tempfile.mkstemp(suffix=".csv")
    os.close(fd)
    q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    dev = os.environ.get("LOCAL_RANK", "0")
    try:
        with open(path, "w") as out:  # the sampler keeps its own descriptor
            p = subprocess.Popen(["nvidia-smi", f"--id={dev}", f"--query-gpu={q}",
                                  "--format=csv,noheader,nounits", "-lms", "200"],
                                 stdout=out, stderr=subprocess.DEVNULL)
    except OSError:
        p = None
    return p, path


def clocks_stop(handle):
    p, path = handle
    if p is None:
        return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
    p.terminate()
    try:
        p.wait(timeout=5)
    except subprocess.TimeoutExpired:
        p.kill()
    sm, smax, reasons = [], None, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    with open(path) as f:
        for line in f:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
    os.unlink(path)
    return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
            "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- ranks

def max_over_ranks(values, device, world):
    """Element-wise max of a list of floats over all ranks (identity at N=1)."""
    if world <= 1:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def free_port():
    import socket
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    return port


def weak_scaling_value(world, tokens_per_rank, ms_per_step):
    """Whole-job tokens/s: every rank processes its own video per step."""
    return world * tokens_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------------- CPU oracle

def oracle_sample(shape, seed=0, vda_heads=2, frames=None, rows_per_frame=128):
    """Time the float64 oracle on a bounded sample of the layer and
    extrapolate to one full layer pass by the work ratio of each step.

    Sample: VDA (prep, solve, both scans, read-out) for `vda_heads` heads over
    all frames; window Softmax for `rows_per_frame` query rows of each
    sampled frame (default {0, 1, 4, 5, T/2, T-3, T-2, T-1}) in one head;
    fuse for 256 rows.  Inputs are drawn on the host with the same laws.
    """
    import oracle
    from threadpoolctl import threadpool_info
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    L, D = shape.L, shape.D
    sub = synth.Shape(T, N, vda_heads, d)
    x = {k: v.numpy() for k, v in synth.make_inputs(sub, dtype=torch.float32, seed=seed).items()}
    t0 = time.perf_counter()
    oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], T, N, vda_heads, d)
    t_vda = (time.perf_counter() - t0) * H / vda_heads

    if frames is None:
        frames = [0, 1, 4, 5, T // 2, T - 3, T - 2, T - 1]
    frames = sorted(set(frames))
    rows = np.concatenate([np.arange(f * N, f * N + min(rows_per_frame, N)) for f in frames])
    c = slice(0, d)
    t0 = time.perf_counter()
    oracle.window_attn_rows(x["q"][:, c], x["k"][:, c], x["v"][:, c], T, N, 1, d, rows)
    t_win_s = time.perf_counter() - t0
    sampled_pairs = sum(len(oracle.visible_key_frames(int(r) // N, T)) * N for r in rows)
    t_win = t_win_s * (mask_pair_count(T) * N * N * H) / sampled_pairs

    g = torch.Generator().manual_seed(seed + 7)
    nr = 256
    xr = torch.randn((nr, D), generator=g).numpy()
    o_s = torch.randn((nr, D), generator=g).numpy()
    o_l = torch.randn((nr, D), generator=g).numpy()
    W = [(0.02 * torch.randn((D, D), generator=g)).numpy() for _ in range(4)]
    t0 = time.perf_counter()
    oracle.hybrid_fuse_rows(xr, o_s, o_l, W[0], W[1], np.ones(D), 1e-6, W[2], W[3], H,
                            np.arange(nr))
    t_fuse = (time.perf_counter() - t0) * L / nr
    total = t_vda + t_win + t_fuse
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return {
        "value": L / total, "unit": "tokens/s", "cores": threads, "kind": "oracle",
        "sample": ("float64 numpy oracle, extrapolated by work: VDA %d of %d heads x %d frames "
                   "(%.1f s), window Softmax %d query rows of frames %s x 1 head (%.1f s), "
                   "fuse %d rows (%.1f s); full layer est. %.0f s"
                   % (vda_heads, H, T, t_vda * vda_heads / H, len(rows), frames, t_win_s, nr,
                      t_fuse * nr / L, total)),
        "seconds_per_layer": total,
    }


# ---------------------------------------------------------------- GPU arm

def run_gpu(args, shape, rank, world):
    from video_diffusion_hybrid_vda_b200 import vdn
    vdn.set_vda_solver(vdn.SOLVER_GAUSS_JORDAN if args.solver == "gauss-jordan"
                       else vdn.SOLVER_CHOLESKY)
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev, with_fuse=True)
    layer = vdn.HybridLayer(shape.T, shape.N, shape.H, shape.d, inp["W_gs"], inp["W_gl"],
                            inp["W_os"], inp["W_ol"], inp["gamma"], device=dev)
    acts = [inp[k] for k in ("q", "k", "v", "beta", "alpha", "x")]
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        """One layer pass; ``ev`` = 4 events bracketing the three C-ABI calls."""
        q, k, v, beta, alpha, x = acts
        cf, wc, an = layer.mask
        if ev is not None:
            ev[0].record(stream)
        vdn.window_attn(q, k, v, shape.T, shape.N, shape.H, shape.d, cf, wc, an,
                        out=layer.o_s, ws=layer.ws_win, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        vdn.vda_scan(q, k, v, beta, alpha, shape.T, shape.N, shape.H, shape.d,
                     out=layer.o_vda, ws=layer.ws_vda, stream=stream)
        if ev is not None:
            ev[2].record(stream)
        vdn.hybrid_fuse(x, layer.o_s, layer.o_vda, layer.W_gs, layer.W_gl, layer.gamma,
                        layer.W_os, layer.W_ol, shape.H, out=layer.y, ws=layer.ws_fuse,
                        stream=stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if layer.status() != 0:
        raise RuntimeError("device status after warm-up: %d" % layer.status())

    def barrier():
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()

    call_events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)]
                   for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = clocks_start()
    barrier()
    start.record(stream)
    for i in range(args.steps):
        step(call_events[i])
    end.record(stream)
    barrier()
    clocks = clocks_stop(clk)
    ms = start.elapsed_time(end)
    win_ms = [e[0].elapsed_time(e[1]) for e in call_events]
    vda_ms = [e[1].elapsed_time(e[2]) for e in call_events]
    fuse_ms = [e[2].elapsed_time(e[3]) for e in call_events]
    status = layer.status()
    if status != 0:
        raise RuntimeError("device status after timed steps: %d" % status)

    # ---- end to end through HybridLayer.forward_many: every step copies its
    # inputs from pinned host memory and reads y back into pinned host memory;
    # the copies of neighbouring steps overlap the current step's compute.
    # Two pinned input sets alternate between steps (host RAM), so every
    # step's copy is a real transfer.
    host_sets = [[t.to("cpu").pin_memory() for t in acts] for _ in range(2)]
    e2e_steps = max(8, args.steps)  # a pipelined stream: 8 videos amortise its fill and drain
    host_outs = [torch.empty((shape.L, shape.D), dtype=torch.bfloat16).pin_memory()
                 for _ in range(2)]
    batches = [host_sets[i % 2] for i in range(e2e_steps)]
    outs = [host_outs[i % 2] for i in range(e2e_steps)]
    h2d = sum(t.numel() * t.element_size() for t in host_sets[0])
    d2h = host_outs[0].numel() * host_outs[0].element_size()
    layer.forward_many(batches[:2], outs[:2], stream=stream)     # warm-up of the path
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    layer.forward_many(batches, outs, stream=stream)
    stream.wait_event(layer._read[-1])                           # last read-back done
    e1.record(stream)
    barrier()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if layer.status() != 0:
        raise RuntimeError("device status after end-to-end steps")

    t = max_over_ranks([ms, e2e_ms, sum(win_ms), sum(vda_ms), sum(fuse_ms)], dev, world)
    ms, e2e_ms = t[0], t[1]
    return dict(ms=ms, win_ms=t[2] / args.steps, vda_ms=t[3] / args.steps,
                fuse_ms=t[4] / args.steps, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
                clocks=clocks, launches=layer.kernels_per_forward * args.steps)


def run_seq_sharded(args, shape, rank, world):
    """One video split over the ranks (SeqShardedLayer): each rank holds a
    block of token rows; all-to-alls move its heads' rows in and the branch
    outputs back; time of `steps` layer passes, max over ranks."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=0, device=dev, with_fuse=True)
    layer = vdn.SeqShardedLayer(shape.T, shape.N, shape.H, shape.d, inp["W_gs"], inp["W_gl"],
                                inp["W_os"], inp["W_ol"], inp["gamma"], device=dev)
    r = layer.rows
    mine = [inp[n][r].contiguous() for n in ("q", "k", "v", "beta")] + \
        [inp["alpha"], inp["x"][r].contiguous()]
    del inp
    torch.cuda.empty_cache()
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        layer.forward(*mine)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = clocks_start()
    torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        layer.forward(*mine)
    end.record(stream)
    torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = clocks_stop(clk)
    if max(get_status(w) for w in layer.workspaces) != 0:
        raise RuntimeError("device status after the sharded steps")
    ms = max_over_ranks([start.elapsed_time(end)], dev, world)[0]
    return ms / args.steps, clocks


def run_head_sharded(args, shape, rank, world):
    """One video split over the ranks by heads (HeadShardedLayer): every rank
    holds the full activations, runs both branches on its H/G heads and the
    row-parallel fuse on its columns, and one reduce-scatter (NCCL, or the
    fused GEMM + reduce-scatter over peer mappings) leaves it a row block of
    y; time of `steps` layer passes, max over ranks."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=0, device=dev, with_fuse=True)
    layer = vdn.HeadShardedLayer(shape.T, shape.N, shape.H, shape.d, inp["W_gs"], inp["W_gl"],
                                 inp["W_os"], inp["W_ol"], inp["gamma"], device=dev,
                                 output="rows", collective=args.collective)
    acts = [inp[n] for n in ("q", "k", "v", "beta", "alpha", "x")]
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        layer.forward(*acts)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = clocks_start()
    torch.distributed.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for _ in range(args.steps):
        layer.forward(*acts)
    end.record(stream)
    torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks = clocks_stop(clk)
    if max(get_status(w) for w in layer.workspaces) != 0:
        raise RuntimeError("device status after the sharded steps")
    ms = max_over_ranks([start.elapsed_time(end)], dev, world)[0]
    layer.close()
    return ms / args.steps, clocks


def get_status(ws):
    from video_diffusion_hybrid_vda_b200 import vdn
    return vdn.get_device_status(ws)


def run_vda_solvers(args, shape, rank, world):
    """Device time of the VDA branch (prep, solve, scan, read-out; ms, max
    over ranks) with each solver of (I + A_t)^-1; they differ only in the
    solve kernel."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev)
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    o = torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev)
    ws = vdn.alloc_workspace(vdn.vda_scan_workspace(T, N, H, d), dev)
    stream = torch.cuda.current_stream(dev)
    solvers = (("gauss_jordan", vdn.SOLVER_GAUSS_JORDAN), ("cholesky", vdn.SOLVER_CHOLESKY))
    calls = 20  # per round: the branch is ~3.6 ms, so a round is long enough to time
    best = {name: float("inf") for name, _ in solvers}
    for rnd in range(3):  # the solvers alternate, so clock drift hits both alike
        for name, solver in solvers:
            vdn.set_vda_solver(solver)
            for _ in range(args.warmup):
                vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H,
                             d, out=o, ws=ws, stream=stream)
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(calls):
                vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H,
                             d, out=o, ws=ws, stream=stream)
            e1.record(stream)
            if world > 1:
                torch.distributed.barrier()
            torch.cuda.synchronize()
            ms = max_over_ranks([e0.elapsed_time(e1) / calls], dev, world)[0]
            best[name] = min(best[name], ms)
    res = {name + "_ms": ms for name, ms in best.items()}
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the solver comparison")
    vdn.set_vda_solver(vdn.SOLVER_GAUSS_JORDAN if args.solver == "gauss-jordan"
                       else vdn.SOLVER_CHOLESKY)
    del inp, o, ws
    torch.cuda.empty_cache()
    res["default"] = "gauss-jordan"
    res["note"] = ("VDA branch (4 launches) with each solve, best of 3 alternating rounds of "
                   "20 calls; the other three kernels are shared")
    return res


def run_vda_backward(args, shape, rank, world):
    """Device time of one VDA gradient pass (ms, max over ranks)."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1000 + rank)
    d_o = torch.randn((shape.L, shape.D), generator=gen, device=dev).to(torch.bfloat16)
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    outs = [torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev) for _ in range(3)]
    dbeta = torch.empty((shape.L, H), dtype=torch.float32, device=dev)
    dalpha = torch.empty((T, H), dtype=torch.float32, device=dev)
    ws = vdn.alloc_workspace(vdn.vda_backward_workspace(T, N, H, d), dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], d_o, T, N, H,
                         d, dq=outs[0], dk=outs[1], dv=outs[2], dbeta=dbeta, dalpha=dalpha,
                         ws=ws, stream=stream)

    for _ in range(args.warmup):
        step()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the gradient pass warm-up")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the timed gradient passes")
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev, world)[0]

    # the same pass taking P and the states from a forward run on its workspace
    o_vda = torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev)
    vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H, d, out=o_vda,
                 ws=ws, stream=stream)

    def step_saved():
        vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], d_o, T, N, H,
                         d, dq=outs[0], dk=outs[1], dv=outs[2], dbeta=dbeta, dalpha=dalpha,
                         ws=ws, stream=stream, reuse_forward=True)

    for _ in range(args.warmup):
        step_saved()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(args.steps):
        step_saved()
    e1.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the gradient passes on a saved forward")
    ms_saved = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev, world)[0]
    del inp, d_o, outs, ws, o_vda
    torch.cuda.empty_cache()
    return ms, ms_saved


def run_fuse_mxfp8(args, shape, rank, world):
    """Device time of the MXFP8 fuse (ms, max over ranks) and the max
    relative deviation of its output from the bf16 fuse's on the same inputs."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev, with_fuse=True)
    gen = torch.Generator(device=dev)
    gen.manual_seed(2000 + rank)
    o_s = torch.randn((shape.L, shape.D), generator=gen, device=dev).to(torch.bfloat16)
    o_vda = torch.randn((shape.L, shape.D), generator=gen, device=dev).to(torch.bfloat16)
    wg, wo = vdn.mxfp8_fuse_weights(inp["W_gs"], inp["W_gl"], inp["W_os"], inp["W_ol"])
    y = torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev)
    ws = vdn.alloc_workspace(vdn.lib().vdn_hybrid_fuse_mxfp8_workspace(shape.L, shape.D, shape.H),
                             dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        vdn.hybrid_fuse_mxfp8(inp["x"], o_s, o_vda, wg, inp["gamma"], wo, shape.H, out=y, ws=ws,
                              stream=stream)

    for _ in range(args.warmup):
        step()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the MXFP8 fuse warm-up")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev, world)[0]
    y_bf16, _ = vdn.hybrid_fuse(inp["x"], o_s, o_vda, inp["W_gs"], inp["W_gl"], inp["gamma"],
                                inp["W_os"], inp["W_ol"], shape.H)
    dev_rel = float(((y.float() - y_bf16.float()).abs().max() / y_bf16.float().abs().max()).item())
    del inp, o_s, o_vda, wg, wo, y, ws, y_bf16
    torch.cuda.empty_cache()
    return ms, dev_rel


def run_window_mxfp8(args, shape, rank, world):
    """Device time of the MXFP8 window Softmax (quantization of q, k, v and
    the attention; ms, max over ranks) and the max relative deviation of its
    output from the bf16 window Softmax's on the same inputs."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev)
    T, N, H, d = shape.T, shape.N, shape.H, shape.d
    o = torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev)
    ws = vdn.alloc_workspace(vdn.window_attn_mxfp8_workspace(T, N, H, d), dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        vdn.window_attn_mxfp8(inp["q"], inp["k"], inp["v"], T, N, H, d, out=o, ws=ws,
                              stream=stream)

    for _ in range(args.warmup):
        step()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the MXFP8 window warm-up")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev, world)[0]
    o_bf16, _ = vdn.window_attn(inp["q"], inp["k"], inp["v"], T, N, H, d)
    dev_rel = float(((o.float() - o_bf16.float()).abs().max() /
                     o_bf16.float().abs().max()).item())
    del inp, o, ws, o_bf16
    torch.cuda.empty_cache()
    return ms, dev_rel


def run_layer_mxfp8(args, shape, rank, world):
    """Device time of one layer pass with both MXFP8 modes (the window
    Softmax's products and both fuse GEMMs on MXFP8 operands; ms, max over
    ranks) and the max relative deviation of its y from the bf16 layer's."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = synth.make_inputs(shape, seed=rank, device=dev, with_fuse=True)
    w = [inp[n] for n in ("W_gs", "W_gl", "W_os", "W_ol")]
    acts = [inp[n] for n in ("q", "k", "v", "beta", "alpha", "x")]
    layer = vdn.HybridLayer(shape.T, shape.N, shape.H, shape.d, *w, inp["gamma"], device=dev,
                            projections="mxfp8", softmax="mxfp8")
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        layer.forward(*acts, stream=stream)
    torch.cuda.synchronize()
    if layer.status() != 0:
        raise RuntimeError("device status after the MXFP8 layer warm-up")
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        y = layer.forward(*acts, stream=stream)
    e1.record(stream)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = max_over_ranks([e0.elapsed_time(e1) / args.steps], dev, world)[0]
    y = y.clone()
    del layer
    torch.cuda.empty_cache()
    ref = vdn.HybridLayer(shape.T, shape.N, shape.H, shape.d, *w, inp["gamma"], device=dev)
    y_bf16 = ref.forward(*acts, stream=stream)
    dev_rel = float(((y.float() - y_bf16.float()).abs().max() / y_bf16.float().abs().max()).item())
    del ref, inp, acts, y, y_bf16
    torch.cuda.empty_cache()
    return ms, dev_rel


def layer_mxfp8_row(shape, ms, dev_rel):
    return {"ms": ms, "tokens_per_s": shape.L / (ms / 1e3),
            "launches_per_pass": 11,
            "max_rel_vs_bf16_layer": dev_rel,
            "note": "window Softmax and both projections on MXFP8 operands (q, k, v, x "
                    "quantized inside the pass, weights beforehand); VDA in bf16 / fp32"}


def window_mxfp8_row(work, peaks, ms, dev_rel):
    """The MXFP8 window Softmax against its two bounds: FP8 tensor work at
    2 x the measured sustained bf16 rate, and one MUFU exponential per
    visible (query, key) pair at the MUFU rate from unit counts and the
    maximum clock (16 per clock per SM, 148 SMs, 1965 MHz)."""
    peak = 2.0 * peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    tensor_ms = work["softmax_flop"] / (peak * 1e12) * 1e3
    exps = work["pairs"] * work["heads"]
    mufu_ms = exps / MUFU_EXP_PER_S * 1e3
    bound_ms = max(tensor_ms, mufu_ms)
    tf = work["softmax_flop"] / (ms / 1e3) / 1e12
    return {"ms": ms, "bound": "mufu" if mufu_ms >= tensor_ms else "tensor",
            "roofline_ms": bound_ms, "frac": bound_ms / ms, "achieved_tflops": tf,
            "tensor_ms": tensor_ms, "fp8_peak_tflops": peak, "mufu_ms": mufu_ms,
            "exponentials": exps, "max_rel_vs_bf16_window": dev_rel,
            "launches_per_call": 4,
            "note": "q, k, v quantized inside the timed call (3 launches) + the attention"}


def run_scan_sweep(args, rank, world, peaks):
    """The VDA branch alone (prep, solve, both scans, read-out: one
    vdn_vda_scan call) at every point of the scan-only sweep, each timed with
    CUDA events over `steps` calls after `warmup`; one row per point with its
    roofline (HBM bytes at the measured copy bandwidth plus FP32 work at the
    FP32 peak, the same terms as the layer's VDA row)."""
    from video_diffusion_hybrid_vda_b200 import vdn
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    rows = []
    for shape in synth.sweep_shapes():
        T, N, H, d = shape.T, shape.N, shape.H, shape.d
        inp = synth.make_inputs(shape, seed=rank, device=dev)
        out = torch.empty((shape.L, shape.D), dtype=torch.bfloat16, device=dev)
        ws = vdn.alloc_workspace(vdn.vda_scan_workspace(T, N, H, d), dev)

        def call():
            vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], T, N, H, d,
                         out=out, ws=ws, stream=stream)

        for _ in range(args.warmup):
            call()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize()
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
        if vdn.get_device_status(ws) != 0:
            raise RuntimeError("device status after the sweep point %s" % (shape,))
        ms = max_over_ranks([statistics.median(a.elapsed_time(b) for a, b in evs)], dev,
                            world)[0]
        w = work_model(shape)
        roof_ms = (w["vda_bytes"] / (peaks["hbm_gbs"] * 1e9) +
                   w["vda_alu_flop"] / (FP32_TFLOPS * 1e12)) * 1e3
        rows.append({"T": T, "N": N, "d": d, "H": H, "ms": ms,
                     "tokens_per_s": shape.L / (ms / 1e3), "roofline_ms": roof_ms,
                     "frac": roof_ms / ms, "hbm_bytes": w["vda_bytes"],
                     "fp32_alu_flop": w["vda_alu_flop"]})
        del inp, out, ws
        torch.cuda.empty_cache()
    return rows


def mxfp8_row(work, peaks, ms, dev_rel):
    peak = 2.0 * peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    tf = work["proj_flop"] / (ms / 1e3) / 1e12
    return {"ms": ms, "bound": "tensor", "achieved_tflops": tf, "peak_tflops": peak,
            "frac": tf / peak, "peak_source": "measured bf16_tflops_sustained x 2 (nominal "
                                              "fp8 / bf16 dense ratio)",
            "max_rel_vs_bf16_fuse": dev_rel, "launches_per_call": 3}


def backward_row(work, peaks, ms, ms_saved):
    hbm_ms = work["vda_bwd_bytes"] / (peaks["hbm_gbs"] * 1e9) * 1e3
    roof_ms = hbm_ms + work["vda_bwd_alu_flop"] / (FP32_TFLOPS * 1e12) * 1e3
    roof_saved = hbm_ms + work["vda_bwd_saved_alu_flop"] / (FP32_TFLOPS * 1e12) * 1e3
    return {"ms": ms, "bound": "hbm + fp32 alu", "roofline_ms": roof_ms, "frac": roof_ms / ms,
            "hbm_bytes": work["vda_bwd_bytes"], "fp32_alu_flop": work["vda_bwd_alu_flop"],
            "launches_per_pass": 7,
            "ms_saved_forward": ms_saved, "launches_saved_forward": 4,
            "roofline_ms_saved_forward": roof_saved, "frac_saved_forward": roof_saved / ms_saved,
            "fp32_alu_flop_saved_forward": work["vda_bwd_saved_alu_flop"],
            "note": "ms: forward recomputed inside; ms_saved_forward: P and states taken "
                    "from a forward run on the same workspace (same HBM bytes, without the "
                    "forward's solve and scans)"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="vdn", choices=["vdn", "reference"])
    ap.add_argument("--workload", default="layer102", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--solver", default="gauss-jordan", choices=["gauss-jordan", "cholesky"],
                    help="solver of (I + A)^-1 in the VDA branch")
    ap.add_argument("--parallel", default="videos", choices=["videos", "heads", "seq"],
                    help="with several GPUs: every rank runs its own video (videos, weak "
                         "scaling); or one video is split over the ranks (strong scaling) by "
                         "heads, every rank holding the full activations and keeping a row "
                         "block of y (heads), or by token rows with head-parallel attention "
                         "in between (seq)")
    ap.add_argument("--collective", default="reduce_scatter",
                    choices=["reduce_scatter", "fused"],
                    help="--parallel heads: NCCL reduce-scatter of the fp32 partials, or the "
                         "output GEMM adding its rows into the owners' blocks over peer "
                         "mappings")
    ap.add_argument("--part", default="all",
                    choices=["all", "layer", "vda_backward", "fuse_mxfp8", "window_mxfp8",
                             "layer_mxfp8", "scan_sweep"],
                    help="what to time: the layer step and its side rows (all), one side "
                         "row, the layer step alone (layer), or the VDA branch over the "
                         "scan-only sweep (scan_sweep)")
    args = ap.parse_args()
    shape = WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    work = work_model(shape)
    config = {"workload": f"hybrid_layer_T{shape.T}_N{shape.N}_H{shape.H}_d{shape.d}",
              "latent_frames": shape.T, "tokens_per_frame": shape.N, "grid": "48x84",
              "heads": shape.H, "head_dim": shape.d, "hidden": shape.D, "tokens": shape.L,
              "mask": "chunk 5, +-1 chunk, first/last-frame anchors",
              "global_batch": world, "parallelism": f"independent videos x{world}",
              "vda_solver": args.solver,
              "l2": "inputs larger than L2 (%.2f GB per activation), no flush"
                    % (shape.L * shape.D * 2 / 1e9)}

    if args.impl == "reference":
        if rank != 0:
            return
        # each step: a smaller bounded sample (1 VDA head, 4 sampled frames)
        small = dict(vda_heads=1, frames=[0, 5, shape.T // 2, shape.T - 1])
        for i in range(args.warmup):
            oracle_sample(shape, seed=100 + i, **small)
        runs = [oracle_sample(shape, seed=i, **small) for i in range(args.steps)]
        secs = statistics.median(r["seconds_per_layer"] for r in runs)
        cpu = dict(runs[0])
        cpu["value"] = shape.L / secs
        cpu["sample"] = ("median of %d steps, each: " % args.steps) + cpu["sample"]
        line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": secs * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": config,
                "cpu_baseline": {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")},
                "e2e": {"value": cpu["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    if world > 1:
        torch.distributed.init_process_group(
            "nccl", device_id=torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0))),
            timeout=__import__("datetime").timedelta(seconds=300))
    peaks, peak_kind = load_peaks()
    if args.parallel in ("seq", "heads"):
        if world == 1:
            torch.distributed.init_process_group(
                "nccl", rank=0, world_size=1, init_method="tcp://127.0.0.1:%d" % free_port(),
                device_id=torch.device("cuda", 0))
        if args.parallel == "seq":
            ms, clocks = run_seq_sharded(args, shape, rank, world)
            par = f"sequence x{world}, head-parallel attention (all-to-all)"
        else:
            ms, clocks = run_head_sharded(args, shape, rank, world)
            par = (f"heads x{world}, row-parallel fuse + "
                   + ("NCCL reduce-scatter" if args.collective == "reduce_scatter"
                      else "fused GEMM + reduce-scatter over peer mappings"))
        if rank == 0:
            config.update({"global_batch": 1, "parallelism": par})
            print(json.dumps({
                "metric": METRIC, "value": shape.L / (ms / 1e3), "unit": "tokens/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": ms, "higher_is_better": True, "scaling": "strong",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": config,
                "gpu_launches": 7 * args.steps, "clocks": clocks}))
        torch.distributed.destroy_process_group()
        return
    if args.part == "vda_backward":
        ms, ms_saved = run_vda_backward(args, shape, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "VDA gradient pass ms (dq, dk, dv, dbeta, dalpha)",
                              "value": ms, "unit": "ms", "higher_is_better": False,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "dtype": "bf16", "data": "synthetic", "config": config,
                              "vda_backward": backward_row(work, peaks, ms, ms_saved)}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.part == "scan_sweep":
        rows = run_scan_sweep(args, rank, world, peaks)
        if rank == 0:
            print(json.dumps({"metric": "VDA branch ms and tokens/s over the scan-only sweep "
                                        "(prep, solve, both scans, read-out)",
                              "value": statistics.median(r["frac"] for r in rows),
                              "unit": "median fraction of roofline", "higher_is_better": True,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "dtype": "bf16 inputs, fp32 state", "data": "synthetic",
                              "config": {"workload": "vda_scan_sweep T{42,72,102} x "
                                                     "N{1008,4032} x d{64,128} x H{24,48}",
                                         "timing": "median of steps, CUDA events"},
                              "rows": rows}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.part == "window_mxfp8":
        ms, dev_rel = run_window_mxfp8(args, shape, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "MXFP8 window Softmax ms (q, k, v quantized inside)",
                              "value": ms, "unit": "ms", "higher_is_better": False,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "dtype": "mxfp8 (e4m3, ue8m0 / 32)", "data": "synthetic",
                              "config": config,
                              "window_mxfp8": window_mxfp8_row(work, peaks, ms, dev_rel)}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.part == "layer_mxfp8":
        ms, dev_rel = run_layer_mxfp8(args, shape, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "hybrid layer ms with both MXFP8 modes",
                              "value": ms, "unit": "ms", "higher_is_better": False,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "dtype": "mxfp8 (e4m3, ue8m0 / 32) products, fp32 VDA state",
                              "data": "synthetic", "config": config,
                              "layer_mxfp8": layer_mxfp8_row(shape, ms, dev_rel)}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    if args.part == "fuse_mxfp8":
        ms, dev_rel = run_fuse_mxfp8(args, shape, rank, world)
        if rank == 0:
            print(json.dumps({"metric": "MXFP8 fuse ms (both projection GEMMs in MXFP8)",
                              "value": ms, "unit": "ms", "higher_is_better": False,
                              "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                              "dtype": "mxfp8 (e4m3, ue8m0 / 32)", "data": "synthetic",
                              "config": config,
                              "fuse_mxfp8": mxfp8_row(work, peaks, ms, dev_rel)}))
        if world > 1:
            torch.distributed.destroy_process_group()
        return
    r = run_gpu(args, shape, rank, world)
    ms_step = r["ms"] / args.steps
    tokens_per_s = weak_scaling_value(world, shape.L, ms_step)
    win_tflops = work["softmax_flop"] / (r["win_ms"] / 1e3) / 1e12
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    traffic = None
    if os.path.exists(KERNEL_TRAFFIC_FILE):
        with open(KERNEL_TRAFFIC_FILE) as f:
            tr = json.load(f)
        # only counters taken on this workload and on these kernel sources
        if (tr.get("workload") == config["workload"] and
                tr.get("source_sha256") == window_source_hash()):
            traffic = tr.get("bytes_per_launch")
    # layer roofline: sum over steps of the binding resource at the measured peaks
    roof_ms = (work["softmax_flop"] / (peak * 1e12) + work["proj_flop"] / (peak * 1e12) +
               work["vda_bytes"] / (peaks["hbm_gbs"] * 1e9)) * 1e3
    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; q,k,v,x ~ N(0,1), k L2-normalised, beta = sigmoid(N), "
                "alpha ~ U(0.9,1), weights ~ N(0,0.02))",
        "config": config,
        "roofline": {"bound": "tensor", "achieved": win_tflops, "peak": peak, "unit": "TFLOP/s",
                     "frac": win_tflops / peak, "traffic": traffic,
                     "kernel": "window_attn_kernel<128> (window-and-anchor Softmax)",
                     "peak_source": f"{peak_kind} bf16_tflops_sustained",
                     "flop_per_launch": work["softmax_flop"], "ms_per_launch": r["win_ms"]},
        "layer_roofline": {"ms": roof_ms, "frac": roof_ms / ms_step,
                           "terms": "softmax + projections at sustained bf16 peak, VDA bytes "
                                    "at measured HBM"},
        "rows": {
            "window_softmax": {"ms": r["win_ms"], "bound": "tensor",
                               "frac": (work["softmax_flop"] / (peak * 1e12) * 1e3) / r["win_ms"]},
            "vda_prep_solve_scan_readout": {
                "ms": r["vda_ms"], "bound": "hbm + fp32 alu",
                "roofline_ms": (work["vda_bytes"] / (peaks["hbm_gbs"] * 1e9) +
                                work["vda_alu_flop"] / (FP32_TFLOPS * 1e12)) * 1e3,
                "frac": ((work["vda_bytes"] / (peaks["hbm_gbs"] * 1e9) +
                          work["vda_alu_flop"] / (FP32_TFLOPS * 1e12)) * 1e3) / r["vda_ms"]},
            "fuse_gemms": {"ms": r["fuse_ms"], "bound": "tensor",
                           "achieved_tflops": work["proj_flop"] / (r["fuse_ms"] / 1e3) / 1e12,
                           "frac": (work["proj_flop"] / (peak * 1e12) * 1e3) / r["fuse_ms"]},
            "fp32_peak_tflops": FP32_TFLOPS,
        },
        "e2e": {"value": weak_scaling_value(world, shape.L, r["e2e_ms"]), "unit": "tokens/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "ms_per_step": r["e2e_ms"]},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if args.part == "all":
        line["vda_by_solver"] = run_vda_solvers(args, shape, rank, world)
        line["vda_backward"] = backward_row(work, peaks,
                                            *run_vda_backward(args, shape, rank, world))
        line["fuse_mxfp8"] = mxfp8_row(work, peaks, *run_fuse_mxfp8(args, shape, rank, world))
        line["window_mxfp8"] = window_mxfp8_row(work, peaks,
                                                *run_window_mxfp8(args, shape, rank, world))
        line["layer_mxfp8"] = layer_mxfp8_row(shape, *run_layer_mxfp8(args, shape, rank, world))
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(shape)
        line["cpu_baseline"] = {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
