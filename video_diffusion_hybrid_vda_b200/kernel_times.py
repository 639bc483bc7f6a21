"""Device time of each libvdn kernel in the VDA forward or gradient pass.

    python -m video_diffusion_hybrid_vda_b200.kernel_times --part vda_forward
    python -m video_diffusion_hybrid_vda_b200.kernel_times --part vda_backward
    python -m video_diffusion_hybrid_vda_b200.kernel_times --part window

Runs the pass on seeded synthetic inputs (102 latent frames x 4032 tokens x
24 heads x 128 unless given), three untimed passes, then ``--passes`` passes
under torch.profiler (CUPTI kernel records, no replay: the kernels run as
they do in the layer), writing 256 MB between passes so each starts with a
cold L2.  Prints one JSON line: per kernel, its mean device time per pass
in ms.  ``--part window`` runs the window Softmax alone, timed with CUDA
events (no profiler, so a counter capture can wrap it).
"""

import argparse
import json
import re

import torch
from torch.profiler import ProfilerActivity, profile

from . import synth, vdn


def kernel_name(name):
    m = (re.search(r"(vda_\w+?_kernel)<([^>]*)>", name) or
         re.search(r"(vda_\w+?_kernel)", name))
    return m.group(0) if m else None


def window_only(s, inp, passes):
    """The window Softmax alone (3 warm-up launches, then ``passes`` timed
    ones with CUDA events; q, k, v and o are the only large buffers), for
    counter captures of that one kernel at a given shape."""
    o = torch.empty((s.L, s.D), dtype=torch.bfloat16, device="cuda")
    ws = vdn.alloc_workspace(vdn.window_attn_workspace(s.T, s.N, s.H, s.d))

    def run():
        vdn.window_attn(inp["q"], inp["k"], inp["v"], s.T, s.N, s.H, s.d, out=o, ws=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(passes):
        run()
    e1.record()
    torch.cuda.synchronize()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the timed launches: %d" % vdn.get_device_status(ws))
    print(json.dumps({"part": "window", "shape": [s.T, s.N, s.H, s.d], "passes": passes,
                      "ms_per_launch": round(e0.elapsed_time(e1) / max(passes, 1), 4)}))


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--part", choices=["vda_forward", "vda_backward", "window"],
                    default="vda_forward")
    ap.add_argument("--shape", type=int, nargs=4, default=[102, 4032, 24, 128],
                    metavar=("T", "N", "H", "d"))
    ap.add_argument("--passes", type=int, default=5)
    ap.add_argument("--lib", default=None, help="path of a libvdn.so other than the in-tree one")
    ap.add_argument("--solver", choices=["gauss-jordan", "cholesky"], default="gauss-jordan")
    args = ap.parse_args(argv)
    if args.lib:
        vdn.LIB_PATH = args.lib
    vdn.set_vda_solver(vdn.SOLVER_GAUSS_JORDAN if args.solver == "gauss-jordan"
                       else vdn.SOLVER_CHOLESKY)
    s = synth.Shape(*args.shape)
    inp = synth.make_inputs(s, seed=0, device="cuda")
    if args.part == "window":
        window_only(s, inp, args.passes)
        return
    if args.part == "vda_forward":
        ws = vdn.alloc_workspace(vdn.vda_scan_workspace(s.T, s.N, s.H, s.d))

        def run():
            vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                         s.T, s.N, s.H, s.d, ws=ws)
    else:
        g = torch.Generator(device="cuda")
        g.manual_seed(7)
        d_o = torch.randn((s.L, s.D), generator=g, device="cuda").to(torch.bfloat16)
        ws = vdn.alloc_workspace(vdn.vda_backward_workspace(s.T, s.N, s.H, s.d))

        def run():
            vdn.vda_backward(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], d_o,
                             s.T, s.N, s.H, s.d, ws=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(args.passes):
            flush.fill_(1)
            run()
        torch.cuda.synchronize()
    if vdn.get_device_status(ws) != 0:
        raise RuntimeError("device status after the timed passes: %d" % vdn.get_device_status(ws))
    per = {}
    for e in prof.events():
        if e.device_type.name != "CUDA":
            continue
        n = kernel_name(e.name)
        if n is not None:
            per[n] = per.get(n, 0.0) + e.device_time_total / 1000.0
    out = {k: round(v / args.passes, 4) for k, v in per.items()}
    print(json.dumps({"part": args.part, "shape": args.shape, "solver": args.solver,
                      "passes": args.passes,
                      "ms_per_pass": out, "sum_ms": round(sum(out.values()), 4)}))


if __name__ == "__main__":
    main()
