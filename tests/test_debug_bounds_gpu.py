"""The bounds-checking debug build (libvdn_debug.so, VDN_DEBUG_BOUNDS=1) on
the GPU: its self-test records VDN_ERR_BOUNDS for an index outside its
tensor and nothing for one inside, and the window Softmax, the VDA scan and
gradient pass, and the fuse (plain and reduce-scatter form) run with a
clean status word and give outputs bit-identical to the release library's
(the checks change no arithmetic).  The debug library runs in a child
process, since one process loads one libvdn."""

import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

from tests.parity_util import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu

_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, {root!r})
from video_diffusion_hybrid_vda_b200 import vdn, synth
if {debug}:
    vdn.LIB_PATH = {lib!r}
out = {{}}
st = []
s = synth.Shape(12, 96, 2, 128)
x = synth.make_inputs(s, seed=7, device="cuda", with_fuse=True)
o, ws = vdn.window_attn(x["q"], x["k"], x["v"], s.T, s.N, s.H, s.d)
out["o_s"] = o; st.append(vdn.get_device_status(ws))
o2, ws2 = vdn.vda_scan(x["q"], x["k"], x["v"], x["beta"], x["alpha"], s.T, s.N, s.H, s.d)
out["o_vda"] = o2; st.append(vdn.get_device_status(ws2))
g = torch.Generator(device="cuda"); g.manual_seed(3)
d_o = torch.randn((s.L, s.D), generator=g, device="cuda").to(torch.bfloat16)
*grads, wsb = vdn.vda_backward(x["q"], x["k"], x["v"], x["beta"], x["alpha"], d_o, s.T, s.N, s.H, s.d)
for i, t in enumerate(grads):
    out["grad%d" % i] = t
st.append(vdn.get_device_status(wsb))
y, wsf = vdn.hybrid_fuse(x["x"], o, o2, x["W_gs"], x["W_gl"], x["gamma"], x["W_os"], x["W_ol"], s.H)
out["y"] = y; st.append(vdn.get_device_status(wsf))
owner = torch.zeros((s.L, s.D), dtype=torch.float32, device="cuda")
wss = vdn.alloc_workspace(int(vdn.lib().vdn_hybrid_fuse_shard_workspace(s.L, s.D, s.H, s.d)))
vdn.hybrid_fuse_shard_rs(x["x"], o, o2, x["W_gs"], x["W_gl"], x["gamma"], x["W_os"], x["W_ol"], s.d, 0, [owner], ws=wss)
out["y_rs"] = owner; st.append(vdn.get_device_status(wss))
torch.cuda.synchronize()
np.savez({path!r}, **{{k: v.float().cpu().numpy() for k, v in out.items()}},
         status=np.array(st), enabled=np.array(int(vdn.debug_bounds_enabled())))
"""


def _run(debug, lib, path):
    code = _CHILD.format(root=ROOT, debug=bool(debug), lib=lib, path=path)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    return np.load(path)


@pytest.fixture(scope="module")
def debug_lib():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import build
    return build.build(debug_bounds=True)


def test_debug_build_selftest_records_out_of_range(debug_lib, tmp_path):
    code = r"""
import sys, torch
sys.path.insert(0, {root!r})
from video_diffusion_hybrid_vda_b200 import vdn
vdn.LIB_PATH = {lib!r}
assert vdn.debug_bounds_enabled()
ws = vdn.alloc_workspace(256)
vdn.selftest_bounds(ws, 5, 10, 0, 128, 3072)          # inside
assert vdn.get_device_status(ws) == 0
vdn.selftest_bounds(ws, 10, 10, 0, 128, 3072)         # row == rows
assert vdn.get_device_status(ws) == 7
vdn.reset_device_status(ws)
vdn.selftest_bounds(ws, 0, 10, 3000, 128, 3072)       # columns past the width
assert vdn.get_device_status(ws) == 7
vdn.reset_device_status(ws)
vdn.selftest_bounds(ws, -1, 10, 0, 8, 64)             # negative row
assert vdn.get_device_status(ws) == 7
print("ok")
""".format(root=ROOT, lib=debug_lib)
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and "ok" in r.stdout, r.stderr[-3000:]


def test_release_build_selftest_records_nothing():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn
    ws = vdn.alloc_workspace(256)
    vdn.selftest_bounds(ws, 10, 10, 0, 128, 3072)
    assert vdn.get_device_status(ws) == 0


def test_debug_build_matches_release_with_clean_status(debug_lib, tmp_path):
    rel = _run(False, debug_lib, str(tmp_path / "rel.npz"))
    dbg = _run(True, debug_lib, str(tmp_path / "dbg.npz"))
    assert int(rel["enabled"]) == 0 and int(dbg["enabled"]) == 1
    assert list(dbg["status"]) == [0] * len(dbg["status"])
    assert list(rel["status"]) == [0] * len(rel["status"])
    for k in rel.files:
        if k in ("status", "enabled"):
            continue
        assert np.array_equal(rel[k], dbg[k]), k
