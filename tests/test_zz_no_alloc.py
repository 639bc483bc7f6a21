"""The allocation-free VDA entry point, vdn_vda_scan_static.

It is for callers that cannot allocate device memory (a plugin inside a
host framework that owns every device allocation, or a loop with a fixed
memory budget): its scratch is a fixed array of the library's own device
memory instead of a caller-provided workspace.  This test calls it through
the C ABI twice in a row, on different shapes and inputs, and compares each
result with the workspace entry point vdn_vda_scan at the tolerances the
parity tests use.  The file name makes pytest collect it last.
"""

import ctypes

import numpy as np
import pytest
import torch

from tests.parity_util import TOL_BF16, TOL_STATE, ensure_built, host, max_rel
from video_diffusion_hybrid_vda_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _static_call(vdn, shape, inp, out, states, status):
    s = vdn.Shape(shape.T, shape.N, shape.H, shape.d)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    return vdn.lib().vdn_vda_scan_static(
        ctypes.byref(s), p(inp["q"]), p(inp["k"]), p(inp["v"]), inp["q"].stride(0),
        p(inp["beta"]), p(inp["alpha"]), p(out), out.stride(0), p(states), p(status),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_static_matches_workspace_entry_point_twice(vdn):
    for shape, seed in ((synth.Shape(10, 300, 2, 128), 1), (synth.Shape(6, 77, 3, 64), 2)):
        inp = synth.make_inputs(shape, seed=seed, device="cuda")
        st_ref = torch.empty((2, shape.T, shape.H, shape.d, shape.d), device="cuda")
        o_ref, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                                 shape.T, shape.N, shape.H, shape.d, states=st_ref)
        assert vdn.get_device_status(ws) == 0
        out = torch.full((shape.L, shape.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        states = torch.full_like(st_ref, float("nan"))
        status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        assert _static_call(vdn, shape, inp, out, states, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert max_rel(host(out), host(o_ref)) <= TOL_BF16
        for t in range(shape.T):
            for h in range(shape.H):
                for dr in range(2):
                    assert max_rel(host(states[dr, t, h]), host(st_ref[dr, t, h])) <= TOL_STATE


def test_static_rejects_shapes_beyond_its_scratch(vdn):
    shape = synth.Shape(102, 8, 24, 128)          # needs ~940 MB of scratch
    t = torch.zeros((shape.L, shape.D), dtype=torch.bfloat16, device="cuda")
    f = torch.zeros((shape.L, shape.H), dtype=torch.float32, device="cuda")
    inp = {"q": t, "k": t, "v": t, "beta": f, "alpha": f}
    st = torch.zeros(1, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert _static_call(vdn, shape, inp, t, st, status) == 3   # VDN_ERR_WORKSPACE
