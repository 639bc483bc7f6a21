"""The allocation-free VDA entry point, vdn_vda_scan_static.

It is for callers that cannot allocate device memory (a plugin inside a
host framework that owns every device allocation, or a loop with a fixed
memory budget): its scratch is a fixed array of the library's own device
memory instead of a caller-provided workspace.  These tests call it through
the C ABI several times in a row, on different shapes, head dims and inputs,
and compare each result with the workspace entry point vdn_vda_scan and with
the float64 oracle, at the tolerances the parity tests use.  The file name
makes pytest collect it last.
"""

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


# (shape, seed): head dims 128 and 64 run directly, 32 and 16 on padded
# copies inside the scratch array
CASES = ((synth.Shape(10, 300, 2, 128), 1), (synth.Shape(6, 77, 3, 64), 2),
         (synth.Shape(7, 50, 2, 32), 3), (synth.Shape(5, 33, 3, 16), 4))


def test_static_matches_workspace_entry_point_and_oracle(vdn):
    import oracle
    for shape, seed in CASES:
        inp = synth.make_inputs(shape, seed=seed, device="cuda")
        st_ref = torch.empty((2, shape.T, shape.H, shape.d, shape.d), device="cuda")
        o_ref, ws = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                                 shape.T, shape.N, shape.H, shape.d, states=st_ref)
        assert vdn.get_device_status(ws) == 0
        out = torch.full((shape.L, shape.D), float("nan"), dtype=torch.bfloat16, device="cuda")
        states = torch.full_like(st_ref, float("nan"))
        status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
        vdn.vda_scan_static(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], shape.T,
                            shape.N, shape.H, shape.d, out=out, states=states, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        # against the workspace entry point: the same kernels on the same
        # inputs, so the results agree far inside the parity tolerances
        assert max_rel(host(out), host(o_ref)) <= TOL_BF16
        for t in range(shape.T):
            for h in range(shape.H):
                for dr in range(2):
                    assert max_rel(host(states[dr, t, h]), host(st_ref[dr, t, h])) <= TOL_STATE
        # against the oracle
        x = {kk: host(vv).astype(np.float64) for kk, vv in inp.items()}
        o_or, S_f, S_b = oracle.vda(x["q"], x["k"], x["v"], x["beta"], x["alpha"], shape.T,
                                    shape.N, shape.H, shape.d)
        for h in range(shape.H):
            c = slice(h * shape.d, (h + 1) * shape.d)
            assert max_rel(host(out)[:, c], o_or[:, c]) <= TOL_BF16
            for t in range(shape.T):
                assert max_rel(host(states[0, t, h]), S_f[t, h]) <= TOL_STATE
                assert max_rel(host(states[1, t, h]), S_b[t, h]) <= TOL_STATE


def test_static_reports_a_numeric_failure_and_recovers(vdn):
    """A NaN in beta (made on the host) makes the solve's pivots NaN: the
    call's status reads bit 0; the next clean call on the same array reads 0
    (each call clears the status word it uses)."""
    shape = synth.Shape(4, 40, 2, 64)
    inp = synth.make_inputs(shape, seed=9, device="cuda")
    bad = inp["beta"].clone()
    bad[45, 1] = float("nan")
    _, status = vdn.vda_scan_static(inp["q"], inp["k"], inp["v"], bad, inp["alpha"], shape.T,
                                    shape.N, shape.H, shape.d)
    torch.cuda.synchronize()
    assert int(status.item()) & 1
    out, status = vdn.vda_scan_static(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"],
                                      shape.T, shape.N, shape.H, shape.d)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    o_ref, _ = vdn.vda_scan(inp["q"], inp["k"], inp["v"], inp["beta"], inp["alpha"], shape.T,
                            shape.N, shape.H, shape.d)
    assert max_rel(host(out), host(o_ref)) <= TOL_BF16


def test_static_rejects_shapes_beyond_its_scratch(vdn):
    shape = synth.Shape(102, 8, 24, 128)          # needs ~940 MB of scratch
    t = torch.zeros((shape.L, shape.D), dtype=torch.bfloat16, device="cuda")
    f = torch.zeros((shape.L, shape.H), dtype=torch.float32, device="cuda")
    with pytest.raises(vdn.VdnError) as e:
        vdn.vda_scan_static(t, t, t, f, f, shape.T, shape.N, shape.H, shape.d)
    assert e.value.code == 3                      # VDN_ERR_WORKSPACE
