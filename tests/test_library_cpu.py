"""libvdn on the CPU side: it builds for sm_100a, loads, exports every symbol
include/vdn.h declares, and rejects bad arguments on the host before any
CUDA call (so these run without a GPU)."""

import ctypes
import os
import re

import pytest

from tests.parity_util import ensure_built

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn
    return vdn


def _header():
    with open(os.path.join(ROOT, "include", "vdn.h"), encoding="utf-8") as f:
        return f.read()


def _declared():
    src = _header()
    return sorted(set(re.findall(r"^VDN_API\s+[\w\s\*]+?\b(vdn_\w+)\s*\(", src, re.M)))


def _declared_param_counts():
    """Number of parameters of every VDN_API function in include/vdn.h."""
    src = _header()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    out = {}
    for m in re.finditer(r"VDN_API\s+[\w\s\*]+?\b(vdn_\w+)\s*\(([^)]*)\)", src):
        params = m.group(2).strip()
        out[m.group(1)] = 0 if params in ("", "void") else params.count(",") + 1
    return out


def test_binding_argument_counts_match_the_header(L):
    """Every ctypes prototype in the binding has as many arguments as the C
    declaration (a mismatch would pass wrong values at call time)."""
    lib = L.lib()
    counts = _declared_param_counts()
    assert sorted(counts) == _declared()
    for name, n in counts.items():
        fn = getattr(lib, name)
        assert fn.argtypes is not None, name
        assert len(fn.argtypes) == n, (name, len(fn.argtypes), n)


def test_exports_every_declared_symbol(L):
    names = _declared()
    assert len(names) >= 12
    lib = L.lib()
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(L.EXPORTS) == names


def test_status_strings(L):
    for code in range(8):
        assert L.status_string(code)
    assert "unknown" in L.status_string(99)
    assert "sm_100a" in L.version()


def test_workspace_queries(L):
    lib = L.lib()
    s = L.Shape(102, 4032, 24, 128)
    mat = 102 * 24 * 128 * 128 * 4
    # [status][A][B][P][states x2]; the gradient pass adds one matrix (G, then E)
    assert lib.vdn_vda_scan_workspace(ctypes.byref(s)) == 256 + 5 * mat
    assert lib.vdn_vda_backward_workspace(ctypes.byref(s)) == 256 + 6 * mat
    assert lib.vdn_vda_backward_workspace(None) == 0
    assert lib.vdn_vda_scan_workspace(None) == 0
    assert lib.vdn_vda_scan_workspace(ctypes.byref(L.Shape(0, 1, 1, 64))) == 0
    assert lib.vdn_hybrid_fuse_workspace(411264, 3072, 24) == 256 + 411264 * 2 * 3072 * 2
    # hidden 16 = 1 head x 16 runs on one head padded to 256 columns
    assert lib.vdn_hybrid_fuse_workspace(160, 16, 1) > 160 * 2 * 256 * 2
    assert lib.vdn_hybrid_fuse_workspace(160, 16, 3) == 0


def _scan(L, shape, q=16, k=16, v=16, ld=128, beta=16, alpha=16, o=16, ld_o=128, states=None,
          ws=256, ws_bytes=1 << 40):
    lib = L.lib()
    P = ctypes.c_void_p
    return lib.vdn_vda_scan(ctypes.byref(shape) if shape is not None else None,
                            P(q), P(k), P(v), ld, P(beta), P(alpha), P(o), ld_o,
                            P(states) if states else None, P(ws), ws_bytes, None)


def test_vda_scan_rejects_bad_arguments_on_host(L):
    ok = L.Shape(4, 8, 1, 128)
    assert _scan(L, None) == 1
    assert _scan(L, L.Shape(0, 8, 1, 128)) == 1
    assert _scan(L, L.Shape(4, 8, 1, 96)) == 2                 # unsupported head dim
    assert _scan(L, L.Shape(4, 8, 1, 48)) == 2
    assert _scan(L, ok, q=0) == 1                              # null pointer
    assert _scan(L, ok, k=24) == 1                             # misaligned
    assert _scan(L, ok, ld=100) == 1                           # ld % 8
    assert _scan(L, ok, ld=64) == 1                            # ld < D
    assert _scan(L, ok, ld_o=120) == 1
    assert _scan(L, ok, ws=0) == 3                             # no workspace
    assert _scan(L, ok, ws=128) == 3                           # misaligned workspace
    assert _scan(L, ok, ws_bytes=1024) == 3                    # too small


def test_window_and_fuse_reject_bad_arguments_on_host(L):
    lib = L.lib()
    P = ctypes.c_void_p
    s = L.Shape(10, 16, 1, 128)
    r = lib.vdn_window_attn(ctypes.byref(s), None, P(16), P(16), 128, 5, 1, 3, 0.0, P(16), 128,
                            None, P(256), 1 << 30, None)
    assert r in (1, 2)
    r = lib.vdn_hybrid_fuse(16, 128, 1, None, P(16), P(16), P(16), P(16), P(16), 1e-6, P(16),
                            P(16), P(16), P(256), 1 << 30, None)
    assert r in (1, 2)


def test_gradient_and_mxfp8_entry_points_reject_bad_arguments_on_host(L):
    """Every refusal below happens before any CUDA call (no GPU here): the
    pointers are aligned or misaligned fake addresses that are never read."""
    lib = L.lib()
    P = ctypes.c_void_p
    FP = ctypes.c_void_p
    A = 4096  # a 16-byte (and 256-byte) aligned stand-in address

    def bwd(shape, q=A, ld=128, ld_g=128, dbeta=A, ws=A, ws_bytes=1 << 40):
        return lib.vdn_vda_backward(ctypes.byref(shape) if shape is not None else None,
                                    P(q), P(A), P(A), ld, FP(A), FP(A), P(A), 128, P(A), P(A),
                                    P(A), ld_g, FP(dbeta), FP(A), 0, P(ws), ws_bytes, None)

    ok = L.Shape(4, 8, 1, 128)
    assert bwd(None) == 1
    assert bwd(L.Shape(4, 8, 1, 96)) == 2                  # head dim
    assert bwd(ok, q=0) == 1                               # null
    assert bwd(ok, q=A + 8) == 1                           # misaligned activation
    assert bwd(ok, dbeta=A + 2) == 1                       # misaligned fp32 output
    assert bwd(ok, ld=100) == 1
    assert bwd(ok, ld_g=120) == 1
    assert bwd(ok, ws=0) == 3
    assert bwd(ok, ws_bytes=1024) == 3

    q = lib.vdn_mxfp8_quantize
    assert q(None, 4, 128, 128, P(A), P(A), None) == 1
    assert q(P(A), 4, 96, 96, P(A), P(A), None) == 1       # cols not a multiple of 128
    assert q(P(A), 0, 128, 128, P(A), P(A), None) == 1
    assert q(P(A + 4), 4, 128, 128, P(A), P(A), None) == 1

    g = lib.vdn_gemm_mxfp8
    assert g(0, 32, 128, P(A), P(A), P(A), P(A), P(A), 0, P(A), 256, None) == 1
    assert g(128, 32, 96, P(A), P(A), P(A), P(A), P(A), 0, P(A), 256, None) == 2   # K % 128
    assert g(128, 40, 128, P(A), P(A), P(A), P(A), P(A), 0, P(A), 256, None) == 2  # N % 32
    assert g(128, 32, 128, P(A + 8), P(A), P(A), P(A), P(A), 0, P(A), 256, None) == 1
    assert g(128, 32, 128, P(A), P(A), P(A), P(A), P(A), 0, None, 256, None) == 3

    f = lib.vdn_hybrid_fuse_mxfp8
    args = [P(A)] * 5
    assert f(16, 3072, 25, *args, FP(A), 1e-6, P(A), P(A), P(A), P(A), 1 << 40, None) == 1
    assert f(16, 3072, 24, None, *args[1:], FP(A), 1e-6, P(A), P(A), P(A), P(A), 1 << 40,
             None) == 1
    assert f(16, 3000, 24, *args, FP(A), 1e-6, P(A), P(A), P(A), P(A), 1 << 40, None) == 2
    assert f(16, 3072, 24, *args, FP(A), 1e-6, P(A), P(A), P(A), None, 1 << 40, None) == 3

    rs = lib.vdn_hybrid_fuse_shard_rs
    owners = (ctypes.c_void_p * 9)(*([A] * 9))
    common = [P(A), P(A), P(A), 128, P(A), P(A), FP(A), 1e-6, P(A), P(A)]
    assert rs(16, 128, 1, 128, 0, *common, None, 2, P(A), 1 << 40, None) == 1
    assert rs(16, 128, 1, 128, 0, *common, owners, 9, P(A), 1 << 40, None) == 1  # G > 8
    assert rs(16, 128, 1, 128, 0, *common, owners, 0, P(A), 1 << 40, None) == 1
    bad = (ctypes.c_void_p * 2)(A, A + 4)
    assert rs(16, 128, 1, 128, 0, *common, bad, 2, P(A), 1 << 40, None) == 1


def test_window_context_entry_rejects_bad_arguments_on_host(L):
    lib = L.lib()
    P = ctypes.c_void_p
    A = 4096
    s = L.Shape(10, 16, 1, 128)

    def ctx(m_ctx=4, ck=A, ld_ctx=128, cf=5, wc=1, anchors=3, ws=A):
        return lib.vdn_window_attn_ctx(ctypes.byref(s), P(A), P(A), P(A), 128, P(ck), P(A),
                                       ld_ctx, m_ctx, cf, wc, anchors, 0.0, P(A), 128, None,
                                       P(ws), 1 << 30, None)

    assert ctx(m_ctx=-1) == 1
    assert ctx(ck=0) == 1                                   # context keys missing
    assert ctx(ck=A + 8) == 1
    assert ctx(ld_ctx=100) == 1
    assert ctx(cf=0) == 1
    assert ctx(wc=-1) == 1
    assert ctx(anchors=4) == 1
    assert ctx(ws=0) == 3


def test_window_mxfp8_rejects_bad_arguments_on_host(L):
    """Validation before any CUDA call: null pointers, head dims other than
    128, tokens per frame not a multiple of 32, a missing workspace."""
    import ctypes
    lib = L.lib()
    P = lambda a: ctypes.c_void_p(a)
    f = lib.vdn_window_attn_mxfp8
    sh = L.Shape(4, 64, 2, 128)
    assert f(ctypes.byref(sh), None, P(16), P(16), 256, 5, 1, 3, 0.0, P(16), 256, None, P(256),
             1 << 30, None) == 1
    sh_d = L.Shape(4, 64, 2, 64)
    assert f(ctypes.byref(sh_d), P(16), P(16), P(16), 128, 5, 1, 3, 0.0, P(16), 128, None,
             P(256), 1 << 30, None) == 2
    sh_n = L.Shape(4, 40, 2, 128)
    assert f(ctypes.byref(sh_n), P(16), P(16), P(16), 256, 5, 1, 3, 0.0, P(16), 256, None,
             P(256), 1 << 30, None) == 2
    assert f(ctypes.byref(sh), P(16), P(16), P(16), 256, 5, 1, 3, 0.0, P(16), 256, None,
             None, 0, None) == 3
    assert lib.vdn_window_attn_mxfp8_workspace(ctypes.byref(sh)) == \
        256 + 3 * 256 * 256 + 2 * 256 * 8 + 8 * 256


def test_release_library_has_no_bounds_checks(L):
    assert L.debug_bounds_enabled() is False


def test_debug_bounds_variant_builds_and_reports_itself():
    """The VDN_DEBUG_BOUNDS=1 variant (libvdn_debug.so) cross-compiles for
    sm_100a and says so; its checks run on the GPU (test_debug_bounds_gpu)."""
    from video_diffusion_hybrid_vda_b200 import build
    path = build.build(debug_bounds=True)
    dbg = ctypes.CDLL(path)
    dbg.vdn_debug_bounds_enabled.restype = ctypes.c_int
    assert dbg.vdn_debug_bounds_enabled() == 1
