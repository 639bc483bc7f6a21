"""ctypes binding over libvdn.so (declared in include/vdn.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels.  Tensors must live on the current CUDA device; PyTorch provides
device memory and the stream.  If the library is missing, every call raises
(there is no CPU fallback).
"""

import ctypes
import functools
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvdn.so")

VDN_OK = 0
STATUS_NAMES = {0: "VDN_OK", 1: "VDN_ERR_INVALID_ARG", 2: "VDN_ERR_UNSUPPORTED",
                3: "VDN_ERR_WORKSPACE", 4: "VDN_ERR_CUDA", 5: "VDN_ERR_NUMERIC",
                6: "VDN_ERR_TIMEOUT", 7: "VDN_ERR_BOUNDS"}

# every symbol include/vdn.h declares
EXPORTS = ["vdn_vda_scan_workspace", "vdn_vda_scan", "vdn_vda_debug_buffers",
           "vdn_window_attn_workspace", "vdn_window_attn", "vdn_hybrid_fuse_workspace",
           "vdn_hybrid_fuse", "vdn_status_string", "vdn_get_device_status",
           "vdn_reset_device_status", "vdn_set_wait_budget_ns", "vdn_version",
           "vdn_vda_scan_static", "vdn_selftest_exp2", "vdn_window_attn_ctx",
           "vdn_set_vda_solver", "vdn_hybrid_fuse_shard_workspace", "vdn_hybrid_fuse_shard",
           "vdn_vda_backward_workspace", "vdn_vda_backward", "vdn_vda_backward_debug_buffers",
           "vdn_mxfp8_scale_bytes", "vdn_mxfp8_quantize", "vdn_gemm_mxfp8",
           "vdn_hybrid_fuse_mxfp8_workspace", "vdn_hybrid_fuse_mxfp8",
           "vdn_hybrid_fuse_shard_rs", "vdn_window_attn_schedule",
           "vdn_window_attn_mxfp8_workspace", "vdn_window_attn_mxfp8", "vdn_copy2d_async",
           "vdn_debug_bounds_enabled", "vdn_selftest_bounds"]

SOLVER_CHOLESKY = 0
SOLVER_GAUSS_JORDAN = 1
SOLVER_DEFAULT = SOLVER_GAUSS_JORDAN


class VdnError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(code, code)} ({status_string(code)})")


class Shape(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int),
                ("d", ctypes.c_int)]


_lib = None
_P = ctypes.c_void_p
_FP = ctypes.POINTER(ctypes.c_float)
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


def lib():
    """Load libvdn.so once; raise if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"libvdn.so not found at {LIB_PATH}; build it with "
                           "`python -m video_diffusion_hybrid_vda_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    S = ctypes.POINTER(Shape)
    L.vdn_vda_scan_workspace.argtypes = [S]
    L.vdn_vda_scan_workspace.restype = _SZ
    L.vdn_debug_bounds_enabled.argtypes = []
    L.vdn_debug_bounds_enabled.restype = ctypes.c_int
    L.vdn_selftest_bounds.argtypes = [_P, _I64, _I64, _I64, _I64, _I64, _P]
    L.vdn_selftest_bounds.restype = ctypes.c_int
    L.vdn_vda_scan.argtypes = [S, _P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _SZ, _P]
    L.vdn_vda_scan.restype = ctypes.c_int
    L.vdn_vda_debug_buffers.argtypes = [S, _P] + [ctypes.POINTER(_P)] * 3
    L.vdn_vda_debug_buffers.restype = ctypes.c_int
    L.vdn_window_attn_workspace.argtypes = [S]
    L.vdn_window_attn_workspace.restype = _SZ
    L.vdn_window_attn.argtypes = [S, _P, _P, _P, _I64, ctypes.c_int, ctypes.c_int,
                                  ctypes.c_uint, ctypes.c_float, _P, _I64, _P, _P, _SZ, _P]
    L.vdn_window_attn.restype = ctypes.c_int
    L.vdn_window_attn_ctx.argtypes = [S, _P, _P, _P, _I64, _P, _P, _I64, ctypes.c_int,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_uint, ctypes.c_float,
                                      _P, _I64, _P, _P, _SZ, _P]
    L.vdn_window_attn_ctx.restype = ctypes.c_int
    L.vdn_window_attn_schedule.argtypes = [S, ctypes.c_int, ctypes.c_int, ctypes.c_uint,
                                           ctypes.POINTER(ctypes.c_int), ctypes.c_int,
                                           ctypes.POINTER(ctypes.c_int)]
    L.vdn_window_attn_schedule.restype = ctypes.c_int
    L.vdn_hybrid_fuse_workspace.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int]
    L.vdn_hybrid_fuse_workspace.restype = _SZ
    L.vdn_hybrid_fuse.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, _P, _P, _P, _P, _P,
                                  _P, ctypes.c_float, _P, _P, _P, _P, _SZ, _P]
    L.vdn_hybrid_fuse.restype = ctypes.c_int
    L.vdn_status_string.argtypes = [ctypes.c_int]
    L.vdn_status_string.restype = ctypes.c_char_p
    L.vdn_get_device_status.argtypes = [_P, _P]
    L.vdn_get_device_status.restype = ctypes.c_int
    L.vdn_reset_device_status.argtypes = [_P, _P]
    L.vdn_reset_device_status.restype = ctypes.c_int
    L.vdn_set_wait_budget_ns.argtypes = [ctypes.c_uint64]
    L.vdn_set_wait_budget_ns.restype = None
    L.vdn_selftest_exp2.argtypes = [_P, _P, _P, ctypes.c_int, _P]
    L.vdn_selftest_exp2.restype = ctypes.c_int
    L.vdn_hybrid_fuse_shard_workspace.argtypes = [ctypes.c_int] * 4
    L.vdn_hybrid_fuse_shard_workspace.restype = _SZ
    L.vdn_hybrid_fuse_shard.argtypes = [ctypes.c_int] * 5 + [_P, _P, _P, _I64, _P, _P, _P,
                                                             ctypes.c_float, _P, _P, _P, _P, _SZ, _P]
    L.vdn_hybrid_fuse_shard.restype = ctypes.c_int
    L.vdn_hybrid_fuse_shard_rs.argtypes = [ctypes.c_int] * 5 + [_P, _P, _P, _I64, _P, _P, _P,
                                                                ctypes.c_float, _P, _P,
                                                                ctypes.POINTER(_P), ctypes.c_int,
                                                                _P, _SZ, _P]
    L.vdn_hybrid_fuse_shard_rs.restype = ctypes.c_int
    L.vdn_set_vda_solver.argtypes = [ctypes.c_int]
    L.vdn_set_vda_solver.restype = ctypes.c_int
    L.vdn_vda_backward_workspace.argtypes = [S]
    L.vdn_vda_backward_workspace.restype = _SZ
    L.vdn_vda_backward.argtypes = [S, _P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _P, _I64, _P,
                                   _P, ctypes.c_int, _P, _SZ, _P]
    L.vdn_vda_backward.restype = ctypes.c_int
    L.vdn_vda_backward_debug_buffers.argtypes = [S, _P] + [ctypes.POINTER(_P)] * 3
    L.vdn_vda_backward_debug_buffers.restype = ctypes.c_int
    L.vdn_vda_scan_static.argtypes = [S, _P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _P]
    L.vdn_vda_scan_static.restype = ctypes.c_int
    L.vdn_mxfp8_scale_bytes.argtypes = [_I64, _I64]
    L.vdn_mxfp8_scale_bytes.restype = _SZ
    L.vdn_mxfp8_quantize.argtypes = [_P, _I64, _I64, _I64, _P, _P, _P]
    L.vdn_mxfp8_quantize.restype = ctypes.c_int
    L.vdn_gemm_mxfp8.argtypes = [ctypes.c_int] * 3 + [_P] * 5 + [ctypes.c_int, _P, _SZ, _P]
    L.vdn_gemm_mxfp8.restype = ctypes.c_int
    L.vdn_hybrid_fuse_mxfp8_workspace.argtypes = [ctypes.c_int] * 3
    L.vdn_hybrid_fuse_mxfp8_workspace.restype = _SZ
    L.vdn_hybrid_fuse_mxfp8.argtypes = [ctypes.c_int] * 3 + [_P] * 6 + [ctypes.c_float, _P, _P,
                                                                         _P, _P, _SZ, _P]
    L.vdn_hybrid_fuse_mxfp8.restype = ctypes.c_int
    L.vdn_window_attn_mxfp8_workspace.argtypes = [S]
    L.vdn_window_attn_mxfp8_workspace.restype = _SZ
    L.vdn_window_attn_mxfp8.argtypes = [S, _P, _P, _P, _I64, ctypes.c_int, ctypes.c_int,
                                        ctypes.c_uint, ctypes.c_float, _P, _I64, _P, _P, _SZ, _P]
    L.vdn_window_attn_mxfp8.restype = ctypes.c_int
    L.vdn_copy2d_async.argtypes = [_P, _SZ, _P, _SZ, _SZ, _SZ, _P]
    L.vdn_copy2d_async.restype = ctypes.c_int
    L.vdn_version.argtypes = []
    L.vdn_version.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(code):
    return lib().vdn_status_string(int(code)).decode()


def version():
    return lib().vdn_version().decode()


def _check(code, where):
    if code != VDN_OK:
        raise VdnError(code, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _shape(T, N, H, d):
    return Shape(int(T), int(N), int(H), int(d))


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libvdn takes CUDA tensors only")


def copy_columns_async(dst, dst_c0, src, src_c0, ncols, stream=None):
    """ncols columns of the row-major 2-D tensor src, from column src_c0, into
    dst from column dst_c0 (same row count and dtype; one of them pinned host
    memory, the other CUDA), as one pitched copy on ``stream``."""
    if dst.dim() != 2 or src.dim() != 2 or dst.shape[0] != src.shape[0] or \
            dst.dtype != src.dtype:
        raise ValueError("copy_columns_async: 2-D tensors with the same rows and dtype")
    if dst.stride(1) != 1 or src.stride(1) != 1 or dst_c0 + ncols > dst.shape[1] or \
            src_c0 + ncols > src.shape[1]:
        raise ValueError("copy_columns_async: contiguous rows holding the columns")
    e = dst.element_size()
    _check(lib().vdn_copy2d_async(ctypes.c_void_p(dst.data_ptr() + dst_c0 * e),
                                  dst.stride(0) * e,
                                  ctypes.c_void_p(src.data_ptr() + src_c0 * e),
                                  src.stride(0) * e, ncols * e, dst.shape[0], _stream(stream)),
           "vdn_copy2d_async")


def alloc_workspace(nbytes, device=None):
    """Device workspace with a cleared status word."""
    ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8,
                     device=device or torch.device("cuda"))
    _check(lib().vdn_reset_device_status(_ptr(ws), _stream(None)), "vdn_reset_device_status")
    return ws


def get_device_status(ws, stream=None):
    """Synchronise the stream and return the workspace status code (0 = ok)."""
    return lib().vdn_get_device_status(_ptr(ws), _stream(stream))


def reset_device_status(ws, stream=None):
    _check(lib().vdn_reset_device_status(_ptr(ws), _stream(stream)), "vdn_reset_device_status")


def set_wait_budget_ns(ns):
    lib().vdn_set_wait_budget_ns(int(ns))


def set_vda_solver(solver):
    """SOLVER_GAUSS_JORDAN (default) or SOLVER_CHOLESKY, process-wide."""
    _check(lib().vdn_set_vda_solver(int(solver)), "vdn_set_vda_solver")


def debug_bounds_enabled():
    """True if the loaded library checks store indices against their
    tensors on the device (built with VDN_DEBUG_BOUNDS=1)."""
    return bool(lib().vdn_debug_bounds_enabled())


def selftest_bounds(ws, r, rows, c, width, cols, stream=None):
    """One device-side bounds check of row r and columns [c, c + width)
    against a rows x cols tensor (no memory touched but ws's status word)."""
    _need_cuda(ws)
    _check(lib().vdn_selftest_bounds(_ptr(ws), int(r), int(rows), int(c), int(width), int(cols),
                                     _stream(stream)), "vdn_selftest_bounds")


def selftest_exp2(x, stream=None):
    """(y_fma, y_mufu): the Softmax's two exponential paths on fp32 CUDA x."""
    _need_cuda(x)
    y_fma, y_mufu = torch.empty_like(x), torch.empty_like(x)
    _check(lib().vdn_selftest_exp2(_ptr(x), _ptr(y_fma), _ptr(y_mufu), x.numel(),
                                   _stream(stream)), "vdn_selftest_exp2")
    return y_fma, y_mufu


# ---------------------------------------------------------------- VDA

def vda_scan_workspace(T, N, H, d):
    return int(lib().vdn_vda_scan_workspace(ctypes.byref(_shape(T, N, H, d))))


def vda_scan(q, k, v, beta, alpha, T, N, H, d, out=None, states=None, ws=None, stream=None):
    """Video Delta Attention: o_vda = (S_fwd_t + S_bwd_t) q per token.

    q, k, v: [T*N, ld] bf16; beta [T*N, H] fp32; alpha [T, H] fp32.
    Returns (o_vda, ws).  ``states`` (fp32 [2, T, H, d, d]) receives both
    scans' states when given.
    """
    _need_cuda(q, k, v, beta, alpha, out, states, ws)
    shape = _shape(T, N, H, d)
    if out is None:
        out = torch.empty((T * N, H * d), dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = alloc_workspace(vda_scan_workspace(T, N, H, d), q.device)
    code = lib().vdn_vda_scan(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), q.stride(0),
                              _ptr(beta), _ptr(alpha), _ptr(out), out.stride(0), _ptr(states),
                              _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "vdn_vda_scan")
    return out, ws


def vda_scan_static(q, k, v, beta, alpha, T, N, H, d, out=None, states=None, status=None,
                    stream=None):
    """vda_scan without a workspace (vdn_vda_scan_static): the library's fixed
    device scratch array serves instead, for callers that cannot allocate.
    Returns (o_vda, status) where ``status`` (int32 [1] on the device, or the
    tensor given) receives the call's device status bits.  Calls that overlap
    on the GPU share the array and race."""
    _need_cuda(q, k, v, beta, alpha, out, states, status)
    shape = _shape(T, N, H, d)
    if out is None:
        out = torch.empty((T * N, H * d), dtype=torch.bfloat16, device=q.device)
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device=q.device)
    code = lib().vdn_vda_scan_static(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), q.stride(0),
                                     _ptr(beta), _ptr(alpha), _ptr(out), out.stride(0),
                                     _ptr(states), _ptr(status), _stream(stream))
    _check(code, "vdn_vda_scan_static")
    return out, status


def vda_debug_buffers(ws, T, N, H, d):
    """(A, B, P) views into a VDA workspace, each fp32 [T, H, d, d]."""
    ptrs = [ctypes.c_void_p() for _ in range(3)]
    _check(lib().vdn_vda_debug_buffers(ctypes.byref(_shape(T, N, H, d)), _ptr(ws),
                                       *[ctypes.byref(p) for p in ptrs]), "vdn_vda_debug_buffers")
    base = ws.data_ptr()
    n = T * H * d * d
    flat = ws.view(torch.uint8)
    out = []
    for p in ptrs:
        off = p.value - base
        out.append(flat[off:off + 4 * n].view(torch.float32).view(T, H, d, d))
    return tuple(out)


def vda_backward_workspace(T, N, H, d):
    return int(lib().vdn_vda_backward_workspace(ctypes.byref(_shape(T, N, H, d))))


def vda_backward(q, k, v, beta, alpha, d_o, T, N, H, d, dq=None, dk=None, dv=None, dbeta=None,
                 dalpha=None, ws=None, stream=None, reuse_forward=False):
    """Gradients of o_vda with respect to q, k, v, beta and alpha, given
    d_o = dLoss/do_vda ([T*N, ld] bf16).  Returns (dq, dk, dv, dbeta, dalpha, ws):
    dq/dk/dv bf16 [T*N, H*d], dbeta fp32 [T*N, H], dalpha fp32 [T, H].
    reuse_forward: ``ws`` (of vda_backward_workspace size) last served a
    vda_scan on the same inputs without ``states``; its P and states are
    used instead of recomputing them."""
    _need_cuda(q, k, v, beta, alpha, d_o, dq, dk, dv, dbeta, dalpha, ws)
    shape = _shape(T, N, H, d)
    dev = q.device
    L, D = T * N, H * d
    dq = torch.empty((L, D), dtype=torch.bfloat16, device=dev) if dq is None else dq
    dk = torch.empty((L, D), dtype=torch.bfloat16, device=dev) if dk is None else dk
    dv = torch.empty((L, D), dtype=torch.bfloat16, device=dev) if dv is None else dv
    if not (dq.stride(0) == dk.stride(0) == dv.stride(0)):
        raise ValueError("dq, dk and dv must share one row stride")
    dbeta = torch.empty((L, H), dtype=torch.float32, device=dev) if dbeta is None else dbeta
    dalpha = torch.empty((T, H), dtype=torch.float32, device=dev) if dalpha is None else dalpha
    if ws is None:
        ws = alloc_workspace(vda_backward_workspace(T, N, H, d), dev)
    code = lib().vdn_vda_backward(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), q.stride(0),
                                  _ptr(beta), _ptr(alpha), _ptr(d_o), d_o.stride(0), _ptr(dq),
                                  _ptr(dk), _ptr(dv), dq.stride(0), _ptr(dbeta), _ptr(dalpha),
                                  int(bool(reuse_forward)), _ptr(ws), ws.numel(),
                                  _stream(stream))
    _check(code, "vdn_vda_backward")
    return dq, dk, dv, dbeta, dalpha, ws


def vda_backward_debug_buffers(ws, T, N, H, d):
    """(states [2,T,H,d',d'], adjoint states [2,T,H,d',d'], E [T,H,d',d']) views
    into a backward workspace; d' = 64 for head dims 16 and 32."""
    ptrs = [ctypes.c_void_p() for _ in range(3)]
    _check(lib().vdn_vda_backward_debug_buffers(ctypes.byref(_shape(T, N, H, d)), _ptr(ws),
                                                *[ctypes.byref(p) for p in ptrs]),
           "vdn_vda_backward_debug_buffers")
    dd = 64 if d in (16, 32) else d
    base = ws.data_ptr()
    flat = ws.view(torch.uint8)
    out = []
    for p, lead in zip(ptrs, (2, 2, 1)):
        n = lead * T * H * dd * dd
        off = p.value - base
        out.append(flat[off:off + 4 * n].view(torch.float32).view(lead, T, H, dd, dd))
    return out[0], out[1], out[2][0]


# ---------------------------------------------------------------- MXFP8

def mxfp8_scale_bytes(rows, cols):
    return int(lib().vdn_mxfp8_scale_bytes(int(rows), int(cols)))


def mxfp8_quantize(x, stream=None):
    """bf16 [R, K] (K a multiple of 128) -> (E4M3 codes uint8 [R, K], scale
    bytes uint8 in the GEMM's tile layout)."""
    _need_cuda(x)
    R, K = x.shape
    q = torch.empty((R, K), dtype=torch.uint8, device=x.device)
    sf = torch.empty(max(mxfp8_scale_bytes(R, K), 16), dtype=torch.uint8, device=x.device)
    _check(lib().vdn_mxfp8_quantize(_ptr(x), R, K, x.stride(0), _ptr(q), _ptr(sf), _stream(stream)),
           "vdn_mxfp8_quantize")
    return q, sf


def gemm_mxfp8(a, b, out_f32=False, ws=None, stream=None):
    """C = A B^T for MXFP8 operands a = (codes [M, K], scales), b = (codes [N, K], scales)."""
    (aq, asf), (bq, bsf) = a, b
    _need_cuda(aq, asf, bq, bsf)
    M, K = aq.shape
    N = bq.shape[0]
    c = torch.empty((M, N), dtype=torch.float32 if out_f32 else torch.bfloat16, device=aq.device)
    if ws is None:
        ws = alloc_workspace(256, aq.device)
    _check(lib().vdn_gemm_mxfp8(M, N, K, _ptr(aq), _ptr(asf), _ptr(bq), _ptr(bsf), _ptr(c),
                                int(bool(out_f32)), _ptr(ws), ws.numel(), _stream(stream)),
           "vdn_gemm_mxfp8")
    return c, ws


def mxfp8_fuse_weights(W_gs, W_gl, W_os, W_ol, stream=None):
    """MXFP8 weights of the fuse: the stacked gate weights [W_gs; W_gl] and
    the side-by-side output weights [W_os | W_ol], each (codes, scales)."""
    wg = mxfp8_quantize(torch.cat([W_gs, W_gl], dim=0).contiguous(), stream)
    wo = mxfp8_quantize(torch.cat([W_os, W_ol], dim=1).contiguous(), stream)
    return wg, wo


def hybrid_fuse_mxfp8(x, o_s, o_vda, wg, gamma, wo, H, eps=1e-6, out=None, ws=None, stream=None):
    """The fuse with MXFP8 projections (wg, wo from mxfp8_fuse_weights).
    Returns (y bf16 [L, D], ws)."""
    _need_cuda(x, o_s, o_vda, gamma, out, ws)
    L, D = x.shape
    if out is None:
        out = torch.empty((L, D), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = alloc_workspace(int(lib().vdn_hybrid_fuse_mxfp8_workspace(L, D, H)), x.device)
    _check(lib().vdn_hybrid_fuse_mxfp8(L, D, H, _ptr(x), _ptr(o_s), _ptr(o_vda), _ptr(wg[0]),
                                       _ptr(wg[1]), _ptr(gamma), float(eps), _ptr(wo[0]),
                                       _ptr(wo[1]), _ptr(out), _ptr(ws), ws.numel(),
                                       _stream(stream)),
           "vdn_hybrid_fuse_mxfp8")
    return out, ws


# ---------------------------------------------------------------- window Softmax

SCHEDULE_FIELDS = ("q0", "q1", "tile_base", "ntiles", "nint", "nkv")


def window_attn_schedule(T, N, chunk_frames=5, window_chunks=1, anchors=3):
    """The window Softmax's work plan (host only): a list of segments in
    launch order, each a dict with q0, q1, tile_base, ntiles, nint, nkv and
    'keys', the list of its key intervals (k0, k1)."""
    L = lib()
    shape = Shape(T, N, 1, 128)
    n = ctypes.c_int(0)
    code = L.vdn_window_attn_schedule(ctypes.byref(shape), chunk_frames, window_chunks, anchors,
                                      None, 0, ctypes.byref(n))
    if code not in (VDN_OK, 1) or (code == 1 and n.value == 0):
        _check(code, "vdn_window_attn_schedule")
    buf = (ctypes.c_int * (12 * max(n.value, 1)))()
    _check(L.vdn_window_attn_schedule(ctypes.byref(shape), chunk_frames, window_chunks, anchors,
                                      buf, n.value, ctypes.byref(n)), "vdn_window_attn_schedule")
    segs = []
    for g in range(n.value):
        row = buf[12 * g: 12 * g + 12]
        seg = dict(zip(SCHEDULE_FIELDS, row[:6]))
        seg["keys"] = [(row[6 + 2 * v], row[7 + 2 * v]) for v in range(seg["nint"])]
        segs.append(seg)
    return segs


def window_attn_workspace(T, N, H, d):
    return int(lib().vdn_window_attn_workspace(ctypes.byref(_shape(T, N, H, d))))


def window_attn(q, k, v, T, N, H, d, chunk_frames=5, window_chunks=1, anchors=3, scale=0.0,
                out=None, lse=None, ws=None, stream=None, ctx_k=None, ctx_v=None):
    """Window-and-anchor Softmax.  Returns (o, ws); fills ``lse`` [H, T*N] if given.

    ``ctx_k``/``ctx_v`` ([M, ld] bf16): context (text/audio) keys every video
    query also attends to, in the same softmax.
    """
    _need_cuda(q, k, v, out, lse, ws, ctx_k, ctx_v)
    shape = _shape(T, N, H, d)
    if out is None:
        out = torch.empty((T * N, H * d), dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = alloc_workspace(window_attn_workspace(T, N, H, d), q.device)
    if ctx_k is None:
        code = lib().vdn_window_attn(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), q.stride(0),
                                     int(chunk_frames), int(window_chunks), int(anchors),
                                     float(scale), _ptr(out), out.stride(0), _ptr(lse), _ptr(ws),
                                     ws.numel(), _stream(stream))
        _check(code, "vdn_window_attn")
    else:
        if ctx_v is None or ctx_v.shape != ctx_k.shape or ctx_v.stride(0) != ctx_k.stride(0):
            raise ValueError("ctx_k and ctx_v must have the same shape and row stride")
        code = lib().vdn_window_attn_ctx(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                         q.stride(0), _ptr(ctx_k), _ptr(ctx_v), ctx_k.stride(0),
                                         int(ctx_k.shape[0]), int(chunk_frames),
                                         int(window_chunks), int(anchors), float(scale),
                                         _ptr(out), out.stride(0), _ptr(lse), _ptr(ws),
                                         ws.numel(), _stream(stream))
        _check(code, "vdn_window_attn_ctx")
    return out, ws


def window_attn_mxfp8_workspace(T, N, H, d):
    return int(lib().vdn_window_attn_mxfp8_workspace(ctypes.byref(_shape(T, N, H, d))))


def window_attn_mxfp8(q, k, v, T, N, H, d, chunk_frames=5, window_chunks=1, anchors=3,
                      scale=0.0, out=None, lse=None, ws=None, stream=None):
    """Window-and-anchor Softmax with both products on MXFP8 operands (q, k,
    v quantized into the workspace by the call).  Returns (o, ws)."""
    _need_cuda(q, k, v, out, lse, ws)
    shape = _shape(T, N, H, d)
    if out is None:
        out = torch.empty((T * N, H * d), dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = alloc_workspace(window_attn_mxfp8_workspace(T, N, H, d), q.device)
    code = lib().vdn_window_attn_mxfp8(ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v),
                                       q.stride(0), int(chunk_frames), int(window_chunks),
                                       int(anchors), float(scale), _ptr(out), out.stride(0),
                                       _ptr(lse), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "vdn_window_attn_mxfp8")
    return out, ws


# ---------------------------------------------------------------- fuse

def hybrid_fuse_workspace(L, D, H):
    return int(lib().vdn_hybrid_fuse_workspace(int(L), int(D), int(H)))


def hybrid_fuse(x, o_s, o_vda, W_gs, W_gl, gamma, W_os, W_ol, H, eps=1e-6, out=None, ws=None,
                stream=None):
    """y = (sigmoid(x W_gs^T) o_s) W_os^T + (sigmoid(x W_gl^T) RMSNorm(o_vda)) W_ol^T."""
    _need_cuda(x, o_s, o_vda, W_gs, W_gl, gamma, W_os, W_ol, out, ws)
    L, D = x.shape
    if out is None:
        out = torch.empty((L, D), dtype=torch.bfloat16, device=x.device)
    if ws is None:
        ws = alloc_workspace(hybrid_fuse_workspace(L, D, H), x.device)
    code = lib().vdn_hybrid_fuse(int(L), int(D), int(H), _ptr(x), _ptr(o_s), _ptr(o_vda),
                                 _ptr(W_gs), _ptr(W_gl), _ptr(gamma), float(eps), _ptr(W_os),
                                 _ptr(W_ol), _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "vdn_hybrid_fuse")
    return out, ws


def hybrid_fuse_shard(x, o_s_local, o_vda_local, W_gs, W_gl, gamma, W_os, W_ol, d, head0,
                      eps=1e-6, out=None, ws=None, stream=None):
    """This head shard's fp32 partial of y (sum the partials over shards)."""
    _need_cuda(x, o_s_local, o_vda_local, W_gs, W_gl, gamma, W_os, W_ol, out, ws)
    L, D = x.shape
    H_local = o_s_local.shape[1] // d
    if out is None:
        out = torch.empty((L, D), dtype=torch.float32, device=x.device)
    if ws is None:
        ws = alloc_workspace(int(lib().vdn_hybrid_fuse_shard_workspace(L, D, H_local, d)),
                             x.device)
    code = lib().vdn_hybrid_fuse_shard(int(L), int(D), int(H_local), int(d), int(head0),
                                       _ptr(x), _ptr(o_s_local), _ptr(o_vda_local),
                                       o_s_local.stride(0), _ptr(W_gs), _ptr(W_gl), _ptr(gamma),
                                       float(eps), _ptr(W_os), _ptr(W_ol), _ptr(out), _ptr(ws),
                                       ws.numel(), _stream(stream))
    _check(code, "vdn_hybrid_fuse_shard")
    return out, ws


def hybrid_fuse_shard_rs(x, o_s_local, o_vda_local, W_gs, W_gl, gamma, W_os, W_ol, d, head0,
                         owners, eps=1e-6, ws=None, stream=None):
    """This head shard's contribution to y, added straight into the owners'
    row blocks (the GEMM fused with the reduce-scatter).  ``owners``: the G
    fp32 buffers [ceil(L/G), D] (the last may be shorter), zeroed beforehand;
    device pointers valid on this GPU (local, or peer-mapped)."""
    _need_cuda(x, o_s_local, o_vda_local, W_gs, W_gl, gamma, W_os, W_ol, ws, *owners)
    L, D = x.shape
    H_local = o_s_local.shape[1] // d
    if ws is None:
        ws = alloc_workspace(int(lib().vdn_hybrid_fuse_shard_workspace(L, D, H_local, d)),
                             x.device)
    ptrs = (_P * len(owners))(*[t.data_ptr() for t in owners])
    code = lib().vdn_hybrid_fuse_shard_rs(int(L), int(D), int(H_local), int(d), int(head0),
                                          _ptr(x), _ptr(o_s_local), _ptr(o_vda_local),
                                          o_s_local.stride(0), _ptr(W_gs), _ptr(W_gl),
                                          _ptr(gamma), float(eps), _ptr(W_os), _ptr(W_ol), ptrs,
                                          len(owners), _ptr(ws), ws.numel(), _stream(stream))
    _check(code, "vdn_hybrid_fuse_shard_rs")
    return ws


# ---------------------------------------------------------------- full layer

class HybridLayer:
    """The video-to-video hybrid attention layer on one GPU.

    forward() runs window-and-anchor Softmax, Video Delta Attention and the
    gated fuse (three C-ABI calls, seven kernels) and returns y [T*N, D].
    Inputs may be CUDA tensors, or host tensors (pinned for asynchronous
    copies): host inputs are copied into device buffers owned by the layer
    and, when ``out`` is a host tensor, y is copied back into it.
    ``projections="mxfp8"`` runs both fuse GEMMs on MXFP8 operands (weights
    quantized once here, x on every call); ``softmax="mxfp8"`` runs the
    window Softmax with both products on MXFP8 operands (q, k, v quantized
    on every call; head dim 128, tokens per frame a multiple of 32).
    """

    KERNELS_PER_FORWARD = 7   # prep, solve, scan, read-out, window Softmax, 2 GEMMs

    def __init__(self, T, N, H, d, W_gs, W_gl, W_os, W_ol, gamma, eps=1e-6, chunk_frames=5,
                 window_chunks=1, anchors=3, device=None, projections="bf16", softmax="bf16"):
        self.T, self.N, self.H, self.d = int(T), int(N), int(H), int(d)
        self.L, self.D = self.T * self.N, self.H * self.d
        self.device = torch.device(device or "cuda")
        dev = self.device
        self.W_gs, self.W_gl, self.W_os, self.W_ol = (
            w.to(dev, torch.bfloat16).contiguous() for w in (W_gs, W_gl, W_os, W_ol))
        self.gamma = gamma.to(dev, torch.float32).contiguous()
        self.eps = float(eps)
        self.mask = (int(chunk_frames), int(window_chunks), int(anchors))
        L, D = self.L, self.D
        self.o_s = torch.empty((L, D), dtype=torch.bfloat16, device=dev)
        self.o_vda = torch.empty((L, D), dtype=torch.bfloat16, device=dev)
        self.y = torch.empty((L, D), dtype=torch.bfloat16, device=dev)
        self.ws_vda = alloc_workspace(vda_scan_workspace(T, N, H, d), dev)
        if softmax not in ("bf16", "mxfp8"):
            raise ValueError("softmax: 'bf16' or 'mxfp8'")
        self.softmax = softmax
        self.ws_win = alloc_workspace(
            window_attn_mxfp8_workspace(T, N, H, d) if softmax == "mxfp8"
            else window_attn_workspace(T, N, H, d), dev)
        if projections not in ("bf16", "mxfp8"):
            raise ValueError("projections: 'bf16' or 'mxfp8'")
        self.projections = projections
        if projections == "mxfp8":
            self.wg, self.wo = mxfp8_fuse_weights(self.W_gs, self.W_gl, self.W_os, self.W_ol)
            self.ws_fuse = alloc_workspace(
                int(lib().vdn_hybrid_fuse_mxfp8_workspace(L, D, H)), dev)
            self.kernels_per_forward = self.KERNELS_PER_FORWARD + 1  # + quantize x
        else:
            self.ws_fuse = alloc_workspace(hybrid_fuse_workspace(L, D, H), dev)
            self.kernels_per_forward = self.KERNELS_PER_FORWARD
        if softmax == "mxfp8":
            self.kernels_per_forward += 3  # quantization of q, k, v
        self._staging = None

    def _window_heads(self, q, k, v, hg, out, stream):
        """The window Softmax on hg heads given as column views (row stride D)."""
        T, N, d = self.T, self.N, self.d
        cf, wc, an = self.mask
        if self.softmax == "mxfp8":
            window_attn_mxfp8(q, k, v, T, N, hg, d, cf, wc, an, out=out, ws=self.ws_win,
                              stream=stream)
        else:
            window_attn(q, k, v, T, N, hg, d, cf, wc, an, out=out, ws=self.ws_win,
                        stream=stream)

    def _window(self, q, k, v, stream, ctx_k=None, ctx_v=None):
        T, N, H, d = self.T, self.N, self.H, self.d
        cf, wc, an = self.mask
        if self.softmax == "mxfp8":
            if ctx_k is not None:
                raise ValueError("the MXFP8 window Softmax takes no context keys")
            window_attn_mxfp8(q, k, v, T, N, H, d, cf, wc, an, out=self.o_s, ws=self.ws_win,
                              stream=stream)
        else:
            window_attn(q, k, v, T, N, H, d, cf, wc, an, out=self.o_s, ws=self.ws_win,
                        stream=stream, ctx_k=ctx_k, ctx_v=ctx_v)

    def _fuse(self, x, y, stream):
        if self.projections == "mxfp8":
            hybrid_fuse_mxfp8(x, self.o_s, self.o_vda, self.wg, self.gamma, self.wo, self.H,
                              eps=self.eps, out=y, ws=self.ws_fuse, stream=stream)
        else:
            hybrid_fuse(x, self.o_s, self.o_vda, self.W_gs, self.W_gl, self.gamma, self.W_os,
                        self.W_ol, self.H, eps=self.eps, out=y, ws=self.ws_fuse, stream=stream)

    def _to_device(self, tensors, stream):
        if all(t.is_cuda for t in tensors):
            return tensors
        if self._staging is None:
            self._staging = [torch.empty(t.shape, dtype=t.dtype, device=self.device)
                             for t in tensors]
        with torch.cuda.stream(stream):
            for dst, src in zip(self._staging, tensors):
                dst.copy_(src, non_blocking=True)
        return self._staging

    def forward(self, q, k, v, beta, alpha, x, out=None, stream=None, ctx_k=None, ctx_v=None):
        """y for one video; ``ctx_k``/``ctx_v`` (CUDA, [M, D] bf16) are optional
        text/audio keys the Softmax branch also attends to."""
        stream = stream or torch.cuda.current_stream(self.device)
        q, k, v, beta, alpha, x = self._to_device([q, k, v, beta, alpha, x], stream)
        T, N, H, d = self.T, self.N, self.H, self.d
        self._window(q, k, v, stream, ctx_k, ctx_v)
        vda_scan(q, k, v, beta, alpha, T, N, H, d, out=self.o_vda, ws=self.ws_vda, stream=stream)
        self._fuse(x, self.y, stream)
        if out is not None and not out.is_cuda:
            with torch.cuda.stream(stream):
                out.copy_(self.y, non_blocking=True)
            return out
        return self.y

    def _fuse_rows(self, x, y, r0, r1, stream):
        """The fuse on token rows [r0, r1) (every step of it is per token)."""
        if self.projections == "mxfp8":
            hybrid_fuse_mxfp8(x[r0:r1], self.o_s[r0:r1], self.o_vda[r0:r1], self.wg, self.gamma,
                              self.wo, self.H, eps=self.eps, out=y[r0:r1], ws=self.ws_fuse,
                              stream=stream)
        else:
            hybrid_fuse(x[r0:r1], self.o_s[r0:r1], self.o_vda[r0:r1], self.W_gs, self.W_gl,
                        self.gamma, self.W_os, self.W_ol, self.H, eps=self.eps, out=y[r0:r1],
                        ws=self.ws_fuse, stream=stream)

    # forward_many's fill and drain granularity: the first video's inputs
    # arrive in up to FILL_GROUPS head groups (the largest count that divides
    # H), the last video's fuse and read-back run in up to DRAIN_BLOCKS row
    # blocks (multiples of 128 rows)
    FILL_GROUPS = 4
    DRAIN_BLOCKS = 4

    def _head_groups(self):
        """Head groups of the first video of forward_many."""
        g = next(n for n in range(min(self.FILL_GROUPS, self.H), 0, -1) if self.H % n == 0)
        return [(i * (self.H // g), self.H // g) for i in range(g)]

    def _row_chunks(self):
        """Row blocks of the last video's fuse and read-back."""
        nb = max(1, int(self.DRAIN_BLOCKS))
        step = max(128, (self.L + nb * 128 - 1) // (nb * 128) * 128)
        return [(r, min(r + step, self.L)) for r in range(0, self.L, step)]

    def forward_many(self, batches, outs, stream=None, copy_stream=None):
        """Run the layer over several videos held in (pinned) host memory.

        ``batches`` is a list of (q, k, v, beta, alpha, x) host tensors
        (q, k, v, x [T*N, D], beta [T*N, H], alpha [T, H], rows contiguous)
        and ``outs`` a list of host tensors [T*N, D] bf16 that receive y.
        Copies run on ``copy_stream`` into two device staging sets, so the
        input of video i+1 and the result of video i-1 move while video i
        computes.  The pipeline's fill and drain are cut short:
          * the first video's q, k, v, beta and alpha arrive in head groups
            (pitched copies of their columns), and both attention branches
            start on a group as soon as it has landed;
          * for the other videos q, k, v are copied first: the window
            Softmax, which needs only them, starts before beta, alpha and x;
          * the last video's fuse runs in row blocks, each block's y read
            back while the next one computes.
        Returns after enqueueing; synchronise the streams to read ``outs``.
        """
        if len(batches) != len(outs):
            raise ValueError("one output per batch")
        dev = self.device
        stream = stream or torch.cuda.current_stream(dev)
        copy_stream = copy_stream or getattr(self, "_copy_stream", None)
        if copy_stream is None:
            copy_stream = self._copy_stream = torch.cuda.Stream(dev)
        T, N, H, d = self.T, self.N, self.H, self.d
        groups = self._head_groups()
        if getattr(self, "_stages", None) is None:
            b0 = batches[0]
            self._stages = [[torch.empty(t.shape, dtype=t.dtype, device=dev) for t in b0]
                            for _ in range(2)]
            self._ys = [torch.empty((self.L, self.D), dtype=torch.bfloat16, device=dev)
                        for _ in range(2)]
        if getattr(self, "_grp_key", None) != tuple(groups):
            # per head group: its beta and alpha columns, contiguous (rebuilt
            # whenever the grouping changes)
            self._grp_ba = [(torch.empty((self.L, hg), dtype=torch.float32, device=dev),
                             torch.empty((T, hg), dtype=torch.float32, device=dev))
                            for _, hg in groups]
            self._grp_key = tuple(groups)
        if len(self._grp_ba) != len(groups):
            raise RuntimeError("forward_many: head-group buffers out of step with the grouping")
        stages, ys = self._stages, self._ys
        loaded_qkv = [torch.cuda.Event() for _ in batches]
        loaded = [torch.cuda.Event() for _ in batches]
        computed = [torch.cuda.Event() for _ in batches]
        grp_loaded = [torch.cuda.Event() for _ in groups]
        n = len(batches)

        def load(i):
            with torch.cuda.stream(copy_stream):
                if i >= 2:
                    copy_stream.wait_event(computed[i - 2])   # stage i % 2 is free
                for k_, (dst, src) in enumerate(zip(stages[i % 2], batches[i])):
                    dst.copy_(src, non_blocking=True)
                    if k_ == 2:
                        loaded_qkv[i].record(copy_stream)
                loaded[i].record(copy_stream)

        def load_first_by_groups():
            q, k, v, _, _, x = stages[0]
            hq, hk, hv, hb, ha, hx = batches[0]
            with torch.cuda.stream(copy_stream):
                for (h0, hg), (bg, ag), ev in zip(groups, self._grp_ba, grp_loaded):
                    copy_columns_async(bg, 0, hb, h0, hg)
                    copy_columns_async(ag, 0, ha, h0, hg)
                    for dst, src in ((q, hq), (k, hk), (v, hv)):
                        copy_columns_async(dst, h0 * d, src, h0 * d, hg * d)
                    ev.record(copy_stream)
                x.copy_(hx, non_blocking=True)
                loaded[0].record(copy_stream)

        copy_stream.wait_stream(stream)  # copies start after work already on `stream`
        load_first_by_groups()
        self._read = [torch.cuda.Event() for _ in batches]
        for i in range(n):
            if i + 1 < n:
                load(i + 1)
            if i >= 2:
                stream.wait_event(self._read[i - 2])           # y buffer i % 2 is free
            q, k, v, beta, alpha, x = stages[i % 2]
            y = ys[i % 2]
            if i == 0:
                # both branches per head group, each as soon as it has landed
                for (h0, hg), (bg, ag), ev in zip(groups, self._grp_ba, grp_loaded):
                    stream.wait_event(ev)
                    c = slice(h0 * d, (h0 + hg) * d)
                    self._window_heads(q[:, c], k[:, c], v[:, c], hg, self.o_s[:, c], stream)
                    vda_scan(q[:, c], k[:, c], v[:, c], bg, ag, T, N, hg, d,
                             out=self.o_vda[:, c], ws=self.ws_vda, stream=stream)
            else:
                stream.wait_event(loaded_qkv[i])
                self._window(q, k, v, stream)
                stream.wait_event(loaded[i])                    # beta, alpha, x
                vda_scan(q, k, v, beta, alpha, T, N, H, d, out=self.o_vda, ws=self.ws_vda,
                         stream=stream)
            stream.wait_event(loaded[i])                        # x
            if i + 1 < n:
                self._fuse(x, y, stream)
                computed[i].record(stream)
                with torch.cuda.stream(copy_stream):
                    copy_stream.wait_event(computed[i])
                    outs[i].copy_(y, non_blocking=True)
                    self._read[i].record(copy_stream)
            else:
                # the last video: fuse and read back in row blocks
                for r0, r1 in self._row_chunks():
                    self._fuse_rows(x, y, r0, r1, stream)
                    done = torch.cuda.Event()
                    done.record(stream)
                    with torch.cuda.stream(copy_stream):
                        copy_stream.wait_event(done)
                        outs[i][r0:r1].copy_(y[r0:r1], non_blocking=True)
                computed[i].record(stream)
                self._read[i].record(copy_stream)
        return outs

    def status(self):
        """Worst device status over the layer's workspaces (synchronises)."""
        return max(get_device_status(w) for w in (self.ws_vda, self.ws_win, self.ws_fuse))


class HeadShardedLayer:
    """One video's hybrid layer split by heads over a process group, for a
    caller that holds the full activations on every rank.

    Rank r of G owns heads [r H/G, (r+1) H/G).  The window Softmax and VDA
    branches are per head, so each rank runs them on its own head columns
    (views into the full [T*N, D] activations) with no communication; the
    fuse is row-parallel: each rank forms its hidden columns of the gated
    branch inputs and an fp32 partial of y over the full width
    (vdn_hybrid_fuse_shard).  One reduce-scatter sums the partials and leaves
    rank r the rows [r R, (r+1) R) of y, R = ceil(T*N / G) (the fp32 sum adds
    no bf16 rounding; each rank receives 1/G of the sum instead of all of
    it).  ``output="rows"`` returns that row block in bf16, ``output="full"``
    also all-gathers the bf16 blocks into the whole y on every rank.

    ``collective="fused"`` replaces the partial and the reduce-scatter with
    one kernel (vdn_hybrid_fuse_shard_rs): the output GEMM's epilogue adds
    each row of this rank's partial straight into the row block of the rank
    that owns it, through peer mappings of the other ranks' fp32 row-block
    buffers (CUDA IPC handles exchanged once, at construction; plain
    system-scope atomic adds, no multicast).  Every rank zeroes its own
    block and the ranks meet on the host before the kernel, and again
    after it before a block is read.  No kernel waits on another rank.
    ``ops`` replaces the compute calls (tests only).
    """

    def __init__(self, T, N, H, d, W_gs, W_gl, W_os, W_ol, gamma, eps=1e-6, group=None,
                 device=None, ops=None, act_dtype=torch.bfloat16, acc_dtype=torch.float32,
                 output="full", collective="reduce_scatter"):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if H % self.world:
            raise ValueError("heads must divide evenly over the ranks")
        if output not in ("rows", "full"):
            raise ValueError("output: 'rows' or 'full'")
        if collective not in ("reduce_scatter", "fused"):
            raise ValueError("collective: 'reduce_scatter' or 'fused'")
        self.output = output
        self.collective = collective
        self.T, self.N, self.H, self.d = int(T), int(N), int(H), int(d)
        self.L, self.D = self.T * self.N, self.H * self.d
        self.Hl = self.H // self.world
        self.head0 = self.rank * self.Hl
        self.cols = slice(self.head0 * self.d, (self.head0 + self.Hl) * self.d)
        self.R = -(-self.L // self.world)           # rows of y each rank receives
        self.rows = slice(min(self.rank * self.R, self.L), min((self.rank + 1) * self.R, self.L))
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        dev = self.device
        self.W = [w.to(dev, act_dtype).contiguous() for w in (W_gs, W_gl, W_os, W_ol)]
        self.gamma = gamma.to(dev, acc_dtype).contiguous()
        self.eps = float(eps)
        Dl = self.Hl * self.d
        if ops is None:
            Hl, d = self.Hl, self.d
            ws_win = alloc_workspace(window_attn_workspace(T, N, Hl, d), dev)
            ws_vda = alloc_workspace(vda_scan_workspace(T, N, Hl, d), dev)
            ws_fuse = alloc_workspace(
                int(lib().vdn_hybrid_fuse_shard_workspace(self.L, self.D, Hl, d)), dev)
            ops = {"window_attn": functools.partial(window_attn, ws=ws_win),
                   "vda_scan": functools.partial(vda_scan, ws=ws_vda),
                   "fuse_shard": functools.partial(hybrid_fuse_shard, ws=ws_fuse),
                   "fuse_shard_rs": functools.partial(hybrid_fuse_shard_rs, ws=ws_fuse)}
            self.workspaces = (ws_win, ws_vda, ws_fuse)
        self.ops = ops
        self.o_s = torch.empty((self.L, Dl), dtype=act_dtype, device=dev)
        self.o_vda = torch.empty((self.L, Dl), dtype=act_dtype, device=dev)
        # G*R rows so that every rank's block has R rows; rows past L stay zero
        self.y_partial = torch.zeros((self.world * self.R, self.D), dtype=acc_dtype, device=dev)
        self.y_rows32 = torch.empty((self.R, self.D), dtype=acc_dtype, device=dev)
        self.y_rows = torch.empty((self.R, self.D), dtype=act_dtype, device=dev)
        self.y = (torch.empty((self.world * self.R, self.D), dtype=act_dtype, device=dev)
                  if output == "full" else None)
        if collective == "fused":
            # this rank's row block, and every rank's block mapped here
            self.owner = torch.zeros((self.R, self.D), dtype=acc_dtype, device=dev)
            if self.world == 1:
                self.owners = [self.owner]
            else:
                from torch.multiprocessing.reductions import reduce_tensor
                handles = [None] * self.world
                dist.all_gather_object(handles, reduce_tensor(self.owner)[1], group=group)
                self.owners = [self.owner if g == self.rank else _open_peer_block(handles[g])
                               for g in range(self.world)]

    def forward(self, q, k, v, beta, alpha, x):
        """y (full, [T*N, D]) or this rank's rows of y ([rows, D], rows = self.rows)."""
        c, Hl, d = self.cols, self.Hl, self.d
        h0, h1 = self.head0, self.head0 + self.Hl
        ql, kl, vl = q[:, c], k[:, c], v[:, c]             # views, row stride D
        beta_l = beta[:, h0:h1].contiguous()
        alpha_l = alpha[:, h0:h1].contiguous()
        self.ops["window_attn"](ql, kl, vl, self.T, self.N, Hl, d, out=self.o_s)
        self.ops["vda_scan"](ql, kl, vl, beta_l, alpha_l, self.T, self.N, Hl, d, out=self.o_vda)
        if self.collective == "fused":
            self.owner.zero_()
            self._meet()                                    # every block zeroed
            self.ops["fuse_shard_rs"](x, self.o_s, self.o_vda, *self.W[:2], self.gamma,
                                      *self.W[2:], d, h0, self.owners, eps=self.eps)
            self._meet()                                    # every rank's rows added
            self.y_rows.copy_(self.owner)                   # fp32 sum -> bf16
        else:
            self.ops["fuse_shard"](x, self.o_s, self.o_vda, *self.W[:2], self.gamma,
                                   *self.W[2:], d, h0, eps=self.eps,
                                   out=self.y_partial[:self.L])
            self.dist.reduce_scatter_tensor(self.y_rows32, self.y_partial, group=self.group)
            self.y_rows.copy_(self.y_rows32)                # fp32 sum -> bf16
        if self.output == "rows":
            return self.y_rows[:self.rows.stop - self.rows.start]
        self.dist.all_gather_into_tensor(self.y, self.y_rows, group=self.group)
        return self.y[:self.L]


    def close(self):
        """Release the peer mappings of the fused collective; every rank calls
        it before the process group goes away, so no rank's block is freed
        while another still maps it."""
        if self.collective == "fused" and self.world > 1:
            self._meet()
            self.owners = [self.owner]
            self._meet()

    def _meet(self):
        """All ranks' work enqueued so far is complete (a host-side meeting)."""
        if self.device.type == "cuda":
            torch.cuda.current_stream(self.device).synchronize()
        self.dist.barrier(group=self.group)


def _open_peer_block(args):
    """A tensor over another process's CUDA allocation, from the arguments
    torch's CUDA IPC sharing produced for it (the mapping enables peer
    access lazily; nothing is copied)."""
    from torch.multiprocessing.reductions import rebuild_cuda_tensor
    return rebuild_cuda_tensor(*args)


class SeqShardedLayer:
    """One video's hybrid layer for a caller whose activations are split by
    token rows over a process group (sequence parallelism), with the
    attention run head-parallel in between (all-to-all, Ulysses style).

    Rank r of G holds token rows [r R, (r+1) R) of q, k, v, x and beta,
    R = T*N / G, and the whole alpha.  One all-to-all per tensor gives every
    rank all T*N rows of its H/G heads; the window Softmax and VDA run there
    (both need every token of a head and nothing of the other heads); an
    all-to-all per branch output brings the rows back; the fuse then runs on
    the rank's own rows with the full weights (gates, RMSNorm and both
    projections are per token), so no reduction is needed.  Bytes each rank
    sends per layer: (G-1)/G of 5 activations' row blocks (q, k, v out, o_s,
    o_vda back) plus beta.  The column blocks are packed into and out of the
    contiguous all-to-all buffers with copies.  ``ops`` replaces the compute
    calls (tests only).
    """

    def __init__(self, T, N, H, d, W_gs, W_gl, W_os, W_ol, gamma, eps=1e-6, group=None,
                 device=None, ops=None, act_dtype=torch.bfloat16, acc_dtype=torch.float32):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = G = dist.get_world_size(group)
        self.T, self.N, self.H, self.d = int(T), int(N), int(H), int(d)
        self.L, self.D = self.T * self.N, self.H * self.d
        if self.H % G or self.L % G:
            raise ValueError("heads and token rows must divide evenly over the ranks")
        self.R, self.Hl = self.L // G, self.H // G
        self.C = self.Hl * self.d
        self.head0 = self.rank * self.Hl
        self.rows = slice(self.rank * self.R, (self.rank + 1) * self.R)
        self.device = torch.device(device) if device is not None else torch.device("cuda")
        dev = self.device
        self.W = [w.to(dev, act_dtype).contiguous() for w in (W_gs, W_gl, W_os, W_ol)]
        self.gamma = gamma.to(dev, acc_dtype).contiguous()
        self.eps = float(eps)
        L, R, C, D = self.L, self.R, self.C, self.D
        if ops is None:
            Hl, d = self.Hl, self.d
            ws_win = alloc_workspace(window_attn_workspace(T, N, Hl, d), dev)
            ws_vda = alloc_workspace(vda_scan_workspace(T, N, Hl, d), dev)
            ws_fuse = alloc_workspace(hybrid_fuse_workspace(R, D, self.H), dev)
            ops = {"window_attn": functools.partial(window_attn, ws=ws_win),
                   "vda_scan": functools.partial(vda_scan, ws=ws_vda),
                   "fuse": functools.partial(hybrid_fuse, ws=ws_fuse)}
            self.workspaces = (ws_win, ws_vda, ws_fuse)
        self.ops = ops
        mk = lambda *shape, dt=act_dtype: torch.empty(shape, dtype=dt, device=dev)
        self.send = [mk(G, R, C) for _ in range(3)]          # q, k, v column blocks
        self.heads = [mk(L, C) for _ in range(3)]            # all rows of this rank's heads
        self.beta_send, self.beta_l = mk(G, R, self.Hl, dt=acc_dtype), mk(L, self.Hl, dt=acc_dtype)
        self.o_s, self.o_vda = mk(L, C), mk(L, C)             # branch outputs, this rank's heads
        self.back = [mk(G, R, C) for _ in range(2)]          # their column blocks of my rows
        self.o_s_rows, self.o_vda_rows = mk(R, D), mk(R, D)
        self.y = mk(R, D)

    def _to_heads(self, src, send, recv, width):
        """[R, G*width] row block -> [G*R, width]: all rows of this rank's columns."""
        G, R = self.world, self.R
        send.copy_(src.reshape(R, G, width).transpose(0, 1))
        self.dist.all_to_all_single(recv.view(G, R, width), send, group=self.group)

    def forward(self, q, k, v, beta, alpha, x):
        """This rank's rows of y ([R, D]) from its rows of q, k, v, x ([R, D]),
        beta ([R, H]) and the whole alpha ([T, H])."""
        G, R, C, Hl, d = self.world, self.R, self.C, self.Hl, self.d
        for src, send, recv in zip((q, k, v), self.send, self.heads):
            self._to_heads(src, send, recv, C)
        self._to_heads(beta, self.beta_send, self.beta_l, Hl)
        alpha_l = alpha[:, self.head0:self.head0 + Hl].contiguous()
        ql, kl, vl = self.heads
        self.ops["window_attn"](ql, kl, vl, self.T, self.N, Hl, d, out=self.o_s)
        self.ops["vda_scan"](ql, kl, vl, self.beta_l, alpha_l, self.T, self.N, Hl, d,
                             out=self.o_vda)
        for o, back, rows in zip((self.o_s, self.o_vda), self.back,
                                 (self.o_s_rows, self.o_vda_rows)):
            # chunk g of o holds rank g's rows: it goes back to rank g
            self.dist.all_to_all_single(back, o.view(G, R, C), group=self.group)
            rows.view(R, G, C).copy_(back.transpose(0, 1))
        self.ops["fuse"](x, self.o_s_rows, self.o_vda_rows, self.W[0], self.W[1], self.gamma,
                         self.W[2], self.W[3], self.H, eps=self.eps, out=self.y)
        return self.y
