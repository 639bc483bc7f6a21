"""MXFP8 (OCP Microscaling, E4M3 elements, UE8M0 block scales), float64 CPU
oracle.  TEST INFRASTRUCTURE ONLY.

The MXFP8 variant of the layer's projections ("Video DeltaNet", 10100.com
article, 实验结果 / 效率阶梯, which times 8-step denoising under MXFP8 on one
to eight B200s; the pages give no format details, so the OCP Microscaling
definition of MXFP8 is taken) quantizes every GEMM operand in blocks of 32
consecutive elements along the contraction dimension:

  * element format E4M3 (sign, 4 exponent bits with bias 7, 3 mantissa bits,
    subnormals, no infinities; largest finite 448, smallest subnormal 2^-9);
  * one shared scale per block, a power of two X = 2^e stored as the byte
    e + 127 (UE8M0); e = floor(log2(max |v|)) - 8 (8 = the exponent of
    E4M3's largest normal), clamped to [-127, 127]; a block of zeros gets
    e = -127;
  * elements = v / X rounded to nearest E4M3 (ties to the even code) and
    saturated to +-448.

Everything here is exact float64 arithmetic over the table of the 127
non-negative finite E4M3 values.  The scale bytes are also arranged in the
tile layout the block-scaled tensor-core GEMM reads (``sf_tiled``): per
128-row x 128-column tile a 512-byte block, byte (r % 32) * 16 +
((r % 128) // 32) * 4 + (k_block % 4), tiles ordered [row tile][column tile].
"""

import numpy as np

from .fuse import sigmoid, rmsnorm_heads

BLOCK = 32
E4M3_MAX = 448.0
E4M3_EMAX = 8


def _e4m3_table():
    """Non-negative finite E4M3 values, indexed by their 7-bit code."""
    vals = []
    for code in range(127):  # 0x7F is NaN
        e, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7))
    return np.array(vals)


E4M3_VALUES = _e4m3_table()


def e4m3_encode(x):
    """Round to nearest E4M3 (ties to even code), saturating at +-448; the
    sign bit is kept, so negative values that round to zero give 0x80."""
    x = np.asarray(x, dtype=np.float64)
    a = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(E4M3_VALUES, a, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo, d_hi = a - E4M3_VALUES[lo], E4M3_VALUES[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    # the sign survives rounding to zero (IEEE: a negative tiny value gives -0)
    return code | np.where(np.signbit(x), 0x80, 0).astype(np.uint8)


def e4m3_decode(code):
    code = np.asarray(code, dtype=np.uint8)
    v = E4M3_VALUES[code & 0x7F]
    return np.where(code & 0x80, -v, v)


def mx_block_exponents(v):
    """Shared exponent e per 32-element block of the last axis."""
    v = np.asarray(v, dtype=np.float64)
    blocks = np.abs(v).reshape(*v.shape[:-1], v.shape[-1] // BLOCK, BLOCK)
    amax = blocks.max(axis=-1)
    # floor(log2(amax)) read off the float64 exponent (exact): amax = m 2^p, m in [1/2, 1)
    e = np.where(amax > 0, np.frexp(np.where(amax > 0, amax, 1.0))[1] - 1 - E4M3_EMAX, -127)
    return np.clip(e, -127, 127).astype(np.int64)


def mx_quantize(v):
    """v [..., K] (K a multiple of 32) -> (E4M3 codes [..., K], scale bytes [..., K/32])."""
    v = np.asarray(v, dtype=np.float64)
    e = mx_block_exponents(v)
    scale = np.repeat(np.ldexp(1.0, e), BLOCK, axis=-1)
    return e4m3_encode(v / scale), (e + 127).astype(np.uint8)


def mx_dequantize(codes, scale_bytes):
    e = scale_bytes.astype(np.int64) - 127
    return e4m3_decode(codes) * np.repeat(np.ldexp(1.0, e), BLOCK, axis=-1)


def sf_tiled(scale_bytes):
    """[R, K/32] scale bytes -> the tile layout of the GEMM (rows padded to
    128 with the byte 127, i.e. scale 1)."""
    R, KB = scale_bytes.shape
    rt, kt = -(-R // 128), KB // 4
    out = np.full(rt * kt * 512, 127, dtype=np.uint8)
    r = np.arange(R)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * kt + kb // 4) * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + kb % 4
    out[off] = scale_bytes
    return out


def gemm_mx(a_codes, a_scales, b_codes, b_scales):
    """C = A B^T on the dequantized operands (A [M, K], B [N, K])."""
    return mx_dequantize(a_codes, a_scales) @ mx_dequantize(b_codes, b_scales).T


def hybrid_fuse_mxfp8(x, o_s, o_vda, W_gs, W_gl, gamma, eps, W_os, W_ol, H):
    """The fuse with MXFP8 projections: x and both weight stacks quantized,
    the gated branch inputs Z = [g_s o_s | g_l RMSNorm(o_vda) gamma] formed
    in float64 from the quantized gate GEMM and quantized again, then
    y = Z [W_os | W_ol]^T on the quantized operands."""
    x = np.asarray(x, dtype=np.float64)
    D = x.shape[1]
    xq = mx_quantize(x)
    wgq = mx_quantize(np.concatenate([W_gs, W_gl], axis=0))
    G = gemm_mx(*xq, *wgq)
    n = rmsnorm_heads(o_vda, H, D // H, gamma, eps)
    Z = np.concatenate([sigmoid(G[:, :D]) * np.asarray(o_s, dtype=np.float64),
                        sigmoid(G[:, D:]) * n], axis=1)
    zq = mx_quantize(Z)
    woq = mx_quantize(np.concatenate([W_os, W_ol], axis=1))
    return gemm_mx(*zq, *woq)


# ---------------------------------------------------------------- window Softmax

def mx_quantize_columns(x):
    """MX quantization along the rows of x [R, C] (R a multiple of 32): blocks
    of 32 consecutive rows of each column, as for the value operand of the PV
    product (its contraction runs over key tokens).  Returns the dequantized
    values [R, C]."""
    codes, scales = mx_quantize(np.asarray(x, dtype=np.float64).T)
    return mx_dequantize(codes, scales).T


def window_attn_mxfp8_rows(q, k, v, T, N, H, d, rows, chunk_frames=5, window_chunks=1,
                           anchors=3, scale=None, heads=None):
    """Window-and-anchor Softmax with both products on MXFP8 operands, for the
    given query token rows.  Returns (o [len(rows), H*d], lse [H, len(rows)]).

    Every operand is quantized in blocks of 32 along the contraction of its
    product (OCP MX, as ``mx_quantize``):
      * q and k per token and head along d (the S = q k^T contraction);
      * v per column along the key tokens, in blocks of 32 consecutive token
        rows counted from row 0 (the P V contraction);
      * the probabilities per query row along the keys, in blocks of 32
        consecutive keys of each visible key interval.
    With s = q^ . k^ * scale, s2 = s log2(e) and m = ceil(max over the row's
    visible keys of s2) (an integer, so the block quantization of P does not
    depend on which upper bound of the row maximum is subtracted):
      P = 2^(s2 - m),  l = sum P,  o = sum_keys P^ v^ / l,
      lse = (m + log2 l) ln 2.
    The row sum l is taken over the unquantized P.  The visible key
    intervals (whole frames) start and end on multiples of 32, i.e. N is a
    multiple of 32.
    """
    if N % 32 or d % 32:
        raise ValueError("tokens per frame and head dim must be multiples of 32")
    from .window_attn import visible_key_frames
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    rows = np.asarray(rows, dtype=np.int64)
    heads = range(H) if heads is None else heads
    out = np.zeros((len(rows), H * d))
    lse = np.zeros((H, len(rows)))
    frames = rows // N
    log2e = 1.0 / np.log(2.0)
    for h in heads:
        c = slice(h * d, (h + 1) * d)
        kq_cache, vq_cache = {}, {}

        def quantized_frames(tk):
            # a frame's keys and values: 32-aligned row blocks of the tensor
            if tk not in kq_cache:
                r = slice(tk * N, (tk + 1) * N)
                kq_cache[tk] = mx_dequantize(*mx_quantize(np.asarray(k[r, c], dtype=np.float64)))
                vq_cache[tk] = mx_quantize_columns(np.asarray(v[r, c], dtype=np.float64))
            return kq_cache[tk], vq_cache[tk]

        for tq in np.unique(frames):
            sel = np.nonzero(frames == tq)[0]
            kf = visible_key_frames(int(tq), T, chunk_frames, window_chunks, anchors)
            Kq = np.vstack([quantized_frames(tk)[0] for tk in kf])
            Vq = np.vstack([quantized_frames(tk)[1] for tk in kf])
            Qq = mx_dequantize(*mx_quantize(np.asarray(q[rows[sel], c], dtype=np.float64)))
            s2 = (Qq @ Kq.T) * scale * log2e
            m = np.ceil(s2.max(axis=1, keepdims=True))
            P = np.exp2(s2 - m)
            l = P.sum(axis=1, keepdims=True)
            # blocks of 32 keys: the keys are whole frames of N (a multiple of
            # 32) tokens, so consecutive 32-key groups of the row are the blocks
            Pq = mx_dequantize(*mx_quantize(P))
            out[sel, c] = (Pq @ Vq) / l
            lse[h, sel] = (m[:, 0] + np.log2(l[:, 0])) / log2e
    return out, lse


def window_attn_mxfp8(q, k, v, T, N, H, d, chunk_frames=5, window_chunks=1, anchors=3,
                      scale=None):
    """window_attn_mxfp8_rows for every token row."""
    return window_attn_mxfp8_rows(q, k, v, T, N, H, d, np.arange(T * N), chunk_frames,
                                  window_chunks, anchors, scale)
