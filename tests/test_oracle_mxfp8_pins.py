"""Pins of the MXFP8 oracle: the E4M3 value table against its defining
constants, encoding against torch's independent float8_e4m3fn conversion,
round-to-nearest-even ties, saturation, the block-scale rule on blocks with
known maxima, the quantization error bound, and the tile layout of the
scale bytes on hand-computed offsets."""

import numpy as np
import pytest
import torch

from oracle import mxfp8


def test_e4m3_table_constants():
    v = mxfp8.E4M3_VALUES
    assert v.shape == (127,)
    assert np.all(np.diff(v) > 0)
    assert v[0x7E] == 448.0                    # largest finite
    assert v[0x38] == 1.0                      # exponent field 7 = bias
    assert v[0x08] == 2.0 ** -6                # smallest normal
    assert v[0x01] == 2.0 ** -9                # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9            # largest subnormal


def test_encode_matches_torch_float8_on_the_rounding_range():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.uniform(-4, 2.6, 20000),
                        mxfp8.E4M3_VALUES, -mxfp8.E4M3_VALUES,
                        (mxfp8.E4M3_VALUES[1:] + mxfp8.E4M3_VALUES[:-1]) / 2])  # every tie
    x = x[np.abs(x) <= 464.0].astype(np.float32)
    ours = mxfp8.e4m3_encode(x.astype(np.float64))
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_round_trip_ties_and_saturation():
    v = mxfp8.E4M3_VALUES
    np.testing.assert_array_equal(mxfp8.e4m3_decode(mxfp8.e4m3_encode(v)), v)
    np.testing.assert_array_equal(mxfp8.e4m3_decode(mxfp8.e4m3_encode(-v[1:])), -v[1:])
    assert mxfp8.e4m3_encode(1.0625) == 0x38      # tie between 1.0 and 1.125 -> even code
    assert mxfp8.e4m3_encode(1.1875) == 0x3A      # tie between 1.125 and 1.25 -> even code
    assert mxfp8.e4m3_encode(2.0 ** -10) == 0x00  # tie between 0 and 2^-9
    assert mxfp8.e4m3_encode(1000.0) == 0x7E
    assert mxfp8.e4m3_encode(-1e9) == 0xFE
    assert mxfp8.e4m3_encode(-2.0 ** -12) == 0x80  # negative, rounds to -0


def test_block_scale_rule():
    blk = np.zeros((5, 32))
    blk[0, 3] = 1.0            # max 1      -> e = 0 - 8
    blk[1, 7] = -3.5           # max 3.5    -> e = 1 - 8
    blk[2, 0] = 2.0 ** -20     # max 2^-20  -> e = -28
    blk[3, 0] = 1e38           # e = 126 - 8 = 118
    codes, sb = mxfp8.mx_quantize(blk)
    assert list(sb[:, 0].astype(int) - 127) == [-8, -7, -28, 118, -127]
    assert np.all(codes[4] == 0)                           # a zero block
    # the scaled block maximum lies in [256, 512) and saturates above 448
    assert mxfp8.e4m3_decode(codes[0, 3]) * 2.0 ** -8 == 1.0
    assert mxfp8.e4m3_decode(codes[1, 7]) * 2.0 ** -7 == -3.5
    big = np.full((1, 32), 1.0)
    big[0, 0] = 1.99                                        # 1.99 * 2^8 = 509 -> 448
    c, s = mxfp8.mx_quantize(big)
    assert mxfp8.mx_dequantize(c, s)[0, 0] == 448 * 2.0 ** -8


def test_quantization_error_bound():
    """Every element within half an E4M3 step of its value (relative 2^-4 of
    the element for the normal range, 2^-10 of the block scale's 2^8 for the
    subnormal range), except a saturated block maximum (at most 1/8 low)."""
    rng = np.random.default_rng(1)
    v = rng.standard_normal((64, 256)) * np.exp(rng.uniform(-6, 6, (64, 1)))
    c, s = mxfp8.mx_quantize(v)
    dq = mxfp8.mx_dequantize(c, s)
    scale = np.repeat(np.ldexp(1.0, s.astype(int) - 127), 32, axis=1)
    x = v / scale
    err = np.abs(dq / scale - x)
    ok = (err <= np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10)) | \
         ((np.abs(x) > 448) & (err <= np.abs(x) / 8))
    assert ok.all()


def test_scale_tile_layout_offsets():
    R, K = 300, 512
    sb = np.arange(R * (K // 32), dtype=np.int64).reshape(R, K // 32) % 251
    t = mxfp8.sf_tiled(sb.astype(np.uint8))
    assert t.size == 3 * 4 * 512                       # ceil(300/128) x (512/128) tiles
    # row 33, k-block 5: tile (0, 1), row 1 of the 32-row group 1, byte 1
    assert t[512 + 1 * 16 + 1 * 4 + 1] == sb[33, 5]
    # row 299, k-block 15: tile (2, 3); 299 % 128 = 43 -> group 1, row 11
    assert t[(2 * 4 + 3) * 512 + 11 * 16 + 1 * 4 + 3] == sb[299, 15]
    # padding rows hold the unit scale
    assert t[(2 * 4 + 0) * 512 + 31 * 16 + 3 * 4] == 127


def test_gemm_mx_is_the_product_of_dequantized_operands():
    rng = np.random.default_rng(2)
    a, b = rng.standard_normal((7, 64)), rng.standard_normal((5, 64))
    aq, bq = mxfp8.mx_quantize(a), mxfp8.mx_quantize(b)
    c = mxfp8.gemm_mx(*aq, *bq)
    A, B = mxfp8.mx_dequantize(*aq), mxfp8.mx_dequantize(*bq)
    for i in range(7):
        for j in range(5):
            assert abs(c[i, j] - sum(A[i, k] * B[j, k] for k in range(64))) < 1e-12
    # and close to the unquantized product (E4M3 keeps ~2 significant digits)
    assert np.abs(c - a @ b.T).max() < 0.1 * np.abs(a @ b.T).max()


def test_fuse_is_exact_on_operands_the_format_holds():
    """Special case that reduces to the plain fuse: with zero gate weights
    (gates exactly 1/2), o_vda = 0 (RMSNorm gives 0) and small integers in o_s
    and W_os (every 32-element block then holds only values E4M3 represents
    under its shared scale), every quantization step is exact, so the MXFP8
    fuse equals 0.5 * o_s W_os^T and the float64 fuse exactly."""
    from oracle import fuse as ofuse
    rng = np.random.default_rng(3)
    L, D, H = 64, 128, 2
    x = rng.standard_normal((L, D))
    o_s = rng.integers(-8, 9, (L, D)).astype(np.float64)
    o_vda = np.zeros((L, D))
    W_gs = np.zeros((D, D))
    W_gl = np.zeros((D, D))
    W_os = rng.integers(-8, 9, (D, D)).astype(np.float64)
    W_ol = rng.integers(-8, 9, (D, D)).astype(np.float64)
    gamma = np.ones(D)
    y_mx = mxfp8.hybrid_fuse_mxfp8(x, o_s, o_vda, W_gs, W_gl, gamma, 1e-6, W_os, W_ol, H)
    y = ofuse.hybrid_fuse(x, o_s, o_vda, W_gs, W_gl, gamma, 1e-6, W_os, W_ol, H)
    np.testing.assert_array_equal(y_mx, 0.5 * o_s @ W_os.T)
    np.testing.assert_array_equal(y_mx, y)
    # one value off the format's grid in o_s moves the result: the check
    # above is not vacuous
    o_s2 = o_s.copy()
    o_s2[0, 0] = 7.3
    y2 = mxfp8.hybrid_fuse_mxfp8(x, o_s2, o_vda, W_gs, W_gl, gamma, 1e-6, W_os, W_ol, H)
    assert not np.array_equal(y2[0], 0.5 * o_s2[0] @ W_os.T)


def test_fuse_quantizes_the_gated_branch_inputs():
    """Hand-worked case where the gated Softmax output g_s * o_s lies off the
    E4M3 grid, so the MXFP8 fuse must round Z = [g_s o_s | g_l n] before the
    output GEMM.  Zero gate weights give g = 1/2 exactly, o_vda = 0 gives
    n = 0, W_os = I (every 32-block holds one 1: scale 2^-8, code 256, exact),
    so y = quantized(Z)[:, :D] and the rounding can be read off by hand.

    Per 32-element block of a row of Z (OCP MX: e = floor(log2 amax) - 8,
    elements v / 2^e rounded to nearest E4M3, ties to the even code):
      block 0: only 1.15 (o_s = 2.3): e = -8, 1.15 * 256 = 294.4, E4M3
               neighbours 288 and 320 (step 32 in [256, 512)) -> 288 -> 1.125;
      block 1: only 1.28125 (o_s = 2.5625): 328 -> 320 -> 1.25;
      block 2: 3.0 (o_s = 6) and 1.15: e = floor(log2 3) - 8 = -7, 3 * 128 =
               384 exact; 1.15 * 128 = 147.2, neighbours 144 and 160 (step 16
               in [128, 256)) -> 144 -> 1.125;
      block 3: 1.0625 (o_s = 2.125): 272 lies halfway between 256 (code 0x78,
               even) and 288 (0x79) -> ties to even -> 256 -> 1.0.
    Skipping the quantization of Z would give 1.15, 1.28125, 1.15, 1.0625.
    """
    L, D, H = 4, 128, 2
    o_s = np.zeros((L, D))
    o_s[0, 3] = 2.3
    o_s[0, 40] = 2.5625
    o_s[0, 64], o_s[0, 70] = 6.0, 2.3
    o_s[0, 100] = 2.125
    x = np.random.default_rng(4).standard_normal((L, D))
    zeros = np.zeros((D, D))
    y = mxfp8.hybrid_fuse_mxfp8(x, o_s, np.zeros((L, D)), zeros, zeros, np.ones(D), 1e-6,
                                np.eye(D), zeros, H)
    expect = np.zeros((L, D))
    expect[0, 3], expect[0, 40], expect[0, 64], expect[0, 70], expect[0, 100] = (
        1.125, 1.25, 3.0, 1.125, 1.0)
    np.testing.assert_array_equal(y, expect)


# ---------------------------------------------------------------- window Softmax

def _dense_mxfp8_window(q, k, v, T, N, d, scale):
    """One head of the MXFP8 window Softmax written densely, independently of
    the oracle's interval loop: an explicit [L, L] frame mask, operands
    quantized as whole tensors (q, k along d per row; v along the token rows
    per column), and P quantized in blocks of 32 over each full row of L keys
    (masked keys are 0 there; the visible intervals are 32-aligned, so no block
    mixes visible and masked keys)."""
    import oracle
    L = T * N
    vis = np.array([[oracle.frame_visible(r // N, c // N, T) for c in range(L)]
                    for r in range(L)])
    qq = mxfp8.mx_dequantize(*mxfp8.mx_quantize(q))
    kq = mxfp8.mx_dequantize(*mxfp8.mx_quantize(k))
    vc, vs = mxfp8.mx_quantize(v.T)
    vq = mxfp8.mx_dequantize(vc, vs).T
    s2 = np.where(vis, (qq @ kq.T) * scale / np.log(2.0), -np.inf)
    m = np.ceil(s2.max(axis=1, keepdims=True))
    P = np.where(vis, np.exp2(s2 - m), 0.0)
    Pq = mxfp8.mx_dequantize(*mxfp8.mx_quantize(P))
    l = P.sum(axis=1, keepdims=True)
    return (Pq @ vq) / l, (m[:, 0] + np.log2(l[:, 0])) * np.log(2.0)


@pytest.mark.parametrize("T,N,d", [(17, 32, 64), (12, 64, 32), (6, 32, 32)])
def test_window_mxfp8_equals_dense_brute_force(T, N, d):
    rng = np.random.default_rng(T * 7 + N)
    H = 2
    L = T * N
    q, k, v = (rng.standard_normal((L, H * d)) for _ in range(3))
    o, lse = mxfp8.window_attn_mxfp8(q, k, v, T, N, H, d)
    for h in range(H):
        c = slice(h * d, (h + 1) * d)
        o_ref, lse_ref = _dense_mxfp8_window(q[:, c], k[:, c], v[:, c], T, N, d,
                                             1.0 / np.sqrt(d))
        np.testing.assert_allclose(o[:, c], o_ref, rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(lse[h], lse_ref, rtol=1e-11, atol=1e-11)


def test_window_mxfp8_uniform_scores_give_the_window_mean():
    """Special case that reduces to the float64 window Softmax exactly: k = 0
    gives equal scores, so P = 1 everywhere (exact in E4M3 under its block
    scale) and the output is the mean of the visible values; small integers
    in v are exact under any block scale of their block (|v| <= 8), so the
    MXFP8 result equals the unquantized one."""
    import oracle
    rng = np.random.default_rng(11)
    T, N, H, d = 17, 32, 2, 32
    L = T * N
    q = rng.standard_normal((L, H * d))
    k = np.zeros((L, H * d))
    v = rng.integers(-8, 9, (L, H * d)).astype(np.float64)
    o, lse = mxfp8.window_attn_mxfp8(q, k, v, T, N, H, d)
    o_ref, lse_ref = oracle.window_attn(q, k, v, T, N, H, d)
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-12, atol=1e-12)


def test_window_mxfp8_near_the_exact_softmax_on_layer_like_inputs():
    """What the format costs: on inputs drawn like the layer's (q, v ~ N(0, 1),
    keys L2-normalised per token and head) the MXFP8 window Softmax stays
    within a few per cent (max over the output, relative to max |o|) of the
    float64 one (measured 5.4 % max, 3.9 % RMS: the probabilities of these
    nearly flat rows sit in one binade, where E4M3 steps are 1/8, and the
    output is an average of ~1000 values, small against max |v|)."""
    import oracle
    rng = np.random.default_rng(12)
    T, N, H, d = 17, 64, 2, 128
    L = T * N
    q, v = rng.standard_normal((L, H * d)), rng.standard_normal((L, H * d))
    k = rng.standard_normal((L, H, d))
    k = (k / np.linalg.norm(k, axis=2, keepdims=True)).reshape(L, H * d)
    rows = np.arange(0, L, 7)
    o, _ = mxfp8.window_attn_mxfp8_rows(q, k, v, T, N, H, d, rows)
    o_ref, _ = oracle.window_attn_rows(q, k, v, T, N, H, d, rows)
    err = np.abs(o - o_ref).max() / np.abs(o_ref).max()
    assert 1e-3 < err < 0.1
