"""Window-and-anchor Softmax attention, float64 CPU oracle.  TEST INFRASTRUCTURE ONLY.

Source: "Video DeltaNet" article on 10100.com, 方法概述 item 1
(Sliding-Window Softmax + Boundary Anchors), and the line just before
方法概述 (each query chunk attends to itself and one VAE chunk on each side;
first and last frames are boundary anchors).

* Latent frames are grouped into temporal chunks of 5 (the VAE's temporal
  chunk); chunk c(t) = floor((t - origin) / 5), origin 0 by default.
* A query frame sees a key frame when their chunks differ by at most one
  (a 15-frame window for interior chunks).
* Anchors: every frame sees all tokens of the first and the last latent
  frame, and those two frames see the whole sequence.
* All spatial tokens of a frame share its mask; there is no spatial
  restriction inside the window.
* o = softmax(q k^T * scale) v over the visible keys, per head, with
  scale = 1/sqrt(d) unless given.

``anchors`` is a bit set: 1 = first frame, 2 = last frame.
``origin = 1`` (anchor frames outside the chunk grid) is a study variant.

Context keys: the pages keep every interaction with text or audio tokens as
full Softmax (ai-feeds.com 方法 section; 10100.com 方法概述 item 1).  Reading
taken here: when context keys/values ``ctx_k, ctx_v`` ([M, H*d]) are given,
every video query attends to them in the same softmax as its visible video
keys (one joint normalisation).
"""

import numpy as np


def frame_visible(tq, tk, T, chunk_frames=5, window_chunks=1, anchors=3, origin=0):
    """True when query frame tq may attend to key frame tk."""
    if anchors & 1 and (tq == 0 or tk == 0):
        return True
    if anchors & 2 and (tq == T - 1 or tk == T - 1):
        return True
    cq = (tq - origin) // chunk_frames
    ck = (tk - origin) // chunk_frames
    return abs(cq - ck) <= window_chunks


def visible_key_frames(tq, T, chunk_frames=5, window_chunks=1, anchors=3, origin=0):
    """Ascending list of the key frames query frame tq attends to."""
    return [tk for tk in range(T)
            if frame_visible(tq, tk, T, chunk_frames, window_chunks, anchors, origin)]


def mask_pair_count(T, chunk_frames=5, window_chunks=1, anchors=3, origin=0):
    """Number of (query frame, key frame) pairs that are visible."""
    return sum(len(visible_key_frames(tq, T, chunk_frames, window_chunks, anchors, origin))
               for tq in range(T))


def _softmax_rows(s):
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    z = e.sum(axis=1, keepdims=True)
    return e / z, (m + np.log(z))[:, 0]


def window_attn_rows(q, k, v, T, N, H, d, rows, chunk_frames=5, window_chunks=1,
                     anchors=3, scale=None, origin=0, heads=None, ctx_k=None, ctx_v=None):
    """Window+anchor Softmax for the given query token rows.

    Returns (o [len(rows), H*d], lse [H, len(rows)]) in float64; lse is the
    natural-log sum of exp(scaled scores) over the visible keys (video keys
    and, if given, all context keys).  ``heads`` restricts the computation
    to a subset of heads (others are left 0).
    """
    scale = 1.0 / np.sqrt(d) if scale is None or scale <= 0 else float(scale)
    rows = np.asarray(rows, dtype=np.int64)
    heads = range(H) if heads is None else heads
    out = np.zeros((len(rows), H * d))
    lse = np.zeros((H, len(rows)))
    frames = rows // N
    for tq in np.unique(frames):
        sel = np.nonzero(frames == tq)[0]
        kf = visible_key_frames(int(tq), T, chunk_frames, window_chunks, anchors, origin)
        key_rows = np.concatenate([np.arange(tk * N, (tk + 1) * N) for tk in kf])
        for h in heads:
            c = slice(h * d, (h + 1) * d)
            Q = np.asarray(q[rows[sel], c], dtype=np.float64)
            K = np.asarray(k[key_rows, c], dtype=np.float64)
            V = np.asarray(v[key_rows, c], dtype=np.float64)
            if ctx_k is not None and len(ctx_k) > 0:
                K = np.vstack([K, np.asarray(ctx_k[:, c], dtype=np.float64)])
                V = np.vstack([V, np.asarray(ctx_v[:, c], dtype=np.float64)])
            p, l = _softmax_rows((Q @ K.T) * scale)
            out[sel, c] = p @ V
            lse[h, sel] = l
    return out, lse


def window_attn(q, k, v, T, N, H, d, chunk_frames=5, window_chunks=1, anchors=3,
                scale=None, origin=0, ctx_k=None, ctx_v=None):
    """Window+anchor Softmax for every token.  Returns (o [L, H*d], lse [H, L])."""
    return window_attn_rows(q, k, v, T, N, H, d, np.arange(T * N), chunk_frames,
                            window_chunks, anchors, scale, origin, ctx_k=ctx_k, ctx_v=ctx_v)
