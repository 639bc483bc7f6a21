"""The window Softmax's host-side work plan (vdn_window_attn_schedule, no GPU)
against the oracle's frame mask.

The kernel launch turns the mask into segments of consecutive query frames
that see the same key frames, each with at most three contiguous key
intervals and 256-row CTA tiles, listed heaviest first.  These tests check,
for many frame counts and mask settings, that the plan covers exactly the
pairs the oracle's mask allows (``oracle.window_attn.visible_key_frames``),
that its tile arithmetic is consistent, and that plans the kernel cannot
hold are refused.
"""

import importlib
import math

import pytest

from tests.parity_util import ensure_built

# the module itself (the package re-exports a function of the same name)
ow = importlib.import_module("oracle.window_attn")


@pytest.fixture(scope="module")
def vdn():
    ensure_built()
    from video_diffusion_hybrid_vda_b200 import vdn as _vdn
    return _vdn


def _check_plan(segs, T, N, cf, wc, anchors):
    # 1. segments partition the query frames, whole frames each
    frames = []
    for g in segs:
        assert g["q0"] % N == 0 and g["q1"] % N == 0 and g["q0"] < g["q1"]
        frames += list(range(g["q0"] // N, g["q1"] // N))
    assert sorted(frames) == list(range(T))
    # 2. every query frame of a segment sees exactly the segment's key frames
    for g in segs:
        keys = g["keys"]
        assert 1 <= g["nint"] <= 3 and len(keys) == g["nint"]
        kf = []
        for k0, k1 in keys:
            assert k0 % N == 0 and k1 % N == 0 and k0 < k1
            kf += list(range(k0 // N, k1 // N))
        # ascending, disjoint and maximal (no two intervals touch)
        assert all(keys[v][1] < keys[v + 1][0] for v in range(len(keys) - 1))
        for tq in range(g["q0"] // N, g["q1"] // N):
            assert kf == ow.visible_key_frames(tq, T, cf, wc, anchors), (tq, keys)
        # 3. tile counts
        assert g["ntiles"] == math.ceil((g["q1"] - g["q0"]) / 256)
        assert g["nkv"] == sum(math.ceil((k1 - k0) / 128) for k0, k1 in keys)
    # 4. segments are maximal: neighbouring frames in different segments see
    #    different keys
    by_start = sorted(segs, key=lambda g: g["q0"])
    for a, b in zip(by_start, by_start[1:]):
        assert a["q1"] == b["q0"]
        assert a["keys"] != b["keys"]
    # 5. launch order: heaviest (most visible keys) first, tiles numbered in
    #    that order
    work = [sum(k1 - k0 for k0, k1 in g["keys"]) for g in segs]
    assert work == sorted(work, reverse=True)
    base = 0
    for g in segs:
        assert g["tile_base"] == base
        base += g["ntiles"]
    # 6. the planned (query, key) token pairs are the mask's
    pairs = sum((g["q1"] - g["q0"]) * sum(k1 - k0 for k0, k1 in g["keys"]) for g in segs)
    assert pairs == ow.mask_pair_count(T, cf, wc, anchors) * N * N


@pytest.mark.parametrize("T", list(range(1, 41)) + [42, 72, 101, 102, 130])
def test_schedule_default_mask(vdn, T):
    """Chunks of 5, one chunk each side, both anchors (the layer's mask)."""
    for N in (1, 7, 4032):
        _check_plan(vdn.window_attn_schedule(T, N), T, N, 5, 1, 3)


@pytest.mark.parametrize("cf,wc,anchors", [
    (5, 0, 3), (5, 2, 3), (5, 1, 0), (5, 1, 1), (5, 1, 2), (3, 1, 3), (1, 1, 3),
    (7, 3, 1), (4, 0, 0),
])
def test_schedule_mask_variants(vdn, cf, wc, anchors):
    for T in (1, 2, 6, 11, 17, 26, 42, 102):
        _check_plan(vdn.window_attn_schedule(T, 96, cf, wc, anchors), T, 96, cf, wc, anchors)


def test_schedule_segments_at_the_layer_shape(vdn):
    """102 frames in chunks of 5 (chunk 20 is frames 100-101): 23 segments,
    the two anchor frames (each sees all 102 frames, launched first), frames
    1-4 (the rest of chunk 0), chunks 1..19, and frame 100 (the ragged last
    chunk without its anchor); an interior chunk sees its 15-frame window
    plus both anchors, three key intervals."""
    N = 4032
    segs = vdn.window_attn_schedule(102, N)
    spans = sorted((g["q0"] // N, g["q1"] // N) for g in segs)
    assert spans == ([(0, 1), (1, 5)] + [(5 * c, 5 * c + 5) for c in range(1, 20)] +
                     [(100, 101), (101, 102)])
    assert [g["keys"] for g in segs[:2]] == [[(0, 102 * N)]] * 2
    mid = next(g for g in segs if g["q0"] == 50 * N)
    assert mid["keys"] == [(0, N), (45 * N, 60 * N), (101 * N, 102 * N)]
    assert mid["ntiles"] == math.ceil(5 * N / 256)


def test_schedule_refuses_what_the_kernel_cannot_hold(vdn):
    # one-frame chunks with anchors: every interior frame has its own key set,
    # more than the kernel's 256-segment table
    with pytest.raises(vdn.VdnError) as e:
        vdn.window_attn_schedule(300, 16, 1, 1, 3)
    assert e.value.code == 2  # VDN_ERR_UNSUPPORTED
    with pytest.raises(vdn.VdnError) as e:
        vdn.window_attn_schedule(10, 16, 0, 1, 3)  # chunk_frames < 1
    assert e.value.code == 1  # VDN_ERR_INVALID_ARG
    with pytest.raises(vdn.VdnError) as e:
        vdn.window_attn_schedule(10, 16, 5, 1, 4)  # anchors is a 2-bit set
    assert e.value.code == 1
