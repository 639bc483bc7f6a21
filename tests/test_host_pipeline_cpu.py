"""Host-side partitioning of HybridLayer.forward_many's pipeline, on CPU.

The first video's inputs arrive in head groups (each group's attention
starts as soon as its columns have landed), and the last video's fuse and
read-back run in row blocks. Both partitions must cover every head and
every token row exactly once, whatever the settings: a gap would leave part
of y uncomputed without any error. The helpers are called unbound on a
plain namespace, so no GPU or library call is involved."""

from types import SimpleNamespace

import pytest

from video_diffusion_hybrid_vda_b200.vdn import HybridLayer


def _groups(H, fill):
    return HybridLayer._head_groups(SimpleNamespace(H=H, FILL_GROUPS=fill))


def _chunks(L, drain):
    return HybridLayer._row_chunks(SimpleNamespace(L=L, DRAIN_BLOCKS=drain))


@pytest.mark.parametrize("H", [1, 2, 3, 4, 5, 6, 7, 12, 24, 48])
@pytest.mark.parametrize("fill", [1, 2, 3, 4, 6, 8, 12, 64])
def test_head_groups_partition_the_heads(H, fill):
    groups = _groups(H, fill)
    assert 1 <= len(groups) <= min(fill, H)
    heads = [h for start, count in groups for h in range(start, start + count)]
    assert heads == list(range(H))  # contiguous, in order, each head once
    assert len({count for _, count in groups}) == 1  # equal groups
    # the largest count of equal groups not above the setting
    assert all(H % n or n > fill for n in range(len(groups) + 1, H + 1))


def test_head_groups_at_the_layer_shape():
    assert _groups(24, 4) == [(0, 6), (6, 6), (12, 6), (18, 6)]
    assert _groups(24, 5) == [(0, 6), (6, 6), (12, 6), (18, 6)]
    assert _groups(7, 4) == [(0, 7)]


@pytest.mark.parametrize("L", [1, 96, 127, 128, 129, 700, 1200, 4032, 102 * 4032])
@pytest.mark.parametrize("drain", [0, 1, 2, 3, 4, 8, 1000])
def test_row_chunks_partition_the_rows(L, drain):
    chunks = _chunks(L, drain)
    assert chunks[0][0] == 0 and chunks[-1][1] == L
    for (a0, a1), (b0, _) in zip(chunks, chunks[1:]):
        assert a1 == b0  # no gap, no overlap
    for r0, r1 in chunks:
        assert r1 > r0
        assert r0 % 128 == 0  # every block starts on a 128-row tile
    assert len(chunks) <= max(1, drain)


def test_row_chunks_at_the_layer_shape():
    L = 102 * 4032
    chunks = _chunks(L, 4)
    assert len(chunks) == 4
    sizes = [r1 - r0 for r0, r1 in chunks]
    assert max(sizes) - min(sizes) <= 128 * 4
