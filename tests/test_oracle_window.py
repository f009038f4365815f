"""Pins for the oracle's windowed attention (the Qwen2.5-VL tower), CPU only.

"Qwen2.5-VL-7B-Instruct" (inference-research model record), architecture note: blocks attend
inside 112-px windows (8 x 8 patches of 14 px), except full-attention blocks at depths 7, 15, 23
and 31. What fixes the oracle here, independently of how it builds the windows:

* window counts and sizes of small grids, counted by hand (border windows cut short);
* the members of one window, listed from row / column ranges;
* locality: with one windowed block, perturbing one patch changes exactly the merged tokens of
  its window (hand-listed), and a full-attention block spreads it to every token;
* special cases that reduce to the pinned Qwen2-VL tower: a window covering the frame, and every
  block marked full-attention, give bit-identical outputs;
* the packed order (raster or 2x2-block) does not change the merged tokens.
"""
import numpy as np
import pytest

from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import synthetic as syn


@pytest.mark.parametrize("order", [0, 1])
def test_window_sizes_counted_by_hand(order):
    # 20 x 12 patches, window 8: rows of windows 8, 8, 4 high; columns 8, 4 wide
    assert [len(g) for g in vo.window_groups([(1, 20, 12)], order, 8)] == [64, 32, 64, 32, 32, 16]
    # 6 x 18: one row of windows, 6 high; 8, 8, 2 wide
    assert [len(g) for g in vo.window_groups([(1, 6, 18)], order, 8)] == [48, 48, 12]
    # a video of two 8 x 8 frames: one window per frame, never across frames
    g = vo.window_groups([(2, 8, 8)], order, 8)
    assert [len(x) for x in g] == [64, 64]
    assert g[0].max() < 64 <= g[1].min()
    # two images: windows of the second start after the first image's rows
    g = vo.window_groups([(1, 4, 4), (1, 10, 2)], order, 8)
    assert [len(x) for x in g] == [16, 16, 4]
    assert g[1].min() == 16


def test_window_members_from_ranges():
    # raster order: row of patch (h, w) is h * 12 + w; window 4 = rows 16..19, columns 8..11
    g = vo.window_groups([(1, 20, 12)], 1, 8)
    want = sorted(h * 12 + w for h in range(16, 20) for w in range(8, 12))
    assert g[5].tolist() == want
    want1 = sorted(h * 12 + w for h in range(0, 8) for w in range(8, 12))
    assert g[1].tolist() == want1


@pytest.mark.parametrize("order", [0, 1])
def test_windows_partition_rows_into_whole_merge_groups(order):
    grids = [(1, 20, 12), (3, 6, 10), (1, 2, 2), (1, 18, 4)]
    groups = vo.window_groups(grids, order, 8)
    rows = np.concatenate(groups)
    assert sorted(rows.tolist()) == list(range(syn.n_patches(grids)))
    owner = np.empty(rows.size, np.int64)
    for i, g in enumerate(groups):
        owner[g] = i
    merged = vo.merge_groups(grids, order)                 # [P/4, 4] rows of each merged token
    assert (owner[merged] == owner[merged][:, :1]).all()   # a window never splits a merge group
    frame_of = np.repeat(np.arange(len(vo.segments(grids))), [s[1] for s in vo.segments(grids)])
    for g in groups:
        assert np.unique(frame_of[g]).size == 1             # a window never spans two frames


def test_window_rejects_odd_side():
    with pytest.raises(ValueError):
        vo.window_groups([(1, 8, 8)], 0, 7)


def _encode(patches, grids, wts, order=0, **kw):
    return vo.vit_encode(patches, grids, wts, eps=1e-6, patch_order=order, **kw)


def test_locality_of_one_windowed_block():
    grids = [(1, 20, 12)]
    wts = syn.make_weights(1, 64, 31, affine=True)
    base = syn.bf16_bits_to_f64(syn.make_patches(grids, 31))
    bumped = base.copy()
    bumped[9 * 12 + 3] += 0.5                               # raster order: patch (h, w) = (9, 3)
    a = _encode(base, grids, wts, order=1, window=8)
    b = _encode(bumped, grids, wts, order=1, window=8)
    changed = np.nonzero(np.abs(a - b).max(axis=1) > 0)[0].tolist()
    # its window spans h 8..15, w 0..7: merged rows bh 4..7, columns bw 0..3 of a 10 x 6 grid
    assert changed == [24, 25, 26, 27, 30, 31, 32, 33, 36, 37, 38, 39, 42, 43, 44, 45]
    c = _encode(base, grids, wts, order=1, window=8, full_blocks=(0,))
    d = _encode(bumped, grids, wts, order=1, window=8, full_blocks=(0,))
    assert (np.abs(c - d).max(axis=1) > 0).all()           # full attention reaches every token


@pytest.mark.parametrize("order", [0, 1])
def test_special_cases_reduce_to_the_full_attention_tower(order):
    grids = [(1, 10, 14), (2, 4, 6)]
    wts = syn.make_weights(2, 64, 32, affine=True)
    p = syn.bf16_bits_to_f64(syn.make_patches(grids, 32))
    full = _encode(p, grids, wts, order)
    np.testing.assert_array_equal(_encode(p, grids, wts, order, window=14), full)       # one window
    np.testing.assert_array_equal(_encode(p, grids, wts, order, window=8, full_blocks=(0, 1)), full)
    win = _encode(p, grids, wts, order, window=8)
    assert np.abs(win - full).max() > 1e-6                  # and the windows do change the result


def test_windowed_raster_equals_block_order():
    grids = [(1, 20, 12), (1, 6, 10)]
    wts = syn.make_weights(2, 64, 33)
    raw = syn.bf16_bits_to_f64(syn.make_patches(grids, 33))         # taken as raster order
    rows, start = [], 0
    for t, h, w in grids:
        fh, fw = vo.frame_positions(h, w, 0)
        rows.append(start + fh * w + fw)
        start += h * w
    block = raw[np.concatenate(rows)]
    a = _encode(block, grids, wts, 0, window=8, full_blocks=(1,))
    b = _encode(raw, grids, wts, 1, window=8, full_blocks=(1,))
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12 * np.abs(a).max())


def test_grouped_attention_on_segments_and_permuted_groups():
    rng = np.random.Generator(np.random.PCG64(34))
    P = 40
    q, k, v = (rng.standard_normal((P, vo.HEADS, vo.HEAD_DIM)) for _ in range(3))
    segs = [(0, 12, 0, 0), (12, 28, 0, 0)]
    np.testing.assert_array_equal(vo.grouped_attention(q, k, v, [np.arange(12), np.arange(12, 40)]),
                                  vo.varlen_attention(q, k, v, segs))
    perm = rng.permutation(P)
    inv = np.argsort(perm)
    # groups given through a permutation: attention of the permuted rows, mapped back
    a = vo.grouped_attention(q[perm], k[perm], v[perm], [inv[:12], inv[12:]]).reshape(P, -1)
    b = vo.varlen_attention(q, k, v, segs)
    np.testing.assert_allclose(a[inv], b, rtol=0, atol=1e-12)
