"""Pins for the M-RoPE oracle (CPU only).

* T10: a text-only prompt gets plain 1-D positions on all three axes ("Qwen2-VL-2B-Instruct --
  LiteRT-LM", M-RoPE note: for text tokens M-RoPE equals sequential positions).
* T9: the tiny prompt [8 text][vision_start][16 image][vision_end][8 text] with grid (1,8,8),
  worked out by hand from the cursor rule (values written out below).
* closed forms for one image / one video run, and the malformed-input errors.
"""
import numpy as np
import pytest

from oracle.mrope_oracle import MRopeError, mrope_index
from resolution_vit_vision_b200 import synthetic as syn


def test_text_only_is_1d():
    ids = np.random.default_rng(0).integers(0, syn.TEXT_VOCAB, 57)
    out, delta = mrope_index(ids, np.zeros((0, 3), np.int32))
    for a in range(3):
        np.testing.assert_array_equal(out[a], np.arange(57))
    assert delta == 0


def test_empty_prompt():
    out, delta = mrope_index(np.zeros(0, np.int32), np.zeros((0, 3)))
    assert out.shape == (3, 0) and delta == 0


def test_tiny_worked_example():
    ids, grid = syn.tiny_prompt(0)
    assert len(ids) == 34
    out, delta = mrope_index(ids, grid)
    # text 0..7 and vision_start 8; the 4x4 merged image starts at 9; the cursor then moves by
    # max(1, 4, 4) = 4 to 13: vision_end 13, text 14..21. delta = 22 - 34 = -12.
    head, tail = list(range(9)), list(range(13, 22))
    t_axis = head + [9] * 16 + tail
    h_axis = head + [9] * 4 + [10] * 4 + [11] * 4 + [12] * 4 + tail
    w_axis = head + [9, 10, 11, 12] * 4 + tail
    np.testing.assert_array_equal(out[0], t_axis)
    np.testing.assert_array_equal(out[1], h_axis)
    np.testing.assert_array_equal(out[2], w_axis)
    assert delta == -12


@pytest.mark.parametrize("n_text,h,w", [(0, 2, 2), (5, 8, 4), (3, 2, 12)])
def test_single_image_closed_form(n_text, h, w):
    hh, ww = h // 2, w // 2
    ids = syn.make_prompt([("text", n_text), ("image", hh * ww), ("text", 2)], 1)
    out, delta = mrope_index(ids, [[1, h, w]])
    base = n_text + 1
    run = np.arange(hh * ww)
    np.testing.assert_array_equal(out[0, base:base + hh * ww], base)
    np.testing.assert_array_equal(out[1, base:base + hh * ww], base + run // ww)
    np.testing.assert_array_equal(out[2, base:base + hh * ww], base + run % ww)
    after = base + max(1, hh, ww)
    np.testing.assert_array_equal(out[:, base + hh * ww], [after] * 3)       # vision_end
    assert delta == -(hh * ww - max(1, hh, ww))
    assert out.max() + 1 - len(ids) == delta


def test_video_time_axis():
    ids = syn.make_prompt([("text", 2), ("video", 3 * 2 * 2), ("text", 1)], 2)
    out, delta = mrope_index(ids, [[3, 4, 4]])
    base = 3
    np.testing.assert_array_equal(out[0, base:base + 12], base + np.repeat(np.arange(3), 4))
    np.testing.assert_array_equal(out[1, base:base + 12], base + np.tile([0, 0, 1, 1], 3))
    np.testing.assert_array_equal(out[2, base:base + 12], base + np.tile([0, 1, 0, 1], 3))
    assert delta == -(12 - 3)


def test_video_prompt_shape_and_delta():
    ids, grids = syn.video_prompt()
    assert len(ids) == 3200
    out, delta = mrope_index(ids, grids)
    # video (4,16,16 merged): 1024 tokens advance the cursor by 16; images (1,24,16): 384 by 24
    assert delta == -((1024 - 16) + 2 * (384 - 24))
    assert out.max() + 1 - 3200 == delta


def test_stray_placeholder_without_vision_start_is_1d():
    ids = np.array([5, syn.IMAGE_TOKEN, 7], np.int32)
    out, delta = mrope_index(ids, np.zeros((0, 3)))
    np.testing.assert_array_equal(out, [[0, 1, 2]] * 3)
    assert delta == 0


@pytest.mark.parametrize("case", ["short", "long", "no_grid", "odd_grid"])
def test_malformed(case):
    if case == "short":
        ids, grid = syn.make_prompt([("image", 15)], 0), [[1, 8, 8]]
    elif case == "long":
        ids, grid = syn.make_prompt([("image", 17)], 0), [[1, 8, 8]]
    elif case == "no_grid":
        ids, grid = syn.make_prompt([("image", 16), ("image", 16)], 0), [[1, 8, 8]]
    else:
        ids, grid = syn.make_prompt([("image", 4)], 0), [[1, 3, 8]]
    with pytest.raises(MRopeError):
        mrope_index(ids, grid)
