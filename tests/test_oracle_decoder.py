"""Pins for the oracle's decoder-side steps (CPU only): the 3-D M-RoPE rotation of q / k and the
scatter of merged vision tokens into the decoder's input sequence.

What fixes the oracle, independently of how it computes:

* the printed configuration (tests/golden/decoder_config.json): theta 1e6, sections (16, 24, 24),
  head_dim 128 = 2 * (16 + 24 + 24), 28 / 4 heads of the 7B decoder, 1536 / 12 of the 2B;
* hand-worked rotations of unit vectors: the pair (j, j + 64), the direction of the turn and the
  frequency theta^(-2j/128) at j = 0, 16 and 63, each driven by its own axis;
* the section map, counted by hand: moving only the t (h, w) position changes exactly dims 0..15
  and 64..79 (16..39 and 80..103; 40..63 and 104..127);
* "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, M-RoPE note: for text tokens (t = h = w) it is plain
  1-D RoPE; position 0 is the identity; norms are kept; scores depend only on position offsets;
* the scatter: a hand-worked sequence, and a placeholder count that does not match is rejected.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import decoder_oracle as do
from oracle import mrope_oracle as mo
from resolution_vit_vision_b200 import synthetic as syn

HERE = os.path.dirname(__file__)
CFG = json.load(open(os.path.join(HERE, "golden", "decoder_config.json")))


def test_printed_configuration():
    assert do.MROPE_THETA == CFG["rope_theta"]
    assert list(do.MROPE_SECTIONS) == CFG["mrope_section"]
    assert 2 * sum(CFG["mrope_section"]) == CFG["head_dim_7b"]
    assert CFG["embed_dim_7b"] == CFG["num_heads_7b"] * CFG["head_dim_7b"]
    assert CFG["embed_dim_2b"] // CFG["num_heads_2b"] == 128          # head_dim None -> width / heads
    assert (do.IMAGE_TOKEN_ID, do.VIDEO_TOKEN_ID) == (CFG["image_token_id"], CFG["video_token_id"])


def _unit(d):
    x = np.zeros((1, 1, 128))
    x[0, 0, d] = 1.0
    return x


def test_hand_worked_rotations():
    # dim 0 at t = 1: frequency 1 rad -> (cos 1, sin 1) on dims (0, 64)
    y = do.mrope_apply(_unit(0), np.array([[1], [0], [0]]))[0, 0]
    assert y[0] == pytest.approx(math.cos(1.0), abs=1e-15) and y[64] == pytest.approx(math.sin(1.0), abs=1e-15)
    assert np.count_nonzero(np.abs(y) > 1e-15) == 2
    # dim 64 (the pair's second half) at t = 1 turns the other way round: (-sin 1, cos 1) on (0, 64)
    y = do.mrope_apply(_unit(64), np.array([[1], [0], [0]]))[0, 0]
    assert y[0] == pytest.approx(-math.sin(1.0), abs=1e-15) and y[64] == pytest.approx(math.cos(1.0), abs=1e-15)
    # dim 16 is the first h frequency: 1e6^(-32/128) = 10^-1.5 = 0.0316227766...; h = 2
    y = do.mrope_apply(_unit(16), np.array([[7], [2], [9]]))[0, 0]
    a = 2 * 0.031622776601683794
    assert y[16] == pytest.approx(math.cos(a), abs=1e-15) and y[80] == pytest.approx(math.sin(a), abs=1e-15)
    # dim 63 is the last w frequency: 1e6^(-126/128) = 10^-5.90625 = 1.2409377607517195e-06; w = 5
    y = do.mrope_apply(_unit(63), np.array([[7], [3], [5]]))[0, 0]
    a = 5 * 1.2409377607517195e-06
    assert y[63] == pytest.approx(math.cos(a), abs=1e-15) and y[127] == pytest.approx(math.sin(a), abs=1e-15)


@pytest.mark.parametrize("axis,dims", [(0, list(range(0, 16)) + list(range(64, 80))),
                                       (1, list(range(16, 40)) + list(range(80, 104))),
                                       (2, list(range(40, 64)) + list(range(104, 128)))])
def test_section_map_counted_by_hand(axis, dims):
    rng = np.random.Generator(np.random.PCG64(41))
    x = rng.standard_normal((1, 3, 128))
    p0 = np.array([[3], [5], [11]])
    p1 = p0.copy()
    p1[axis, 0] += 4
    moved = np.nonzero(np.abs(do.mrope_apply(x, p0) - do.mrope_apply(x, p1)).max(axis=(0, 1)) > 1e-12)[0]
    assert moved.tolist() == dims


def test_text_tokens_are_plain_1d_rope_and_identities():
    rng = np.random.Generator(np.random.PCG64(42))
    L = 9
    x = rng.standard_normal((L, 2, 128))
    l = np.arange(L)
    got = do.mrope_apply(x, np.stack([l, l, l]))
    # plain 1-D rope in complex form: z_j = x_j + i x_(j+64) times e^(i l theta^(-j/64))
    f = np.exp(-np.arange(64) / 64.0 * np.log(1.0e6))
    z = (x[..., :64] + 1j * x[..., 64:]) * np.exp(1j * l[:, None, None] * f[None, None, :])
    np.testing.assert_allclose(got, np.concatenate([z.real, z.imag], -1), rtol=0, atol=1e-13)
    np.testing.assert_array_equal(do.mrope_apply(x, np.zeros((3, L))), x)                 # position 0
    np.testing.assert_allclose(np.linalg.norm(got, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


def test_scores_depend_only_on_offsets():
    rng = np.random.Generator(np.random.PCG64(43))
    q, k = rng.standard_normal((1, 1, 128)), rng.standard_normal((1, 1, 128))
    pq, pk = np.array([[4], [9], [2]]), np.array([[1], [3], [7]])
    shift = np.array([[5], [-2], [13]])
    s0 = (do.mrope_apply(q, pq) * do.mrope_apply(k, pk)).sum()
    s1 = (do.mrope_apply(q, pq + shift) * do.mrope_apply(k, pk + shift)).sum()
    assert s0 == pytest.approx(s1, abs=1e-12)


def test_scatter_hand_worked():
    I, V = do.IMAGE_TOKEN_ID, do.VIDEO_TOKEN_ID
    table = np.arange(10 * 4, dtype=np.float64).reshape(10, 4)
    vis = -np.arange(1, 13, dtype=np.float64).reshape(3, 4)
    out = do.scatter_tokens([5, I, I, 7, V, 2], table, vis)
    np.testing.assert_array_equal(out, np.stack([table[5], vis[0], vis[1], table[7], vis[2], table[2]]))
    with pytest.raises(ValueError):
        do.scatter_tokens([5, I, 7], table, vis)                 # one slot, three vision tokens
    with pytest.raises(ValueError):
        do.scatter_tokens([11, I, I, I], table, vis)             # id outside the table


def test_scatter_slots_are_the_mrope_vision_runs():
    # the slots the scatter fills are exactly the tokens M-RoPE gives 3-D (non-diagonal) positions
    ids, grids = syn.video_prompt(5)
    pos, _ = mo.mrope_index(ids, grids)
    slots = np.nonzero((ids == do.IMAGE_TOKEN_ID) | (ids == do.VIDEO_TOKEN_ID))[0]
    n_vis = sum(t * h * w // 4 for t, h, w in grids)
    assert slots.size == n_vis
    table = np.zeros((151657, 2))
    out = do.scatter_tokens(ids, table, np.ones((n_vis, 2)))
    assert (np.nonzero(out[:, 0])[0] == slots).all()
    text = np.setdiff1d(np.arange(ids.size), slots)
    assert (pos[0, text] == pos[1, text]).all() and (pos[1, text] == pos[2, text]).all()
