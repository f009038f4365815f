"""Decoder-side steps on a B200 through the C ABI (include/vit_decoder.h) against the fp64 oracle:
the 3-D M-RoPE rotation of q / k and the scatter of merged vision tokens into the input sequence.

"Qwen2-VL" (ZeroModels Keras docs), Qwen2VLModel table: rope_theta 1e6, mrope_section
(16, 24, 24); "Qwen2.5-VL-7B-Instruct" record: 28 / 4 heads of 128; "Qwen2-VL (Native-Resolution
VLM)" Structure rows 6-10: vision and text tokens form one sequence of width 3584.
Bars: M-RoPE within bf16 rounding of the exact rotation (u |ref| + 1e-5 max|x|); the scatter is a
copy, bit-exact.
"""
import numpy as np
import pytest
import torch

from oracle import decoder_oracle as do
from oracle import mrope_oracle as mo
from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import BF16_REL, bf16_bits_to_torch, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _rope_close(got, ref, x, what):
    err = np.abs(got - ref)
    bound = BF16_REL * np.abs(ref) + 1e-5 * np.abs(x).max()
    assert (err <= bound).all(), f"{what}: max excess {(err - bound).max():.3e}"


@pytest.mark.parametrize("which", ["tiny", "video", "far"])
def test_mrope_apply_7b_heads(which):
    if which == "tiny":
        ids, grids = syn.tiny_prompt(0)
        pos, _ = mo.mrope_index(ids, grids)
    elif which == "video":
        ids, grids = syn.video_prompt(5)
        pos, _ = mo.mrope_index(ids, grids)
    else:   # positions far along a long context: the angle needs more than fp32
        rng = np.random.Generator(np.random.PCG64(81))
        pos = rng.integers(0, 120000, size=(3, 777))
    L = pos.shape[1]
    qb = syn.make_matrix((L, 28 * 128), 82 + L, 1.0).reshape(L, 28, 128)
    kb = syn.make_matrix((L, 4 * 128), 83 + L, 1.0).reshape(L, 4, 128)
    q, k = bf16_bits_to_torch(qb), bf16_bits_to_torch(kb)
    p = torch.from_numpy(np.ascontiguousarray(pos, np.int32)).to(DEV)
    nv.mrope_apply(q, k, p)
    torch.cuda.synchronize()
    _rope_close(to_np(q), do.mrope_apply(qb, pos), do._f64(qb), f"q {which}")
    _rope_close(to_np(k), do.mrope_apply(kb, pos), do._f64(kb), f"k {which}")


def test_mrope_apply_other_head_dim_q_only():
    rng = np.random.Generator(np.random.PCG64(84))
    L, H, D, sec = 300, 3, 64, (8, 12, 12)
    pos = rng.integers(0, 5000, size=(3, L))
    qb = syn.make_matrix((L, H * D), 85, 2.0).reshape(L, H, D)
    q = bf16_bits_to_torch(qb)
    nv.mrope_apply(q, None, torch.from_numpy(pos.astype(np.int32)).to(DEV), sections=sec)
    torch.cuda.synchronize()
    _rope_close(to_np(q), do.mrope_apply(qb, pos, sections=sec), do._f64(qb), "head_dim 64")


def _scatter(ids, table, vision, out_init=None):
    t_ids = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).to(DEV)
    T = bf16_bits_to_torch(table)
    Vt = bf16_bits_to_torch(vision) if vision is not None else None
    out = torch.full((len(ids), table.shape[1]), -3.0, dtype=torch.bfloat16, device=DEV) if out_init is None else out_init
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    nv.scatter_vision_tokens(t_ids, T, Vt, out=out, status=st)
    torch.cuda.synchronize()
    return out.view(torch.int16).cpu().numpy().view(np.uint16), int(st.item())


def test_scatter_video_prompt_full_vocab():
    # the 3200-token video prompt (four 1024-token chunks, the last ragged) into a 152064-row table
    ids, grids = syn.video_prompt(5)
    n_vis = sum(t * h * w // 4 for t, h, w in grids)
    table = syn.make_matrix((152064, 256), 86, 1.0)
    vision = syn.make_matrix((n_vis, 256), 87, 1.0)
    got, st = _scatter(ids, table, vision)
    assert st == 0
    slots = np.nonzero((ids == do.IMAGE_TOKEN_ID) | (ids == do.VIDEO_TOKEN_ID))[0]
    text = np.setdiff1d(np.arange(len(ids)), slots)
    ref = np.empty_like(got)
    ref[slots] = vision
    ref[text] = table[ids[text]]
    np.testing.assert_array_equal(got, ref)
    # and against the oracle's definition
    np.testing.assert_array_equal(do._f64(got), do.scatter_tokens(ids, table, vision))


def test_scatter_decoder_width_small_vocab():
    rng = np.random.Generator(np.random.PCG64(88))
    parts, n_vis = [], 0
    for run in (300, 64, 5, 256, 1100, 1):
        parts.append(rng.integers(0, 2048, size=run))
        parts.append(np.full(run // 2 + 1, do.IMAGE_TOKEN_ID if run % 2 else do.VIDEO_TOKEN_ID))
        n_vis += run // 2 + 1
    ids = np.concatenate(parts).astype(np.int64)
    table = syn.make_matrix((2048, 3584), 89, 1.0)
    vision = syn.make_matrix((n_vis, 3584), 90, 1.0)
    got, st = _scatter(ids, table, vision)
    assert st == 0
    np.testing.assert_array_equal(do._f64(got), do.scatter_tokens(ids, table, vision))


def test_scatter_errors_flag_and_leave_rows():
    I = do.IMAGE_TOKEN_ID
    table = syn.make_matrix((16, 64), 91, 1.0)
    vision = syn.make_matrix((2, 64), 92, 1.0)
    fill = np.full(64, 0xC040, np.uint16)                      # bf16 -3.0
    # three placeholders for two vision tokens: the third is left, the status says so
    got, st = _scatter(np.array([3, I, I, 4, I]), table, vision)
    assert st == nv.VIT_ERR_TOKENS
    np.testing.assert_array_equal(got[:4], np.stack([table[3], vision[0], vision[1], table[4]]))
    np.testing.assert_array_equal(got[4], fill)
    # one placeholder for two vision tokens: every row written, the count mismatch flagged
    got, st = _scatter(np.array([3, I, 4]), table, vision)
    assert st == nv.VIT_ERR_TOKENS
    np.testing.assert_array_equal(got, np.stack([table[3], vision[0], table[4]]))
    # a text id outside the table
    got, st = _scatter(np.array([3, I, 16, I]), table, vision)
    assert st == nv.VIT_ERR_TOKENS
    np.testing.assert_array_equal(got[2], fill)
    np.testing.assert_array_equal(got[3], vision[1])
    # no tokens at all: nothing to do (an empty prompt with vision tokens is a count mismatch)
    got, st = _scatter(np.zeros(0, np.int64), table, None)
    assert st == 0 and got.shape == (0, 64)


def test_scatter_long_prompt_wide_chunks():
    # 40000 tokens: chunks of 96 tokens (three ballots each), placeholders in long and short runs
    rng = np.random.Generator(np.random.PCG64(93))
    ids = rng.integers(0, 500, size=40000)
    runs = rng.integers(0, 40000, size=60)
    for r in runs:
        ids[r:r + int(rng.integers(1, 700))] = do.IMAGE_TOKEN_ID if r % 2 else do.VIDEO_TOKEN_ID
    n_vis = int(((ids == do.IMAGE_TOKEN_ID) | (ids == do.VIDEO_TOKEN_ID)).sum())
    table = syn.make_matrix((500, 64), 94, 1.0)
    vision = syn.make_matrix((n_vis, 64), 95, 1.0)
    got, st = _scatter(ids, table, vision)
    assert st == 0
    np.testing.assert_array_equal(do._f64(got), do.scatter_tokens(ids, table, vision))
