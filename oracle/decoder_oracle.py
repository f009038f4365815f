"""CPU oracle for the decoder-side steps that consume the vision encoder's output (fp64, numpy).

TEST INFRASTRUCTURE ONLY: only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU
legs use it; it shares no code with the CUDA path.

Passages followed:

* M-RoPE application. "Qwen2-VL" (ZeroModels Keras docs): the text decoder's rotary embedding is
  split across time / height / width; ``Qwen2VLModel`` table: rope_theta 1e6, mrope_section
  (16, 24, 24). "Qwen2.5-VL-7B-Instruct" (inference-research model record): head_dim 128 (28
  query heads, 4 key/value heads), the t and h indices share the head-dim halves with w.
  "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, M-RoPE note: for text tokens the 3-D positions are
  the same as plain 1-D positions.
* Token scatter. "Qwen2-VL" (ZeroModels Keras docs), several images in one conversation: the
  processor expands each image marker to that image's own token count; "Qwen2-VL (Native-
  Resolution VLM)" Structure table rows 6-10: the merged image tokens and the embedded text tokens
  form one sequence of the decoder's width.

Readings of what the pages leave open:

* head_dim = 2 * sum(sections); frequency j < head_dim / 2 is theta^(-2j / head_dim) and turns
  dims j and j + head_dim/2 as a pair (rotate-half, the decoder's 1-D convention), by the angle
  pos[a] * freq_j, where axis a is t for the first sections[0] frequencies, h for the next
  sections[1], w for the last sections[2];
* the same rotation for q and k; v untouched;
* every image or video placeholder token takes the next merged vision token, in order of
  appearance; every other token takes its row of the embedding table; the number of placeholders
  must equal the number of vision tokens.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np

IMAGE_TOKEN_ID = 151655
VIDEO_TOKEN_ID = 151656
MROPE_THETA = 1.0e6
MROPE_SECTIONS = (16, 24, 24)


def _f64(a) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def mrope_inv_freq(head_dim: int, theta: float = MROPE_THETA) -> np.ndarray:
    """freq_j = theta^(-2j / head_dim), j < head_dim / 2."""
    j = np.arange(head_dim // 2, dtype=np.float64)
    return theta ** (-2.0 * j / head_dim)


def mrope_axis_of_freq(sections: Sequence[int]) -> np.ndarray:
    """Position axis (0 t, 1 h, 2 w) that drives each frequency."""
    return np.concatenate([np.full(int(n), a, np.int64) for a, n in enumerate(sections)])


def mrope_angles(pos: np.ndarray, head_dim: int, sections=MROPE_SECTIONS, theta: float = MROPE_THETA):
    """[L, head_dim / 2] angles: pos[axis(j), l] * freq_j."""
    pos = np.asarray(pos, np.float64).reshape(3, -1)
    if 2 * sum(sections) != head_dim:
        raise ValueError("sections must cover head_dim / 2 frequencies")
    axis = mrope_axis_of_freq(sections)
    return pos[axis].T * mrope_inv_freq(head_dim, theta)[None, :]


def mrope_apply(x, pos, sections=MROPE_SECTIONS, theta: float = MROPE_THETA) -> np.ndarray:
    """x [L, heads, head_dim] -> rotated copy: pair (j, j + head_dim/2) turned by angle[l, j]."""
    x = _f64(x)
    L, H, D = x.shape
    ang = mrope_angles(pos, D, sections, theta)[:, None, :]        # [L, 1, D/2]
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[..., :D // 2], x[..., D // 2:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=-1)


def scatter_tokens(input_ids, embed_table, vision) -> np.ndarray:
    """[L, D]: the k-th image / video placeholder takes vision[k], every other token its embedding."""
    ids = np.asarray(input_ids, np.int64)
    table = np.asarray(embed_table)          # rows are converted only where used (the table is large)
    vis = _f64(vision)
    slots = np.nonzero((ids == IMAGE_TOKEN_ID) | (ids == VIDEO_TOKEN_ID))[0]
    if slots.size != vis.shape[0]:
        raise ValueError(f"{slots.size} placeholders for {vis.shape[0]} vision tokens")
    text = np.setdiff1d(np.arange(ids.size), slots)
    if text.size and (ids[text].min() < 0 or ids[text].max() >= table.shape[0]):
        raise ValueError("token id outside the embedding table")
    out = np.empty((ids.size, table.shape[1]), np.float64)
    out[text] = _f64(table[ids[text]])
    out[slots] = vis
    return out
