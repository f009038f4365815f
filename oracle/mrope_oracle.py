"""CPU oracle for the decoder's 3-D M-RoPE position ids (pure Python, sequential).

TEST INFRASTRUCTURE ONLY (see ``oracle/vit_oracle.py``): used by ``tests/``, ``smoke()`` and the
benchmark's CPU leg, never by the product path; it shares no code with the CUDA kernel.

Passages followed:

* "Qwen2-VL" (ZeroModels Keras docs), intro: the decoder uses M-RoPE, rotary positions split
  across time / height / width; ``Qwen2VLModel`` table: ``mrope_section`` (16, 24, 24),
  ``spatial_merge_size`` 2, ``image_token_id`` 151655, ``video_token_id`` 151656,
  ``vision_start_token_id`` 151652, ``vision_end_token_id`` 151653.
* "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, "M-RoPE note": for text tokens M-RoPE is the same
  as plain sequential 1-D positions; the 2-D layout of the vision tokens is what differs.
* "Qwen2.5-VL-7B-Instruct" record: tokens per image = pixels / (28*28), i.e. one position per
  merged 2x2 group.

Reading of the rule, which the pages leave open: walk the tokens with a cursor c = (largest id so far) + 1. Every
token outside a vision run, vision_start/end included, gets (c, c, c) and advances c by one.
A vision run starts right after a vision_start whose next token is the image or video id; it
takes the next (t, h, w) from ``grid_thw`` (images and videos in appearance order) and must be
exactly t*(h/2)*(w/2) tokens of that id. Its j-th token gets
(c + j // (h'w'), c + (j // w') % h', c + j % w'), h' = h/2, w' = w/2; afterwards
c += max(t, h', w'). delta = c - L. The (16, 24, 24) sections split the decoder's rotary
frequencies, not the ids, so they do not appear here.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import numpy as np

IMAGE_TOKEN = 151655
VIDEO_TOKEN = 151656
VISION_START = 151652
VISION_END = 151653
SPATIAL_MERGE = 2


class MRopeError(ValueError):
    """Malformed prompt: a vision run whose length does not match its grid, or no grid left."""


def mrope_index(input_ids: Sequence[int], grid_thw) -> Tuple[np.ndarray, int]:
    ids = [int(v) for v in np.asarray(input_ids).reshape(-1)]
    grids = [tuple(int(v) for v in row) for row in np.asarray(grid_thw).reshape(-1, 3)]
    L = len(ids)
    out: List[List[int]] = [[0] * L, [0] * L, [0] * L]
    c = 0
    i = 0
    g = 0
    while i < L:
        opens = (ids[i] == VISION_START and i + 1 < L and ids[i + 1] in (IMAGE_TOKEN, VIDEO_TOKEN))
        # the token itself (text, vision_start, vision_end or a stray placeholder) is 1-D
        for a in range(3):
            out[a][i] = c
        c += 1
        i += 1
        if not opens:
            continue
        if g >= len(grids):
            raise MRopeError(f"vision run at token {i} has no grid left")
        t, h, w = grids[g]
        g += 1
        if t < 1 or h < 2 or w < 2 or h % SPATIAL_MERGE or w % SPATIAL_MERGE:
            raise MRopeError(f"bad grid {(t, h, w)}")
        hh, ww = h // SPATIAL_MERGE, w // SPATIAL_MERGE
        n = t * hh * ww
        tok = ids[i]
        run = 0
        while i + run < L and ids[i + run] == tok:
            run += 1
        if run != n:
            raise MRopeError(f"vision run at token {i} has {run} tokens, grid {(t, h, w)} needs {n}")
        for j in range(n):
            out[0][i + j] = c + j // (hh * ww)
            out[1][i + j] = c + (j // ww) % hh
            out[2][i + j] = c + j % ww
        c += max(t, hh, ww)
        i += n
    return np.array(out, dtype=np.int64), c - L
