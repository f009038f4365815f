"""CPU oracle for the Qwen2-VL native-resolution vision encoder forward (fp64, numpy).

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this module: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline / reference leg use it. It shares no
code with the CUDA path; the only module both sides use is the seeded input generator
(``resolution_vit_vision_b200.synthetic``), which holds no arithmetic of the method.

Plain and slow on purpose: every step is the textbook definition in float64, in the order the
pages give it, with numpy's matmul as the only library primitive. Passages followed:

* "Qwen2-VL" (ZeroModels Keras docs), API, ``Qwen2VLVisionModel``: patch-embed -> rotary blocks
  -> 2x2 merger; ``Qwen2VLModel`` table: vision depth 32, width 1280, 16 heads, mlp ratio 4,
  patch 14, spatial merge 2, temporal patch 2, 3 input channels.
* "Qwen2-VL (Native-Resolution VLM)" (Neurarch), Structure table rows 2-6 (Patchify 14x14 ->
  2D RoPE -> ViT blocks -> Patch Merger 2x2) and the exported ``PatchMerger`` (LayerNorm, group
  k*k consecutive tokens into one row k*k times as wide, Linear -> GELU -> Linear).
* "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, Conversion notes: the tower is native-resolution
  with packed patches, 2-D rope and cu_seqlens; a single image is one full-attention sequence;
  the patch embed is a Conv3d over 2 temporal frames; the 2x2 merge of raster-ordered patches is
  four strided slices, and ordering is irrelevant as long as each patch keeps its own 2-D rope.

Readings of points the pages leave open:

* pre-norm blocks, LayerNorm eps 1e-6 with gamma/beta, exact-erf GELU;
* patch vector order (c, t, ph, pw), c-major: the Conv3d weight [1280, 3, 2, 14, 14] flattened;
* 2-D rope: theta 10000, f_k = theta^(-2k/40) for k < 20; angle of dim d < 40 is h*f_d for
  d < 20 and w*f_(d-20) otherwise; dims d and d+40 are rotated as a pair (rotate-half);
  applied to q and k; positions are (row, column) in patch units inside the frame;
* one attention segment per (image, temporal index); scale 1/sqrt(80); no mask inside;
* patch_order 0 = 2x2-block order (per frame: bh, bw, dh, dw), 1 = raster order (h, w);
  the merged token concatenates its four patches in (dh, dw) = 00, 01, 10, 11 order;
* merger LayerNorm eps 1e-6 (the same as the tower's), GELU exact.

Windowed attention (the Qwen2.5-VL tower): "Qwen2.5-VL-7B-Instruct" (inference-research model
record), architecture note: the same 32-block, 1280-wide tower as Qwen2-VL, but its blocks attend
inside windows of 112 px, except four full-attention blocks at depths 7, 15, 23 and 31. Readings:

* a window is 112 / 14 = 8 x 8 patches, tiled from the frame's top-left corner; windows on the
  bottom and right borders are cut short (no padding tokens take part in the softmax);
* window membership of a patch is (frame, h // 8, w // 8); each frame of a video is windowed on
  its own; the window side is even, so a window never splits a 2x2 merge group;
* the depths are 0-based block indices; the full-attention blocks attend per (image, frame) as
  the Qwen2-VL tower does;
* nothing else in the block changes (the page names no other difference), and the merged tokens
  come out in the same order as without windows.
"""
from __future__ import annotations

import math
from typing import Dict, List, Sequence, Tuple

import numpy as np
from scipy.special import erf as _erf

WIDTH = 1280
HEADS = 16
HEAD_DIM = 80
ROPE_THETA = 10000.0
ROPE_PAIRS = 20          # 40 rotary dims per axis -> 20 frequencies


def _f64(bits_or_array) -> np.ndarray:
    """bf16 bit patterns (uint16) or floats -> float64."""
    a = np.asarray(bits_or_array)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ----------------------------------------------------------------------------------------------
# elementary steps
# ----------------------------------------------------------------------------------------------
def linear(x: np.ndarray, w: np.ndarray, b=None) -> np.ndarray:
    """y = x w^T + b, nn.Linear convention (w is [out, in])."""
    y = _f64(x) @ _f64(w).T
    if b is not None:
        y = y + _f64(b)[None, :]
    return y


def patch_embed(patches, pe_w, pe_b=None) -> np.ndarray:
    """Patchify 14x14 (Neurarch Structure table, row 2) as the Conv3d of the LiteRT card's
    Conversion notes: each 3x2x14x14 patch, flattened (c, t, ph, pw), times the flattened
    kernel [1280, 1176]; stride = kernel, so the convolution is one matrix product."""
    return linear(patches, pe_w, pe_b)


def layer_norm(x, gamma, beta, eps: float) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * gamma + beta (biased var)."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps)
    return y * _f64(gamma) + (_f64(beta) if beta is not None else 0.0)


def gelu_erf(x) -> np.ndarray:
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2))."""
    x = _f64(x)
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def rope_inv_freq() -> np.ndarray:
    """f_k = theta^(-2k/40), k = 0..19 (40 rotary dims for the row, 40 for the column)."""
    k = np.arange(ROPE_PAIRS, dtype=np.float64)
    return ROPE_THETA ** (-2.0 * k / 40.0)


def rope_angles(hpos: np.ndarray, wpos: np.ndarray) -> np.ndarray:
    """Angles [S, 40]: dims 0..19 rotate by h*f_k, dims 20..39 by w*f_k."""
    f = rope_inv_freq()
    return np.concatenate([np.outer(hpos.astype(np.float64), f),
                           np.outer(wpos.astype(np.float64), f)], axis=1)


def apply_rope_2d(x: np.ndarray, hpos: np.ndarray, wpos: np.ndarray) -> np.ndarray:
    """Rotate one head's vectors x [S, 80] by each token's own 2-D position.

    Pair (d, d+40), d < 40, turns by angle a_d:
    x'_d = x_d cos a_d - x_{d+40} sin a_d ;  x'_{d+40} = x_{d+40} cos a_d + x_d sin a_d.
    """
    a = rope_angles(hpos, wpos)
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[:, :40], x[:, 40:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=1)


def softmax_rows(z: np.ndarray) -> np.ndarray:
    z = z - z.max(axis=-1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, chunk: int = 2048) -> np.ndarray:
    """Full (non-causal) attention of one segment and one head: softmax(q k^T / sqrt(d)) v."""
    d = q.shape[-1]
    out = np.empty((q.shape[0], v.shape[1]), np.float64)
    for s0 in range(0, q.shape[0], chunk):
        z = (q[s0:s0 + chunk] @ k.T) / math.sqrt(d)
        out[s0:s0 + chunk] = softmax_rows(z) @ v
    return out


# ----------------------------------------------------------------------------------------------
# packing: segments, positions, merge groups
# ----------------------------------------------------------------------------------------------
def check_grid(grids) -> List[Tuple[int, int, int]]:
    g = [tuple(int(v) for v in row) for row in np.asarray(grids).reshape(-1, 3)]
    for t, h, w in g:
        if t < 1 or h < 2 or w < 2 or h % 2 or w % 2:
            raise ValueError(f"grid (t,h,w)=({t},{h},{w}) must have t>=1 and even h,w>=2")
    return g


def segments(grids) -> List[Tuple[int, int, int, int]]:
    """(start_row, length, h, w) per attention segment: one per (image, temporal index)."""
    out, row = [], 0
    for t, h, w in check_grid(grids):
        for _ in range(t):
            out.append((row, h * w, h, w))
            row += h * w
    return out


def frame_positions(h: int, w: int, patch_order: int) -> Tuple[np.ndarray, np.ndarray]:
    """(row, col) of each patch of one h x w frame, in the packed order of that frame."""
    if patch_order == 1:   # raster
        hh, ww = np.meshgrid(np.arange(h), np.arange(w), indexing="ij")
        return hh.reshape(-1), ww.reshape(-1)
    # 2x2-block order: bh, bw, dh, dw (dw fastest)
    bh, bw, dh, dw = np.meshgrid(np.arange(h // 2), np.arange(w // 2), np.arange(2), np.arange(2),
                                 indexing="ij")
    return (2 * bh + dh).reshape(-1), (2 * bw + dw).reshape(-1)


def patch_positions(grids, patch_order: int) -> Tuple[np.ndarray, np.ndarray]:
    hs, ws = [], []
    for t, h, w in check_grid(grids):
        hp, wp = frame_positions(h, w, patch_order)
        for _ in range(t):
            hs.append(hp)
            ws.append(wp)
    return np.concatenate(hs), np.concatenate(ws)


def window_groups(grids, patch_order: int, window: int) -> List[np.ndarray]:
    """Row indices of every attention window: per image, per frame, the windows of window x window
    patches tiled from the frame's top-left corner (border windows cut short) in raster order of
    the windows; inside a window the rows keep their packed order. A patch at (h, w) belongs to
    window (h // window, w // window) of its frame."""
    if window < 2 or window % 2:
        raise ValueError("window side must be even and >= 2 (whole 2x2 merge groups)")
    out, row = [], 0
    for t, h, w in check_grid(grids):
        hp, wp = frame_positions(h, w, patch_order)
        nwh, nww = -(-h // window), -(-w // window)
        key = (hp // window) * nww + (wp // window)
        for _ in range(t):
            for k in range(nwh * nww):
                out.append(row + np.nonzero(key == k)[0])
            row += h * w
    return out


def merge_groups(grids, patch_order: int) -> np.ndarray:
    """Row indices [P/4, 4]: the four patches of each merged token, (dh, dw) = 00, 01, 10, 11,
    merged tokens per image, per frame, in (bh, bw) raster order."""
    groups, row = [], 0
    for t, h, w in check_grid(grids):
        for _ in range(t):
            if patch_order == 0:
                idx = row + np.arange(h * w).reshape(-1, 4)
            else:
                bh, bw = np.meshgrid(np.arange(h // 2), np.arange(w // 2), indexing="ij")
                bh, bw = bh.reshape(-1), bw.reshape(-1)
                cols = [(2 * bh + dh) * w + (2 * bw + dw) for dh in (0, 1) for dw in (0, 1)]
                idx = row + np.stack(cols, axis=1)
            groups.append(idx)
            row += h * w
    return np.concatenate(groups, axis=0)


# ----------------------------------------------------------------------------------------------
# the tower
# ----------------------------------------------------------------------------------------------
def qkv_rope(h_in: np.ndarray, L: Dict, hpos, wpos) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """q, k, v [P, 16, 80] from the LN1 output, with the 2-D rope applied to q and k."""
    qkv = linear(h_in, L["qkv_w"], L["qkv_b"])
    P = qkv.shape[0]
    q = qkv[:, :WIDTH].reshape(P, HEADS, HEAD_DIM)
    k = qkv[:, WIDTH:2 * WIDTH].reshape(P, HEADS, HEAD_DIM)
    v = qkv[:, 2 * WIDTH:].reshape(P, HEADS, HEAD_DIM)
    q = np.stack([apply_rope_2d(q[:, i], hpos, wpos) for i in range(HEADS)], axis=1)
    k = np.stack([apply_rope_2d(k[:, i], hpos, wpos) for i in range(HEADS)], axis=1)
    return q, k, v


def varlen_attention(q, k, v, segs) -> np.ndarray:
    """Block-diagonal attention: each segment attends only to itself. Returns [P, 1280]."""
    P = q.shape[0]
    out = np.zeros((P, HEADS, HEAD_DIM), np.float64)
    for start, n, _, _ in segs:
        sl = slice(start, start + n)
        for i in range(HEADS):
            out[sl, i] = attention(q[sl, i], k[sl, i], v[sl, i])
    return out.reshape(P, WIDTH)


def grouped_attention(q, k, v, groups) -> np.ndarray:
    """Attention inside each group of rows (index arrays; every row in exactly one group): the
    rows of a group attend to each other and to nothing else. Returns [P, 1280]."""
    P = q.shape[0]
    out = np.zeros((P, HEADS, HEAD_DIM), np.float64)
    for idx in groups:
        for i in range(HEADS):
            out[idx, i] = attention(q[idx, i], k[idx, i], v[idx, i])
    return out.reshape(P, WIDTH)


def vit_block(x: np.ndarray, L: Dict, segs, hpos, wpos, eps: float, groups=None) -> np.ndarray:
    """Pre-norm block: x += proj(attn(rope(qkv(LN1 x)))) ; x += fc2(GELU(fc1(LN2 x))).
    Attention per segment, or inside each of ``groups`` (windows) when given."""
    h = layer_norm(x, L["ln1_w"], L["ln1_b"], eps)
    q, k, v = qkv_rope(h, L, hpos, wpos)
    a = varlen_attention(q, k, v, segs) if groups is None else grouped_attention(q, k, v, groups)
    x = x + linear(a, L["proj_w"], L["proj_b"])
    h = layer_norm(x, L["ln2_w"], L["ln2_b"], eps)
    x = x + linear(gelu_erf(linear(h, L["fc1_w"], L["fc1_b"])), L["fc2_w"], L["fc2_b"])
    return x


def merger(x: np.ndarray, grids, weights: Dict, eps: float, patch_order: int) -> np.ndarray:
    """PatchMerger: LN_q, group each 2x2 into one 5120-wide row, Linear -> GELU -> Linear."""
    y = layer_norm(x, weights["lnq_w"], weights["lnq_b"], eps)
    g = merge_groups(grids, patch_order)
    y4 = y[g].reshape(g.shape[0], 4 * WIDTH)
    hdn = gelu_erf(linear(y4, weights["m0_w"], weights["m0_b"]))
    return linear(hdn, weights["m2_w"], weights["m2_b"])


def vit_encode(patches, grids, weights: Dict, depth: int = None, eps: float = 1e-6,
               patch_order: int = 0, return_hidden: bool = False, window: int = 0,
               full_blocks: Sequence[int] = ()):
    """Patches [P, 1176] + grid_thw -> merged tokens [P/4, out_dim] (float64).
    window > 0: blocks whose index is not in full_blocks attend inside window x window patches."""
    g = check_grid(grids)
    segs = segments(g)
    hpos, wpos = patch_positions(g, patch_order)
    groups = window_groups(g, patch_order, window) if window else None
    depth = len(weights["layers"]) if depth is None else depth
    x = patch_embed(patches, weights["pe_w"], weights.get("pe_b"))
    for l in range(depth):
        windowed = groups is not None and l not in full_blocks
        x = vit_block(x, weights["layers"][l], segs, hpos, wpos, eps, groups if windowed else None)
    out = merger(x, g, weights, eps, patch_order)
    return (out, x) if return_hidden else out

