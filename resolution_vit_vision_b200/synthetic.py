"""Seeded synthetic inputs for the Qwen2-VL vision encoder and the M-RoPE index.

This module is shared by the CUDA path's tests, the benchmark and the CPU oracle checks.
It holds random draws and bf16 rounding only: none of the encoder's arithmetic lives here.

Workloads (Qwen2-VL pages: "Qwen2-VL" API table for the tower sizes and special token ids;
the LiteRT-LM Qwen2-VL-2B card for the 672x672 single-image case):

* weights are drawn first, in descriptor order, from ``numpy.random.Generator(PCG64(seed))``:
  every matrix ~ N(0, 0.02) rounded to bf16; biases 0, LayerNorm gamma 1 and beta 0, unless
  ``affine=True``, which draws biases and beta ~ N(0, 0.02) and gamma ~ 1 + N(0, 0.1) so the
  bias and affine paths are exercised;
* patches come from a second generator seeded ``seed + 1000``: U[-1, 1] rounded to bf16,
  shape [P, 1176] with P = sum over images of t*h*w.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Sequence, Tuple

import numpy as np

WIDTH = 1280          # vision tower width ("vision_embed_dim")
HEADS = 16            # vision attention heads
HEAD_DIM = 80         # 1280 / 16
MLP = 5120            # vision_mlp_ratio 4
PATCH_K = 1176        # 3 channels x 2 frames x 14 x 14
MERGE_K = 4 * WIDTH   # 2x2 merge groups four tokens

IMAGE_TOKEN = 151655
VIDEO_TOKEN = 151656
VISION_START = 151652
VISION_END = 151653
TEXT_VOCAB = 151643   # plain text ids are drawn from [0, 151643)

LAYER_KEYS = ("ln1_w", "ln1_b", "qkv_w", "qkv_b", "proj_w", "proj_b",
              "ln2_w", "ln2_b", "fc1_w", "fc1_b", "fc2_w", "fc2_b")

LAYER_SHAPES = {
    "ln1_w": (WIDTH,), "ln1_b": (WIDTH,),
    "qkv_w": (3 * WIDTH, WIDTH), "qkv_b": (3 * WIDTH,),
    "proj_w": (WIDTH, WIDTH), "proj_b": (WIDTH,),
    "ln2_w": (WIDTH,), "ln2_b": (WIDTH,),
    "fc1_w": (MLP, WIDTH), "fc1_b": (MLP,),
    "fc2_w": (WIDTH, MLP), "fc2_b": (WIDTH,),
}


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    grids: Tuple[Tuple[int, int, int], ...]   # (t, h, w) in patch units, H x W image -> (1, H/14, W/14)
    depth: int
    out_dim: int
    seed: int
    description: str


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", ((1, 8, 8),), 2, 1536, 0,
                     "one 112x112 image, grid (1,8,8), depth 2, out 1536"),
    "2b_448": Workload("2b_448", ((1, 32, 32),), 32, 1536, 2,
                       "Qwen2-VL-2B-shaped tower, one 448x448 image, grid (1,32,32)"),
    "mixed8": Workload("mixed8", ((1, 32, 32), (1, 48, 48), (1, 16, 64), (1, 72, 24),
                                  (1, 64, 40), (1, 24, 24), (1, 80, 56), (1, 40, 100)), 32, 3584, 1,
                       "8 mixed-aspect images packed varlen, Qwen2-VL-7B-shaped tower (out 3584)"),
    "hires_1792": Workload("hires_1792", ((1, 128, 128),), 32, 3584, 4,
                           "one 1792x1792 image, grid (1,128,128), 16384 patches"),
    "video_2img": Workload("video_2img", ((4, 32, 32), (1, 48, 32), (1, 48, 32)), 32, 3584, 5,
                           "8 frames 448x448 (grid (4,32,32)) plus two 672x448 images"),
}


# ----------------------------------------------------------------------------------------------
# bf16 helpers (round to nearest even); values travel as uint16 bit patterns.
# ----------------------------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


def n_patches(grids: Sequence[Tuple[int, int, int]]) -> int:
    return int(sum(t * h * w for t, h, w in grids))


# ----------------------------------------------------------------------------------------------
# weights
# ----------------------------------------------------------------------------------------------
def make_weights(depth: int, out_dim: int, seed: int, affine: bool = False,
                 std: float = 0.02) -> Dict[str, object]:
    """Vision-tower weights as bf16 bit patterns (uint16), nn.Linear [out, in] row-major.

    Returns {"pe_w", "pe_b" (None), "layers": [dict per layer], "lnq_w", "lnq_b",
    "m0_w", "m0_b", "m2_w", "m2_b"}.
    """
    rng = np.random.Generator(np.random.PCG64(seed))

    def mat(shape):
        return f32_to_bf16_bits(rng.standard_normal(shape, dtype=np.float32) * np.float32(std))

    def bias(n):
        if affine:
            return f32_to_bf16_bits(rng.standard_normal((n,), dtype=np.float32) * np.float32(std))
        return np.zeros((n,), np.uint16)

    def gamma(n):
        if affine:
            return f32_to_bf16_bits(1.0 + rng.standard_normal((n,), dtype=np.float32) * np.float32(0.1))
        return f32_to_bf16_bits(np.ones((n,), np.float32))

    w: Dict[str, object] = {}
    w["pe_w"] = mat((WIDTH, PATCH_K))
    w["pe_b"] = bias(WIDTH) if affine else None
    layers: List[Dict[str, np.ndarray]] = []
    for _ in range(depth):
        L = {}
        for k in LAYER_KEYS:
            shape = LAYER_SHAPES[k]
            if k in ("ln1_w", "ln2_w"):
                L[k] = gamma(shape[0])
            elif len(shape) == 1:
                L[k] = bias(shape[0])
            else:
                L[k] = mat(shape)
        layers.append(L)
    w["layers"] = layers
    w["lnq_w"] = gamma(WIDTH)
    w["lnq_b"] = bias(WIDTH)
    w["m0_w"] = mat((MERGE_K, MERGE_K))
    w["m0_b"] = bias(MERGE_K)
    w["m2_w"] = mat((out_dim, MERGE_K))
    w["m2_b"] = bias(out_dim)
    return w


def make_patches(grids: Sequence[Tuple[int, int, int]], seed: int) -> np.ndarray:
    """Patches [P, 1176] as bf16 bits, U[-1, 1], generator seeded ``seed + 1000``."""
    rng = np.random.Generator(np.random.PCG64(seed + 1000))
    P = n_patches(grids)
    x = rng.uniform(-1.0, 1.0, size=(P, PATCH_K)).astype(np.float32)
    return f32_to_bf16_bits(x)


def make_matrix(shape, seed: int, std: float = 1.0, uniform: bool = False) -> np.ndarray:
    """A generic seeded bf16 matrix (bits) for kernel-level parity cases."""
    rng = np.random.Generator(np.random.PCG64(seed))
    if uniform:
        x = rng.uniform(-std, std, size=shape).astype(np.float32)
    else:
        x = rng.standard_normal(shape, dtype=np.float32) * np.float32(std)
    return f32_to_bf16_bits(x)


def make_f32(shape, seed: int, std: float = 1.0) -> np.ndarray:
    rng = np.random.Generator(np.random.PCG64(seed))
    return (rng.standard_normal(shape, dtype=np.float32) * np.float32(std)).astype(np.float32)


def device_normal_bf16(shape, seed: int, std: float = 1.0, device="cuda"):
    """A seeded N(0, std) bf16 tensor drawn on the device (torch's generator), for inputs too
    large to draw on the host; tests copy what the oracle needs back from it."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = max(1, (1 << 28) // max(1, int(np.prod(shape[1:]))))   # bounded fp32 temporaries
    for r0 in range(0, shape[0], rows):
        r1 = min(shape[0], r0 + rows)
        out[r0:r1] = (torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g, device=device) * std).to(torch.bfloat16)
    return out


# ----------------------------------------------------------------------------------------------
# M-RoPE prompts
# ----------------------------------------------------------------------------------------------
def make_prompt(segments, seed: int) -> np.ndarray:
    """Token ids from a layout list.

    ``segments`` is a list of ("text", n) or ("image"|"video", n_tokens). A vision run is wrapped in
    vision_start ... vision_end. Text ids ~ U[0, 151643), which never collides with the special ids.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    out: List[np.ndarray] = []
    for kind, n in segments:
        if kind == "text":
            out.append(rng.integers(0, TEXT_VOCAB, size=n, dtype=np.int64).astype(np.int32))
        else:
            tok = IMAGE_TOKEN if kind == "image" else VIDEO_TOKEN
            out.append(np.array([VISION_START], np.int32))
            out.append(np.full((n,), tok, np.int32))
            out.append(np.array([VISION_END], np.int32))
    return np.concatenate(out) if out else np.zeros((0,), np.int32)


def decoder_prompt(grids, seed: int, text_between: int = 300) -> Tuple[np.ndarray, np.ndarray]:
    """A prefill prompt that carries a whole encoded batch: text, then each image's merged tokens
    (t*h*w/4 image tokens) followed by ``text_between`` text tokens."""
    segs = [("text", 512)]
    for t, h, w in grids:
        segs += [("image", t * h * w // 4), ("text", text_between)]
    return make_prompt(segs, seed), np.asarray(grids, np.int32).reshape(-1, 3)


def tiny_prompt(seed: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """[8 text][vision_start][16 image tokens][vision_end][8 text] with grid (1,8,8)."""
    ids = make_prompt([("text", 8), ("image", 16), ("text", 8)], seed)
    # make_prompt emits vision_start/end around the run; the text after ends the prompt
    return ids, np.array([[1, 8, 8]], np.int32)


def video_prompt(seed: int = 5) -> Tuple[np.ndarray, np.ndarray]:
    """~3.2K-token interleaved prompt: a (4,32,32) video and two (1,48,32) images."""
    ids = make_prompt([("text", 400), ("video", 1024), ("text", 300), ("image", 384),
                       ("text", 300), ("image", 384), ("text", 402)], seed)
    grids = np.array([[4, 32, 32], [1, 48, 32], [1, 48, 32]], np.int32)
    return ids, grids
