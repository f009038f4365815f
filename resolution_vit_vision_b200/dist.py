"""Data-parallel sharding of a packed image batch across ranks (one process per GPU).

Attention never crosses an image (each (image, frame) is its own segment) and the 2x2 merge is
per image, so the images of a batch are independent problems: a batch shards across ranks with
no exchange on the data path. This module holds the host side of that: a longest-processing-time
(LPT) partition of the images by their encoder cost, the per-rank slices, and the max-over-ranks
reduction of step times. Any exchange of the merged tokens (if a consumer wants them on one
rank) happens after the encoder and is not part of the hot path.
"""
from __future__ import annotations

from typing import List, Sequence, Tuple

import torch
import torch.distributed as dist

WIDTH = 1280


def _window_sizes(h: int, w: int, window: int) -> List[int]:
    """Patches per attention window of one h x w frame: window x window tiles from the top-left
    corner, border windows cut short."""
    return [min(window, h - a) * min(window, w - b) for a in range(0, h, window) for b in range(0, w, window)]


def image_cost(grid: Sequence[int], depth: int = 32, window: int = 0, full_blocks: Sequence[int] = ()) -> float:
    """Encoder FLOPs of one image: the per-patch linear layers plus its block-diagonal attention
    (4 * S^2 * 1280 per layer and segment). Segments are the frames (S = h*w), or, in the windowed
    tower's blocks outside ``full_blocks``, the windows of ``window`` x ``window`` patches."""
    t, h, w = (int(v) for v in grid)
    P = t * h * w
    linear = 2.0 * P * (1176 * 1280) + depth * 2.0 * P * (1280 * 3840 + 1280 * 1280 + 2 * 1280 * 5120)
    full = t * 4.0 * (h * w) ** 2 * WIDTH
    if not window:
        return linear + depth * full
    n_full = sum(1 for l in range(depth) if l in full_blocks)
    windowed = t * 4.0 * sum(s * s for s in _window_sizes(h, w, window)) * WIDTH
    return linear + n_full * full + (depth - n_full) * windowed


def lpt_partition(grids: Sequence[Sequence[int]], world: int, depth: int = 32, window: int = 0,
                  full_blocks: Sequence[int] = ()) -> List[List[int]]:
    """Image indices per rank: images taken largest cost first, each to the currently least
    loaded rank (ties to the lower rank; equal costs keep their batch order). Every rank computes
    the same partition from the same grids, with no communication."""
    if world < 1:
        raise ValueError("world must be >= 1")
    cost = [image_cost(g, depth, window, full_blocks) for g in grids]
    order = sorted(range(len(grids)), key=lambda i: (-cost[i], i))
    load = [0.0] * world
    parts: List[List[int]] = [[] for _ in range(world)]
    for i in order:
        r = min(range(world), key=lambda k: (load[k], k))
        parts[r].append(i)
        load[r] += cost[i]
    return [sorted(p) for p in parts]


def shard(grids: Sequence[Sequence[int]], rank: int, world: int, depth: int = 32, window: int = 0,
          full_blocks: Sequence[int] = ()) -> Tuple[List[int], List[Tuple[int, int, int]], List[Tuple[int, int]]]:
    """This rank's images: (indices, their grids, their patch-row ranges in the packed batch)."""
    starts = [0]
    for t, h, w in grids:
        starts.append(starts[-1] + int(t) * int(h) * int(w))
    idx = lpt_partition(grids, world, depth, window, full_blocks)[rank]
    return idx, [tuple(int(v) for v in grids[i]) for i in idx], [(starts[i], starts[i + 1]) for i in idx]


def max_over_ranks(value: float, device=None) -> float:
    """The maximum of a per-rank number (step time) over all ranks; the value itself when no
    process group is initialised."""
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())
