"""Writes the full-depth expected values of the three large encoder workloads from the CPU oracle.

    python tests/golden/make_full_depth.py [mixed8] [hires_1792] [video_2img]

Calls only ``oracle/`` (the fp64 encoder) and the seeded input generator; nothing here touches the
CUDA path. For each workload the whole batch goes through the oracle at its full depth (32) and
``full_depth_<workload>.npz`` keeps:

* ``rows``: sampled output rows -- per image (per frame for a video: each frame is its own
  attention segment) its first and last merged token and evenly spaced ones between;
* ``ref_rows``: those rows of the oracle's output, float16 (relative rounding 2^-11, far below the
  encoder tolerance);
* ``proj``: every output row projected on ``N_PROJ`` random +-1 vectors (``projection_matrix``),
  float32, and ``norm``: every row's Euclidean norm -- so a test can check all rows, not only the
  sampled ones, without storing the whole output;
* ``max_abs``: max |output| over the whole batch (the scale of the tolerance max|err| <= 3e-2
  max|ref|).

The oracle's cost is that of the plain definition: about 1e14 fp64 operations for the three
workloads together, tens of minutes on a few cores.
"""
from __future__ import annotations

import os
import sys
import time

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

N_PROJ = 16
PROJ_SEED = 20240919
ROWS_PER_ITEM = {"mixed8": 16, "hires_1792": 64, "video_2img": 16}


def projection_matrix(dim: int) -> np.ndarray:
    """[dim, N_PROJ] of +-1 (Rademacher), seeded: E |R^T e|^2 = N_PROJ |e|^2 for any vector e."""
    rng = np.random.Generator(np.random.PCG64(PROJ_SEED))
    return (rng.integers(0, 2, size=(dim, N_PROJ)) * 2 - 1).astype(np.float64)


def items(grids):
    """(first merged row, merged rows) of every image, or of every frame of a video."""
    out, row = [], 0
    for t, h, w in grids:
        for _ in range(t):
            out.append((row, h * w // 4))
            row += h * w // 4
    return out


def sampled_rows(grids, per_item: int) -> np.ndarray:
    rows = []
    for start, n in items(grids):
        k = min(per_item, n)
        rows.append(start + np.unique(np.round(np.linspace(0, n - 1, k)).astype(np.int64)))
    return np.concatenate(rows).astype(np.int32)


def path_for(name: str) -> str:
    return os.path.join(HERE, f"full_depth_{name}.npz")


def make(name: str) -> None:
    from oracle import vit_oracle as vo
    from resolution_vit_vision_b200 import synthetic as syn
    wl = syn.WORKLOADS[name]
    t0 = time.time()
    wts = syn.make_weights(wl.depth, wl.out_dim, wl.seed)
    patches = syn.make_patches(wl.grids, wl.seed)
    ref = vo.vit_encode(patches, wl.grids, wts)
    rows = sampled_rows(wl.grids, ROWS_PER_ITEM[name])
    R = projection_matrix(wl.out_dim)
    np.savez_compressed(
        path_for(name), workload=np.array(name), depth=np.int32(wl.depth), seed=np.int32(wl.seed),
        grids=np.asarray(wl.grids, np.int32), rows=rows, ref_rows=ref[rows].astype(np.float16),
        proj=(ref @ R).astype(np.float32), norm=np.linalg.norm(ref, axis=1).astype(np.float32),
        max_abs=np.float64(np.abs(ref).max()))
    print(f"{name}: {ref.shape} in {time.time() - t0:.0f} s, max|ref| {np.abs(ref).max():.4g}", flush=True)


if __name__ == "__main__":
    for n in (sys.argv[1:] or ["mixed8", "hires_1792", "video_2img"]):
        make(n)
