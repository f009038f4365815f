"""Measures, from the oracle alone, how far two exact implementations of the fp8 tower drift apart,
and writes the tolerance of the fp8 tower's parity tests to ``fp8_drift.json``.

    python tests/golden/fp8_drift.py

Every activation that enters an E4M3 product is rounded to 3 mantissa bits: a step function of
its input. Two implementations of the same definition that differ only in the rounding of earlier
arithmetic take a different code wherever a value lies near a step, and the differences then
grow through the blocks. The CUDA path differs from the fp64 oracle in exactly such roundings:
q, k, v, the attention output and the MLP hidden layer are kept in bf16 between kernels, and the
LayerNorms run in fp32. The oracle's own variant with those roundings
(``vit_encode_fp8(..., ln_float32=True, bf16_storage=True)``) is compared with the plain oracle;
the tolerance is that drift with a factor of two: max|err| <= 2 * drift_err * max|ref| and
per-token cosine >= 1 - 2 * (1 - drift_cos). Measured at depth 2 (two workloads; the larger
drift sets the bar) and at depth 32 on the Qwen2-VL-2B-shaped 448 x 448 image (seed 2), where the
run also records how close the fp8 tower stays to the unquantised tower (the pages' 8-bit tower:
correlation 0.90, "Qwen2-VL-2B-Instruct -- LiteRT-LM").
"""
from __future__ import annotations

import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

DEPTH2_CASES = (((1, 8, 8),), ((1, 10, 14), (2, 4, 6), (1, 16, 12)))   # seed 34, out 1536


def stats(a, b):
    cos = (a * b).sum(1) / (np.linalg.norm(a, axis=1) * np.linalg.norm(b, axis=1))
    return {"max_err_rel": float(np.abs(a - b).max() / np.abs(b).max()), "min_cos": float(cos.min()),
            "mean_cos": float(cos.mean()), "corr": float(np.corrcoef(a.ravel(), b.ravel())[0, 1])}


def bar(drifts):
    return {"max_err_rel": 2 * max(d["max_err_rel"] for d in drifts),
            "min_cos": 1 - 2 * max(1 - d["min_cos"] for d in drifts)}


def main():
    from oracle import fp8_oracle as fo
    from oracle import vit_oracle as vo
    from resolution_vit_vision_b200 import synthetic as syn
    out = {"depth2": {"cases": [], "seed": 34, "out_dim": 1536}}
    for grids in DEPTH2_CASES:
        w = syn.make_weights(2, 1536, 34)
        p = syn.make_patches(grids, 34)
        a = fo.vit_encode_fp8(p, grids, w)
        b = fo.vit_encode_fp8(p, grids, w, ln_float32=True, bf16_storage=True)
        out["depth2"]["cases"].append({"grids": [list(g) for g in grids], "drift": stats(b, a)})
    out["depth2"]["bar"] = bar([c["drift"] for c in out["depth2"]["cases"]])
    wl = syn.WORKLOADS["2b_448"]
    w = syn.make_weights(wl.depth, wl.out_dim, wl.seed)
    p = syn.make_patches(wl.grids, wl.seed)
    a = fo.vit_encode_fp8(p, wl.grids, w)
    b = fo.vit_encode_fp8(p, wl.grids, w, ln_float32=True, bf16_storage=True)
    ref = vo.vit_encode(p, wl.grids, w)
    d = stats(b, a)
    out["depth32"] = {"workload": "2b_448", "depth": wl.depth, "seed": wl.seed, "drift": d, "bar": bar([d]),
                      "fp8_vs_unquantised_tower": stats(a, ref)}
    json.dump(out, open(os.path.join(HERE, "fp8_drift.json"), "w"), indent=1)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
