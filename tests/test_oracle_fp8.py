"""Pins of the fp8 (E4M3) oracle (no GPU): the rounding, the scales, the quantiser and the tower.

The E4M3 rounding is pinned against torch's float8_e4m3fn conversion (a library routine) and
hand-worked values; the scale rule against a brute-force search; the tower against the bf16
tower it reduces to when quantisation is the identity, and against the accuracy the pages give
for an 8-bit tower ("Qwen2-VL-2B-Instruct -- LiteRT-LM", correlation note: 0.90 with int8
weights).
"""
import math

import numpy as np
import pytest
import torch

from oracle import fp8_oracle as fo
from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import synthetic as syn


def test_round_e4m3_hand_values():
    cases = {
        1.0: 1.0, 1.0625: 1.0,          # midpoint of 1 and 1.125 -> even mantissa (1.000)
        1.1875: 1.25,                   # midpoint of 1.125 (odd) and 1.25 (even)
        1.2: 1.25, 448.0: 448.0, 440.0: 448.0, 416.0: 416.0, 432.0: 448.0,   # 432: tie, 448 even
        2.0 ** -6: 2.0 ** -6,           # smallest normal
        2.0 ** -9: 2.0 ** -9,           # smallest subnormal
        3 * 2.0 ** -10: 2.0 ** -8,      # tie between 2^-9 (odd) and 2^-8 (even)
        2.0 ** -11: 0.0,                # below half the smallest subnormal
        -3.3: -3.25, 0.0: 0.0,
    }
    for x, want in cases.items():
        assert fo.round_e4m3(x) == want, (x, fo.round_e4m3(x), want)


def test_round_e4m3_matches_torch_float8():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(300_000) * np.exp(rng.uniform(-14, 6, 300_000))
    x = np.concatenate([np.clip(x, -448, 448), np.arange(-448, 449, 0.0625)])
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(fo.round_e4m3(x), want)


def test_pow2_scale_hand_values_and_brute_force():
    assert fo.pow2_scale(448.0) == 1.0
    assert fo.pow2_scale(np.nextafter(448.0, 1e9)) == 2.0
    assert fo.pow2_scale(224.0) == 0.5
    assert fo.pow2_scale(1.0) == 2.0 ** -8          # 1 <= 1.75 = 448 * 2^-8, 1 > 448 * 2^-9
    assert fo.pow2_scale(0.0) == 2.0 ** -126
    rng = np.random.default_rng(1)
    a = np.abs(rng.standard_normal(20_000)) * np.exp(rng.uniform(-60, 60, 20_000))
    a = np.concatenate([a, 448.0 * 2.0 ** np.arange(-60, 60)])   # exact boundaries
    s = fo.pow2_scale(a)
    for ai, si in zip(a[::97], s[::97]):
        e = math.ceil(math.log2(ai / 448.0)) - 2
        while ai > 448.0 * 2.0 ** e:
            e += 1
        assert si == 2.0 ** max(e, -126), (ai, si, e)
    assert np.all(a <= 448.0 * s) and np.all(a > 224.0 * s)


def test_quantize_rows_properties():
    rng = np.random.default_rng(2)
    x = syn.f32_to_bf16_bits(rng.standard_normal((64, 1280)).astype(np.float32) *
                             np.exp(rng.uniform(-8, 8, (64, 1))).astype(np.float32))
    q, s = fo.quantize_rows(x)
    xf = vo._f64(x)
    amax = np.abs(q).max(axis=1)
    assert np.all(amax <= 448.0) and np.all(amax >= 224.0)          # the scale uses the top binade
    deq = fo.dequantize_rows(q, s)
    rel = np.abs(deq - xf) / np.abs(xf)
    big = np.abs(xf) >= 2.0 ** -6 * s[:, None]                     # normal E4M3 range
    assert rel[big].max() <= 2.0 ** -4                             # half a step of 3 mantissa bits
    # re-quantising dequantised values reproduces them (the scale may halve when a row's max
    # rounded down onto 224 s, which doubles its codes but not their values)
    np.testing.assert_array_equal(fo.dequantize_rows(*fo.quantize_rows(deq)), deq)


def test_fp8_tower_reduces_to_bf16_tower_when_quantisation_is_exact(monkeypatch):
    # with the rounding replaced by the identity, the fp8 tower is the bf16 tower exactly
    wl = syn.WORKLOADS["tiny"]
    w = syn.make_weights(2, wl.out_dim, 3)
    p = syn.make_patches(wl.grids, 3)
    monkeypatch.setattr(fo, "round_e4m3", lambda x: np.asarray(x, np.float64))
    np.testing.assert_allclose(fo.vit_encode_fp8(p, wl.grids, w), vo.vit_encode(p, wl.grids, w), rtol=1e-12,
                               atol=1e-12)


def test_fp8_tower_accuracy_against_bf16_tower():
    # the 8-bit tower stays close to the unquantised one: the pages report correlation 0.90 for
    # their int8 tower; this scheme keeps a per-token cosine above 0.99 on the tiny workload
    wl = syn.WORKLOADS["tiny"]
    w = syn.make_weights(wl.depth, wl.out_dim, wl.seed)
    p = syn.make_patches(wl.grids, wl.seed)
    a, b = fo.vit_encode_fp8(p, wl.grids, w), vo.vit_encode(p, wl.grids, w)
    cos = (a * b).sum(1) / np.linalg.norm(a, axis=1) / np.linalg.norm(b, axis=1)
    assert cos.min() > 0.99
    assert np.corrcoef(a.ravel(), b.ravel())[0, 1] > 0.99
    assert not np.allclose(a, b, rtol=1e-3)        # and it is a different function


def test_layer_norm_f32_is_layer_norm():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((16, 1280)) * 3 + 1
    g = syn.f32_to_bf16_bits((1 + 0.1 * rng.standard_normal(1280)).astype(np.float32))
    b = syn.f32_to_bf16_bits((0.02 * rng.standard_normal(1280)).astype(np.float32))
    np.testing.assert_allclose(fo.layer_norm_f32(x, g, b, 1e-6), vo.layer_norm(x, g, b, 1e-6), atol=2e-5)
