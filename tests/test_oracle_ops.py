"""Pins for the oracle's elementary steps (CPU only).

Each check ties the oracle to something other than itself: a library routine computing the
same textbook operation (torch.nn.functional in float64), a closed form, or an invariant.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import vit_oracle as vo

pytestmark = pytest.mark.filterwarnings("ignore")


def _rng(seed):
    return np.random.Generator(np.random.PCG64(seed))


# ------------------------------------------------------------------ LayerNorm
def test_layer_norm_matches_torch():
    r = _rng(1)
    x = r.standard_normal((37, 1280)) * 3 + 0.5
    g = 1 + 0.1 * r.standard_normal(1280)
    b = 0.02 * r.standard_normal(1280)
    ref = F.layer_norm(torch.from_numpy(x), (1280,), torch.from_numpy(g), torch.from_numpy(b), eps=1e-6)
    np.testing.assert_allclose(vo.layer_norm(x, g, b, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_layer_norm_closed_form_two_values():
    # LN([a, b]) with gamma 1, beta 0 and eps 0 is (-1, +1) for a < b
    y = vo.layer_norm(np.array([[2.0, 5.0]]), np.ones(2), np.zeros(2), 0.0)
    np.testing.assert_allclose(y, [[-1.0, 1.0]], atol=1e-15)


def test_layer_norm_moments():
    x = _rng(2).standard_normal((5, 1280)) * 7
    y = vo.layer_norm(x, np.ones(1280), np.zeros(1280), 1e-6)
    np.testing.assert_allclose(y.mean(-1), 0, atol=1e-12)
    var = x.var(-1)
    np.testing.assert_allclose(y.var(-1), var / (var + 1e-6), rtol=1e-12)


# ------------------------------------------------------------------ GELU
def test_gelu_matches_torch_exact():
    x = np.linspace(-8, 8, 2001)
    ref = F.gelu(torch.from_numpy(x), approximate="none").numpy()
    np.testing.assert_allclose(vo.gelu_erf(x), ref, rtol=1e-13, atol=1e-15)


def test_gelu_identities():
    x = np.linspace(-5, 5, 101)
    assert vo.gelu_erf(np.array([0.0]))[0] == 0.0
    # x*Phi(x) - (-x)*Phi(-x) = x
    np.testing.assert_allclose(vo.gelu_erf(x) - vo.gelu_erf(-x), x, atol=1e-14)
    # Phi(1) = 0.841344746068543 (standard normal table)
    np.testing.assert_allclose(vo.gelu_erf(np.array([1.0]))[0], 0.841344746068543, rtol=1e-14)


# ------------------------------------------------------------------ Linear
def test_linear_matches_torch():
    r = _rng(3)
    x, w, b = r.standard_normal((9, 33)), r.standard_normal((17, 33)), r.standard_normal(17)
    ref = F.linear(torch.from_numpy(x), torch.from_numpy(w), torch.from_numpy(b)).numpy()
    np.testing.assert_allclose(vo.linear(x, w, b), ref, rtol=1e-13, atol=1e-13)


def test_linear_reads_bf16_bits():
    # bit pattern 0x3F80 is 1.0, 0xC000 is -2.0 in bf16
    x = np.array([[0x3F80, 0xC000]], np.uint16)
    w = np.array([[0x3F80, 0x3F80]], np.uint16)
    assert vo.linear(x, w)[0, 0] == -1.0


# ------------------------------------------------------------------ attention
def test_attention_matches_torch_sdpa():
    r = _rng(4)
    S, d = 57, 80
    q, k, v = (r.standard_normal((S, d)) for _ in range(3))
    ref = F.scaled_dot_product_attention(torch.from_numpy(q)[None], torch.from_numpy(k)[None],
                                         torch.from_numpy(v)[None]).numpy()[0]
    np.testing.assert_allclose(vo.attention(q, k, v), ref, rtol=1e-12, atol=1e-12)


def test_attention_single_key_returns_its_value():
    r = _rng(5)
    q, k, v = r.standard_normal((4, 80)), r.standard_normal((1, 80)), r.standard_normal((1, 80))
    np.testing.assert_allclose(vo.attention(q, k, v), np.repeat(v, 4, 0), atol=1e-15)


def test_attention_equal_keys_average_values():
    r = _rng(6)
    q = r.standard_normal((3, 80))
    k = np.repeat(r.standard_normal((1, 80)), 9, 0)
    v = r.standard_normal((9, 80))
    np.testing.assert_allclose(vo.attention(q, k, v), np.repeat(v.mean(0, keepdims=True), 3, 0), atol=1e-14)


def test_attention_chunking_does_not_change_result():
    r = _rng(7)
    q, k, v = r.standard_normal((300, 80)), r.standard_normal((300, 80)), r.standard_normal((300, 80))
    np.testing.assert_allclose(vo.attention(q, k, v, chunk=7), vo.attention(q, k, v), rtol=1e-13, atol=1e-14)


def test_varlen_attention_is_block_diagonal():
    r = _rng(8)
    grids = [(1, 4, 6), (2, 2, 4), (1, 6, 2)]
    segs = vo.segments(grids)
    P = sum(n for _, n, _, _ in segs)
    q, k, v = (r.standard_normal((P, 16, 80)) for _ in range(3))
    packed = vo.varlen_attention(q, k, v, segs)
    # dense torch SDPA with a block-diagonal boolean mask
    mask = torch.zeros(P, P, dtype=torch.bool)
    for s, n, _, _ in segs:
        mask[s:s + n, s:s + n] = True
    tq, tk, tv = (torch.from_numpy(a).permute(1, 0, 2) for a in (q, k, v))
    ref = F.scaled_dot_product_attention(tq, tk, tv, attn_mask=mask).permute(1, 0, 2).reshape(P, 1280)
    np.testing.assert_allclose(packed, ref.numpy(), rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ 2-D rope
def test_rope_frequencies():
    f = vo.rope_inv_freq()
    assert f.shape == (20,)
    assert f[0] == 1.0
    np.testing.assert_allclose(f[1], 10000 ** (-1 / 20), rtol=1e-15)
    np.testing.assert_allclose(f[19], 10000 ** (-38 / 40), rtol=1e-15)


def test_rope_unit_vectors_closed_form():
    # e_0 at row 1 turns by angle 1 rad into dim 40; e_20 at column 1 turns into dim 60
    e0 = np.zeros((1, 80)); e0[0, 0] = 1
    y = vo.apply_rope_2d(e0, np.array([1]), np.array([0]))
    exp = np.zeros(80); exp[0] = math.cos(1.0); exp[40] = math.sin(1.0)
    np.testing.assert_allclose(y[0], exp, atol=1e-15)
    e20 = np.zeros((1, 80)); e20[0, 20] = 1
    y = vo.apply_rope_2d(e20, np.array([5]), np.array([1]))
    exp = np.zeros(80); exp[20] = math.cos(1.0); exp[60] = math.sin(1.0)
    np.testing.assert_allclose(y[0], exp, atol=1e-15)
    # the second row frequency: e_1 at row 3 turns by 3 * 10000^(-1/20)
    e1 = np.zeros((1, 80)); e1[0, 41] = 1
    a = 3 * 10000 ** (-1 / 20)
    y = vo.apply_rope_2d(e1, np.array([3]), np.array([0]))
    exp = np.zeros(80); exp[41] = math.cos(a); exp[1] = -math.sin(a)
    np.testing.assert_allclose(y[0], exp, atol=1e-15)


def test_rope_identity_at_origin_and_norm():
    r = _rng(9)
    x = r.standard_normal((20, 80))
    np.testing.assert_allclose(vo.apply_rope_2d(x, np.zeros(20, int), np.zeros(20, int)), x, atol=0)
    hp, wp = r.integers(0, 128, 20), r.integers(0, 128, 20)
    y = vo.apply_rope_2d(x, hp, wp)
    pair = lambda z: z[:, :40] ** 2 + z[:, 40:] ** 2
    np.testing.assert_allclose(pair(y), pair(x), rtol=1e-12)


def test_rope_scores_depend_on_relative_position_only():
    r = _rng(10)
    q, k = r.standard_normal((1, 80)), r.standard_normal((1, 80))
    def score(hq, wq, hk, wk):
        return (vo.apply_rope_2d(q, np.array([hq]), np.array([wq]))
                @ vo.apply_rope_2d(k, np.array([hk]), np.array([wk])).T)[0, 0]
    base = score(3, 7, 1, 2)
    np.testing.assert_allclose(score(3 + 11, 7 + 5, 1 + 11, 2 + 5), base, rtol=1e-11)
    assert abs(score(3, 8, 1, 2) - base) > 1e-6


def test_rope_matches_complex_rotation():
    # (x_d + i x_{d+40}) * exp(i a_d), the same rotation written with complex numbers (torch)
    r = _rng(11)
    x = r.standard_normal((13, 80))
    hp, wp = r.integers(0, 100, 13), r.integers(0, 100, 13)
    f = torch.tensor(10000.0, dtype=torch.float64) ** (-torch.arange(0, 40, 2, dtype=torch.float64) / 40)
    ang = torch.cat([torch.outer(torch.from_numpy(hp).double(), f), torch.outer(torch.from_numpy(wp).double(), f)], 1)
    z = torch.complex(torch.from_numpy(x[:, :40]), torch.from_numpy(x[:, 40:])) * torch.polar(torch.ones_like(ang), ang)
    ref = torch.cat([z.real, z.imag], 1).numpy()
    np.testing.assert_allclose(vo.apply_rope_2d(x, hp, wp), ref, rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ positions / packing
def test_block_order_positions_small():
    h, w = vo.frame_positions(4, 4, 0)
    # first merge group is the top-left 2x2, dw fastest
    assert list(zip(h[:8], w[:8])) == [(0, 0), (0, 1), (1, 0), (1, 1), (0, 2), (0, 3), (1, 2), (1, 3)]
    hr, wr = vo.frame_positions(2, 4, 1)
    assert list(zip(hr, wr)) == [(0, 0), (0, 1), (0, 2), (0, 3), (1, 0), (1, 1), (1, 2), (1, 3)]


def test_segments_per_frame():
    segs = vo.segments([(2, 4, 6), (1, 2, 2)])
    assert segs == [(0, 24, 4, 6), (24, 24, 4, 6), (48, 4, 2, 2)]


def test_bad_grids_rejected():
    for g in [(0, 4, 4), (1, 3, 4), (1, 4, 5), (1, 0, 4)]:
        with pytest.raises(ValueError):
            vo.check_grid([g])
