"""Kernel-level parity on a B200: every CUDA kernel of the path, called through the C ABI
(include/vit_ops.h), against the fp64 oracle on the same bf16 inputs (seeded, synthetic)."""
import numpy as np
import pytest
import torch

from oracle import mrope_oracle as mo
from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import (assert_attention_close, assert_bf16_close, assert_fp32_close, bf16_bits_to_torch,
                          to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bits(shape, seed, std=1.0, uniform=False):
    return syn.make_matrix(shape, seed, std, uniform)


def _status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# ------------------------------------------------------------------ GEMM
# Products with fewer 256 x 256 tiles than the device has SM pairs run on 256 x 128 tiles
# (gemm_use_narrow); the first seven cases take that path, the last two the wide one.
GEMM_CASES = [
    # (M, N, K): ragged M over several tiles, K tail (1176 = 18*64 + 24), N tails (N % 256 != 0)
    (300, 1280, 1176),
    (129, 1536, 1280),
    (64, 256, 64),
    (517, 5120, 1280),
    (385, 1280, 5120),
    (1, 3584, 5120),
    (200, 304, 72),
    (4800, 1280, 1280),      # enough 256 x 256 tiles to fill the SM pairs: the wide tiles
    (2100, 5120, 1280),
    (2100, 1328, 1280),      # wide tiles with an N tail: the two epilogue groups get unequal chunks
]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
@pytest.mark.parametrize("epi", [nv.EPI_STORE_F32, nv.EPI_ADD_F32, nv.EPI_STORE_BF16, nv.EPI_GELU_BF16])
def test_gemm_epilogues(M, N, K, epi):
    a, b = _bits((M, K), 1 + M, 1.0, uniform=True), _bits((N, K), 2 + N, 0.02)
    bias = _bits((N,), 3 + K, 0.5)
    A, B, Bi = bf16_bits_to_torch(a), bf16_bits_to_torch(b), bf16_bits_to_torch(bias)
    ref = vo.linear(a, b, bias)
    st = _status()
    if epi in (nv.EPI_STORE_F32, nv.EPI_ADD_F32):
        x0 = syn.make_f32((M, N), 4, 1.0)
        C = torch.from_numpy(x0.copy()).to(DEV) if epi == nv.EPI_ADD_F32 else torch.empty((M, N), device=DEV)
        nv.op_gemm(A, B, Bi, C, epi, status=st)
        if epi == nv.EPI_ADD_F32:
            ref = ref + x0
        assert_fp32_close(to_np(C), ref, 1e-4, f"gemm epi {epi}")
    else:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        nv.op_gemm(A, B, Bi, C, epi, status=st)
        if epi == nv.EPI_GELU_BF16:
            ref = vo.gelu_erf(ref)
        assert_bf16_close(to_np(C), ref, f"gemm epi {epi}")
    assert int(st.item()) == 0


def test_gemm_no_bias_and_large_k():
    M, N, K = 260, 512, 5120
    a, b = _bits((M, K), 11, 1.0), _bits((N, K), 12, 0.02)
    C = torch.empty((M, N), device=DEV)
    nv.op_gemm(bf16_bits_to_torch(a), bf16_bits_to_torch(b), None, C, nv.EPI_STORE_F32)
    assert_fp32_close(to_np(C), vo.linear(a, b), 1e-4, "gemm no bias")


@pytest.mark.parametrize("grids,order", [([(1, 8, 8)], 0), ([(1, 10, 14), (2, 4, 6), (1, 6, 2)], 0),
                                         ([(1, 10, 14), (1, 6, 8)], 1)])
def test_qkv_rope_epilogue(grids, order):
    P = syn.n_patches(grids)
    h_in, w = _bits((P, 1280), 21, 1.0), _bits((3840, 1280), 22, 0.02)
    b = _bits((3840,), 23, 0.1)
    pos, _ = nv.op_positions(grids, order)
    cs = nv.op_rope_table(max(max(g[1], g[2]) for g in grids) + 1)
    C = torch.empty((P, 3840), dtype=torch.bfloat16, device=DEV)
    nv.op_gemm(bf16_bits_to_torch(h_in), bf16_bits_to_torch(w), bf16_bits_to_torch(b), C, nv.EPI_QKV_ROPE,
               pos=pos, rope_cs=cs)
    hp, wp = vo.patch_positions(grids, order)
    q, k, v = vo.qkv_rope(h_in, {"qkv_w": w, "qkv_b": b}, hp, wp)
    ref = np.concatenate([q.reshape(P, -1), k.reshape(P, -1), v.reshape(P, -1)], 1)
    assert_bf16_close(to_np(C), ref, "qkv+rope")


# ------------------------------------------------------------------ positions / rope table
@pytest.mark.parametrize("order", [0, 1])
def test_positions_and_merge_rows(order):
    grids = [(1, 6, 10), (3, 4, 4), (1, 2, 2), (1, 12, 2)]
    pos, mr = nv.op_positions(grids, order)
    hp, wp = vo.patch_positions(grids, order)
    got = pos.cpu().numpy()
    np.testing.assert_array_equal(got >> 16, hp)
    np.testing.assert_array_equal(got & 0xFFFF, wp)
    # merge_row: the merger reads rows 4m..4m+3 of the scattered buffer for merged token m
    g = vo.merge_groups(grids, order)
    inv = np.empty(g.size, np.int64)
    inv[mr.cpu().numpy()] = np.arange(g.size)
    np.testing.assert_array_equal(inv.reshape(-1, 4), g)


def test_rope_table():
    cs = nv.op_rope_table(130).cpu().numpy().astype(np.float64)
    ang = np.outer(np.arange(130), vo.rope_inv_freq())
    np.testing.assert_allclose(cs[..., 0], np.cos(ang), atol=1e-7)
    np.testing.assert_allclose(cs[..., 1], np.sin(ang), atol=1e-7)


# ------------------------------------------------------------------ LayerNorm
@pytest.mark.parametrize("rows", [1, 7, 1000])
def test_layernorm(rows):
    x = syn.make_f32((rows, 1280), 31, 3.0) + 0.7
    g = _bits((1280,), 32, 1.0)
    b = _bits((1280,), 33, 0.5)
    Y = torch.empty((rows, 1280), dtype=torch.bfloat16, device=DEV)
    nv.op_layernorm(torch.from_numpy(x).to(DEV), bf16_bits_to_torch(g), bf16_bits_to_torch(b), Y, 1e-6)
    assert_bf16_close(to_np(Y), vo.layer_norm(x, g, b, 1e-6), "layernorm")


def test_layernorm_scatter_rows():
    grids = [(1, 4, 6)]
    _, mr = nv.op_positions(grids, 1)
    x = syn.make_f32((24, 1280), 34, 1.0)
    g = syn.f32_to_bf16_bits(np.ones(1280, np.float32))
    Y = torch.empty((24, 1280), dtype=torch.bfloat16, device=DEV)
    nv.op_layernorm(torch.from_numpy(x).to(DEV), bf16_bits_to_torch(g), None, Y, 1e-6, out_row=mr)
    ref = vo.layer_norm(x, g, None, 1e-6)
    assert_bf16_close(to_np(Y)[mr.cpu().numpy()], ref, "layernorm scatter")


# ------------------------------------------------------------------ attention
ATTN_CASES = [
    [64],                    # one tile, ragged
    [128],                   # exactly one tile
    [300, 64, 129],          # several tiles, ragged tails, varied lengths
    [576, 1024],             # 336^2 and 448^2 images
    [0, 40, 0, 257],         # empty segments
    [4, 4, 4],               # tiny segments
]


@pytest.mark.parametrize("lens", ATTN_CASES)
def test_attention_varlen(lens):
    P = sum(lens)
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    qkv = _bits((P, 3840), 41 + P, 1.0)
    out = torch.full((P, 1280), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = _status()
    nv.op_attention(bf16_bits_to_torch(qkv), cu, out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = vo._f64(qkv)
    q, k, v = (x[:, i * 1280:(i + 1) * 1280].reshape(P, 16, 80) for i in range(3))
    segs = [(int(cu[i]), int(lens[i]), 0, 0) for i in range(len(lens)) if lens[i] > 0]
    ref = vo.varlen_attention(q, k, v, segs)
    assert_attention_close(to_np(out), ref, np.abs(v).max(), f"attention {lens}")


def test_attention_more_segments_than_one_launch():
    # 700 segments: more than one launch's segment table holds, so the work is split across
    # launches; lengths 0..40 (empty, tiny and ragged segments)
    lens = np.random.Generator(np.random.PCG64(77)).integers(0, 41, size=700)
    P = int(lens.sum())
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    qkv = _bits((P, 3840), 78, 1.0)
    out = torch.full((P, 1280), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = _status()
    nv.op_attention(bf16_bits_to_torch(qkv), cu, out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    x = vo._f64(qkv)
    q, k, v = (x[:, i * 1280:(i + 1) * 1280].reshape(P, 16, 80) for i in range(3))
    segs = [(int(cu[i]), int(lens[i]), 0, 0) for i in range(len(lens)) if lens[i] > 0]
    ref = vo.varlen_attention(q, k, v, segs)
    assert_attention_close(to_np(out), ref, np.abs(v).max(), "attention, 700 segments")


@pytest.mark.slow
def test_attention_one_segment_across_launches():
    # one segment longer than a launch's work table (4096 pairs of 128-query tiles): its query
    # tiles continue in a second launch, which must still see every key of the segment. Inputs
    # are drawn on the device (seeded); the oracle takes sampled query rows one by one against
    # all keys, on four of the heads.
    P = 4096 * 256 + 3000
    qkv = syn.device_normal_bf16((P, 3840), 79, 1.0)
    out = torch.full((P, 1280), float("nan"), dtype=torch.bfloat16, device=DEV)
    st = _status()
    nv.op_attention(qkv, np.array([0, P], np.int32), out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    rows = np.array([0, 1, 123457, 1048575, 1048576, 1048577, 1050000, P - 1])
    for h in (0, 5, 10, 15):
        q = to_np(qkv[rows, h * 80:(h + 1) * 80])
        k = to_np(qkv[:, 1280 + h * 80:1280 + (h + 1) * 80])
        v = to_np(qkv[:, 2560 + h * 80:2560 + (h + 1) * 80])
        ref = vo.attention(q, k, v)
        assert_attention_close(to_np(out[rows, h * 80:(h + 1) * 80]), ref, np.abs(v).max(),
                               f"one {P}-row segment, head {h}")
    del qkv, out
    torch.cuda.empty_cache()


def test_exp2_fma_dense_sweep():
    # the FMA-pipe exponential of the softmax against the exact 2^x: relative error within the
    # minimax bound (7.5e-5) plus float32 rounding wherever 2^x is a normal number, exactly 0 at
    # and below -127.5 (masked scores are -inf), and nothing above 2^-126 in between
    xs = np.concatenate([np.linspace(-140.0, 20.0, 4_000_001), np.arange(-130, 21, dtype=np.float64),
                         np.arange(-130, 21) + 0.5, [-np.inf, -127.5, -126.0, 0.0, -0.0, 8.0]]).astype(np.float32)
    x = torch.from_numpy(xs).to(DEV)
    y = nv.op_exp2_fma(x).cpu().numpy().astype(np.float64)
    ref = np.exp2(xs.astype(np.float64))
    normal = xs >= -125.0            # results >= 2^-125: normal numbers whatever 2^f's exponent
    rel = np.abs(y[normal] / ref[normal] - 1.0)
    assert rel.max() <= 7.5e-5 + 4 * 2.0 ** -24, rel.max()
    assert (y[xs <= -127.5] == 0.0).all()
    mid = (xs > -127.5) & (xs < -125.0)
    assert ((y[mid] >= 0.0) & (y[mid] <= 2.0 ** -124)).all()
    assert np.isfinite(y).all() and (y >= 0).all()
    # a smooth sweep: the polynomial's error matters, not a single point
    assert rel.mean() < 5e-5


def test_attention_large_scores():
    # sharply peaked softmax: scores of order 100 exercise the running-max rescale
    lens = [384]
    P = 384
    qkv = _bits((P, 3840), 51, 6.0)
    cu = np.array([0, P], np.int32)
    out = torch.empty((P, 1280), dtype=torch.bfloat16, device=DEV)
    nv.op_attention(bf16_bits_to_torch(qkv), cu, out)
    x = vo._f64(qkv)
    q, k, v = (x[:, i * 1280:(i + 1) * 1280].reshape(P, 16, 80) for i in range(3))
    ref = vo.varlen_attention(q, k, v, [(0, P, 0, 0)])
    assert_attention_close(to_np(out), ref, np.abs(v).max(), "attention peaked")


# ------------------------------------------------------------------ M-RoPE
def _mrope_gpu(ids, grids):
    t = torch.from_numpy(np.ascontiguousarray(ids, np.int32)).to(DEV)
    st = _status()
    out = torch.full((3, len(ids)), -7, dtype=torch.int32, device=DEV)
    delta = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    nv.mrope_index(t, grids, out=out, delta=delta, status=st)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(delta.item()), int(st.item())


@pytest.mark.parametrize("which", ["tiny", "video", "text", "two_images"])
def test_mrope_bit_exact(which):
    if which == "tiny":
        ids, grids = syn.tiny_prompt(0)
    elif which == "video":
        ids, grids = syn.video_prompt(5)
    elif which == "text":
        ids, grids = syn.make_prompt([("text", 2500)], 3), np.zeros((0, 3), np.int32)
    else:
        ids = syn.make_prompt([("image", 12), ("image", 6), ("text", 5)], 4)
        grids = np.array([[1, 6, 8], [1, 2, 12]], np.int32)
    ref, rdelta = mo.mrope_index(ids, grids)
    got, delta, st = _mrope_gpu(ids, grids)
    assert st == 0
    np.testing.assert_array_equal(got, ref)
    assert delta == rdelta


@pytest.mark.parametrize("case", ["short", "long", "no_grid", "odd_grid", "zero_t", "huge_grid"])
def test_mrope_malformed_sets_status(case):
    if case == "short":
        ids, grids = syn.make_prompt([("image", 15)], 0), [[1, 8, 8]]
    elif case == "long":
        ids, grids = syn.make_prompt([("image", 17)], 0), [[1, 8, 8]]
    elif case == "no_grid":
        ids, grids = syn.make_prompt([("image", 16), ("image", 16)], 0), [[1, 8, 8]]
    elif case == "odd_grid":      # a consumed grid with an odd side
        ids, grids = syn.make_prompt([("image", 4)], 0), [[1, 3, 8]]
    elif case == "zero_t":
        ids, grids = syn.make_prompt([("image", 4)], 0), [[0, 4, 4]]
    else:                         # factors whose product would overflow
        ids, grids = syn.make_prompt([("image", 4)], 0), [[1 << 30, 1 << 30, 1 << 30]]
    if case in ("odd_grid", "zero_t", "huge_grid"):
        with pytest.raises(mo.MRopeError):
            mo.mrope_index(ids, grids)
    got, delta, st = _mrope_gpu(ids, grids)
    assert st == nv.VIT_ERR_TOKENS
    assert (got == -7).all() and delta == -7      # nothing written


def test_mrope_ignores_unused_trailing_grids():
    # the oracle checks a grid only when a vision run consumes it; malformed grids after the
    # last consumed one change nothing
    ids = syn.make_prompt([("text", 7), ("image", 16), ("text", 9), ("video", 12), ("text", 3)], 21)
    used = [[1, 8, 8], [3, 4, 4]]
    ref, rdelta = mo.mrope_index(ids, used)
    for tail in ([[1, 3, 8]], [[0, 4, 4], [1, 1 << 30, 1 << 30]], [[-5, 7, 9]]):
        grids = np.array(used + tail, np.int32)
        r2, d2 = mo.mrope_index(ids, grids)
        np.testing.assert_array_equal(r2, ref)
        got, delta, st = _mrope_gpu(ids, grids)
        assert st == 0, tail
        np.testing.assert_array_equal(got, ref)
        assert delta == rdelta == d2


def test_mrope_empty_prompt():
    t = torch.zeros(0, dtype=torch.int32, device=DEV)
    out, delta = nv.mrope_index(t, None)
    torch.cuda.synchronize()
    assert out.shape == (3, 0) and int(delta.item()) == 0


# ------------------------------------------------------------------ bounded waits
def test_bounded_wait_times_out_and_context_survives():
    # a wait that nothing satisfies must end with VIT_ERR_TIMEOUT, not hang; the GPU stays usable
    st = _status()
    nv.op_wait_selftest(st, 2_000_000)
    torch.cuda.synchronize()
    assert int(st.item()) == nv.VIT_ERR_TIMEOUT
    a, b = _bits((130, 64), 61, 1.0), _bits((256, 64), 62, 0.02)
    C = torch.empty((130, 256), device=DEV)
    nv.op_gemm(bf16_bits_to_torch(a), bf16_bits_to_torch(b), None, C, nv.EPI_STORE_F32)
    assert_fp32_close(to_np(C), vo.linear(a, b), 1e-4, "gemm after timeout test")
