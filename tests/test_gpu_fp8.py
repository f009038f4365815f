"""The fp8 (E4M3) tower on a B200 against the fp8 oracle (``oracle/fp8_oracle.py``).

* Quantisation of bf16 rows (vit_quantize_fp8): bit-exact -- the input is exact, the scale is a
  power of two decided from the exact row maximum, and the code is one rounding of an exact value.
* LayerNorm + quantisation: the normalised value is computed in fp32 on the GPU and in fp64 in
  the oracle, so codes may differ where the oracle's value lies within fp32 rounding of a step
  between two codes (or a row's maximum within rounding of a scale boundary); every other code
  must be equal, and each differing one must be such a case.
* The E4M3 product (vit_op_gemm_fp8) given the same codes and scales: the products of codes are
  exact in fp32, so the fp32-accumulate bar (1e-4 max|ref|) holds, and one bf16 rounding on the
  bf16 epilogues.
* The whole fp8 tower, at depth 2 and 32: within twice the drift between two exact
  implementations of the fp8 definition that differ only in the roundings the GPU makes (bf16
  storage of q, k, v, the attention output and the MLP hidden layer; fp32 LayerNorms), measured
  by the oracle alone (``tests/golden/fp8_drift.json``); every rounding to E4M3 is a step
  function of its input, so no bound follows from the arithmetic alone. And the closeness to the
  unquantised tower that the pages' 8-bit tower reaches (correlation 0.90, "Qwen2-VL-2B-Instruct
  -- LiteRT-LM").
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import fp8_oracle as fo
from oracle import vit_oracle as vo
from resolution_vit_vision_b200 import native as nv
from resolution_vit_vision_b200 import synthetic as syn
from tests.parity import assert_bf16_close, assert_fp32_close, bf16_bits_to_torch, to_np

pytestmark = pytest.mark.gpu
DEV = "cuda"
HERE = os.path.dirname(os.path.abspath(__file__))


def _e4m3_values(codes: torch.Tensor) -> np.ndarray:
    return codes.cpu().view(torch.float8_e4m3fn).double().numpy()


def _codes_from_values(q: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(q)).to(torch.float8_e4m3fn).view(torch.uint8).to(DEV)


@pytest.mark.parametrize("rows,cols", [(37, 1280), (5, 5120), (130, 8), (3, 3840)])
def test_quantize_bit_exact(rows, cols):
    rng = np.random.default_rng(rows + cols)
    x = (rng.standard_normal((rows, cols)) * np.exp(rng.uniform(-20, 20, (rows, 1)))).astype(np.float32)
    x[0] = 0.0                                      # an all-zero row
    if rows > 2:
        x[1, :] = 448.0 * 2.0 ** rng.integers(-10, 10)   # a row whose max is a scale boundary
        x[2, :4] = [1.0625, 1.1875, -3.0 * 2 ** -10, 2.0 ** -11]   # rounding ties and tiny values
    bits = syn.f32_to_bf16_bits(x)
    codes, scales = nv.quantize_fp8(bf16_bits_to_torch(bits))
    q, s = fo.quantize_rows(bits)
    np.testing.assert_array_equal(scales.cpu().numpy().astype(np.float64), s)
    np.testing.assert_array_equal(_e4m3_values(codes), q)


def test_layernorm_fp8_codes():
    rows = 300
    x = syn.make_f32((rows, 1280), 31, 2.0) + 0.5
    wts = syn.make_weights(1, 1536, 32, affine=True)["layers"][0]
    g, b = wts["ln1_w"], wts["ln1_b"]
    codes, scales = nv.op_layernorm_fp8(torch.from_numpy(x).to(DEV), bf16_bits_to_torch(g), bf16_bits_to_torch(b))
    y = vo.layer_norm(x, g, b, 1e-6)
    q, s = fo.quantize_rows(y)
    gq, gs = _e4m3_values(codes), scales.cpu().numpy().astype(np.float64)
    same = gs == s
    # a scale may differ only where the row's maximum lies within fp32 rounding of a boundary
    amax = np.abs(y).max(axis=1)
    for r in np.nonzero(~same)[0]:
        assert abs(amax[r] / (448.0 * s[r] / 2) - 1) < 1e-5 or abs(amax[r] / (448.0 * s[r]) - 1) < 1e-5
    assert same.mean() > 0.99
    diff = (gq != q) & same[:, None]
    # a code may differ only where y / s lies within fp32 rounding of the midpoint of two codes
    t = y / s[:, None]
    lo, hi = np.minimum(gq, q), np.maximum(gq, q)
    mid = (lo + hi) / 2
    assert np.all(np.abs(t[diff] - mid[diff]) <= 1e-5 * np.abs(t[diff]) + 1e-9)
    assert np.all(np.abs(hi[diff] - lo[diff]) <= np.maximum(np.abs(lo[diff]), np.abs(hi[diff])) / 4 + 2.0 ** -9)
    assert diff.sum() <= 1e-3 * diff.size


# the first, third, fourth and fifth case run on 256 x 128 tiles (few tiles), the others on the
# wide 256 x 256 tiles
GEMM_CASES = [(300, 1280, 1280), (129, 3840, 1280), (517, 5120, 1280), (385, 1280, 5120), (70, 256, 1328),
              (4800, 1280, 1280), (2100, 5120, 1280)]


@pytest.mark.parametrize("M,N,K", GEMM_CASES)
@pytest.mark.parametrize("epi", [nv.EPI_ADD_F32, nv.EPI_GELU_BF16, nv.EPI_STORE_BF16, nv.EPI_QKV_ROPE])
def test_gemm_fp8_epilogues(M, N, K, epi):
    if epi == nv.EPI_QKV_ROPE and N != 3840:
        pytest.skip("the rope epilogue is the QKV product's")
    rng = np.random.default_rng(M + N + K)
    a = syn.f32_to_bf16_bits(rng.uniform(-1, 1, (M, K)).astype(np.float32) * np.exp(rng.uniform(-3, 3, (M, 1))).astype(np.float32))
    bw = syn.make_matrix((N, K), 2 + N, 0.02)
    qa, sa = fo.quantize_rows(a)
    qb, sb = fo.quantize_rows(bw)
    bias = syn.make_matrix((N,), 3 + K, 0.5)
    A, B = _codes_from_values(qa), _codes_from_values(qb)
    SA, SB = (torch.from_numpy(v.astype(np.float32)).to(DEV) for v in (sa, sb))
    ref = vo.linear(fo.dequantize_rows(qa, sa), fo.dequantize_rows(qb, sb), bias)
    st = torch.zeros(1, dtype=torch.int32, device=DEV)
    Bi = bf16_bits_to_torch(bias)
    if epi == nv.EPI_ADD_F32:
        x0 = syn.make_f32((M, N), 4, 1.0)
        C = torch.from_numpy(x0.copy()).to(DEV)
        nv.op_gemm_fp8(A, SA, B, SB, Bi, C, epi, status=st)
        assert_fp32_close(to_np(C), ref + x0, 1e-4, "gemm fp8 add")
    elif epi == nv.EPI_QKV_ROPE:
        hp = np.arange(M) % 37             # a position per row, (h, w) inside a 37 x 41 frame
        wp = (np.arange(M) * 7) % 41
        pos = torch.from_numpy(((hp << 16) | wp).astype(np.int32)).to(DEV)
        cs = nv.op_rope_table(64)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        nv.op_gemm_fp8(A, SA, B, SB, Bi, C, epi, pos=pos, rope_cs=cs, status=st)
        r = ref.copy()
        for part in (0, 1):      # rope on the q and k heads
            for h in range(16):
                c0 = part * 1280 + h * 80
                r[:, c0:c0 + 80] = vo.apply_rope_2d(ref[:, c0:c0 + 80], hp, wp)
        assert_bf16_close(to_np(C), r, "gemm fp8 qkv rope")
    else:
        C = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        nv.op_gemm_fp8(A, SA, B, SB, Bi, C, epi, status=st)
        assert_bf16_close(to_np(C), vo.gelu_erf(ref) if epi == nv.EPI_GELU_BF16 else ref, f"gemm fp8 epi {epi}")
    torch.cuda.synchronize()
    assert int(st.item()) == 0


def _encode_fp8(grids, depth, out_dim, seed, wts=None, patches=None):
    wts = wts if wts is not None else syn.make_weights(depth, out_dim, seed)
    patches = patches if patches is not None else syn.make_patches(grids, seed)
    wd = nv.weights_to_device(wts)
    enc = nv.VisionEncoder(wd, out_dim, fp8=nv.fp8_layers_device(wd))
    out = to_np(enc.encode(bf16_bits_to_torch(patches), grids))
    assert enc.device_status() == 0
    return out, wts, patches


def test_fp8_weights_quantised_on_device_match_the_oracle():
    wts = syn.make_weights(1, 1536, 33)
    wd = nv.weights_to_device(wts)
    q8 = nv.fp8_layers_device(wd)[0]
    for k in nv.FP8_LINEARS:
        q, s = fo.quantize_rows(wts["layers"][0][f"{k}_w"])
        np.testing.assert_array_equal(_e4m3_values(q8[k][0]), q)
        np.testing.assert_array_equal(q8[k][1].cpu().numpy().astype(np.float64), s)


def _drift_bar(which):
    return json.load(open(os.path.join(HERE, "golden", "fp8_drift.json")))[which]["bar"]


def _assert_within(got, ref, bar, what):
    assert np.isfinite(got).all(), what
    err = np.abs(got - ref).max() / np.abs(ref).max()
    cos = (got * ref).sum(1) / (np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1))
    assert err <= bar["max_err_rel"], f"{what}: max|err| {err:.4f} of max|ref| > {bar['max_err_rel']:.4f}"
    assert cos.min() >= bar["min_cos"], f"{what}: min cosine {cos.min():.5f} < {bar['min_cos']:.5f}"


@pytest.mark.parametrize("grids", [[(1, 8, 8)], [(1, 10, 14), (2, 4, 6), (1, 16, 12)]])
def test_fp8_tower_depth2(grids):
    got, wts, patches = _encode_fp8(grids, 2, 1536, 34)
    ref = fo.vit_encode_fp8(patches, grids, wts)
    _assert_within(got, ref, _drift_bar("depth2"), f"fp8 tower depth 2 {grids}")


def test_fp8_handle_rejected_by_noalloc_entry_point():
    wts = syn.make_weights(1, 1536, 35)
    wd = nv.weights_to_device(wts)
    enc = nv.VisionEncoder(wd, 1536, fp8=nv.fp8_layers_device(wd))
    p = torch.zeros((64, 1176), dtype=torch.bfloat16, device=DEV)
    out = torch.zeros((16, 1536), dtype=torch.bfloat16, device=DEV)
    g = np.array([[1, 8, 8]], np.int32)
    assert nv.lib().vit_encode_noalloc(p.data_ptr(), nv._gp(g), 1, enc.handle, out.data_ptr(), None,
                                       torch.cuda.current_stream().cuda_stream) == nv.VIT_ERR_ARG


@pytest.mark.slow
def test_fp8_tower_2b_full_depth():
    wl = syn.WORKLOADS["2b_448"]
    got, wts, patches = _encode_fp8(wl.grids, wl.depth, wl.out_dim, wl.seed)
    ref = fo.vit_encode_fp8(patches, wl.grids, wts)
    _assert_within(got, ref, _drift_bar("depth32"), "fp8 tower, 2B 448x448, depth 32")
    # and the 8-bit tower stays close to the unquantised one (the pages' int8 tower: 0.90)
    full = vo.vit_encode(patches, wl.grids, wts)
    assert np.corrcoef(got.ravel(), full.ravel())[0, 1] > 0.99
