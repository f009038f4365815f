"""CPU oracle for the fp8 (E4M3) variant of the vision tower (fp64, numpy).

TEST INFRASTRUCTURE ONLY (see ``oracle/vit_oracle.py``): used by ``tests/`` and ``bench.py``'s CPU
leg, never by the product path; it shares no code with the CUDA kernels.

Passage: "Qwen2-VL-2B-Instruct -- LiteRT-LM" card, file table (Vision row: the vision tower ships
with int8 weights) and its correlation note (the static rewrite correlates 1.0 with the reference
in fp32, 0.90 with int8 weights). The pages name an 8-bit tower and its accuracy, not a
quantisation scheme. Readings taken here (the plainest scheme that an 8-bit tensor-core contraction
computes exactly):

* 8-bit format: FP8 E4M3 (1 sign, 4 exponent bits of bias 7, 3 mantissa bits; largest finite
  448, smallest normal 2^-6, subnormal step 2^-9; no infinities). A real number is coded by
  rounding to the nearest E4M3 value, ties to the even mantissa.
* Scales are powers of two, so dividing by them is exact and every code is decided by one
  rounding of an exact value. A vector v with max |v| = a gets the scale 2^e, e the smallest
  integer with a <= 448 * 2^e, but at least -126 (so that the scale and its inverse are normal
  float32 numbers; an all-zero vector gets 2^-126 too).
* Weights: every output channel (row of an nn.Linear weight [out, in]) has its own scale;
  codes q = RNE(w / s). The dequantised weight is s * q.
* Activations: every row of the product's input (one token) has its own scale, taken at run time
  from that row; dequantised likewise.
* Which products: the four linears of every ViT block (QKV, out-proj, fc1, fc2), 98% of the
  tower's linear work. The patch embed (raw pixels in) and the merger stay as in the bf16 tower.
* y = (s_row * q_row) . (s_out * q_out) + bias: the product of dequantised operands, i.e.
  s_row * s_out * sum(q_row * q_out), which an E4M3 tensor-core product with fp32 accumulation
  computes exactly up to the order of the sum.

Everything else (LayerNorm, rope, attention, GELU, the residual stream) is the bf16 tower's
definition (``vit_oracle``), in fp64.
"""
from __future__ import annotations

from typing import Dict

import numpy as np

from oracle import vit_oracle as vo

E4M3_MAX = 448.0
E4M3_MIN_NORMAL_EXP = -6          # smallest normal 2^-6
E4M3_MANT_BITS = 3
FP8_LINEARS = ("qkv_w", "proj_w", "fc1_w", "fc2_w")


def round_e4m3(x) -> np.ndarray:
    """Nearest E4M3 value (ties to even mantissa), as float64. |x| <= 448 is assumed (the scales
    guarantee it); larger magnitudes are clipped to 448."""
    x = np.asarray(x, np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))          # a = m 2^ex, m in [1/2, 1)
    e = np.maximum(ex - 1, E4M3_MIN_NORMAL_EXP)         # binade of a (subnormals share 2^-6's)
    step = np.ldexp(1.0, e - E4M3_MANT_BITS)            # spacing of E4M3 values in that binade
    return np.clip(np.round(x / step) * step, -E4M3_MAX, E4M3_MAX)   # np.round: half to even


def pow2_scale(amax) -> np.ndarray:
    """2^e with e the smallest integer such that amax <= 448 * 2^e, and e >= -126.

    Exactly, without dividing: amax = M 2^E with M in [1, 2) and 448 = 1.75 * 2^8, so
    amax <= 448 * 2^e  <=>  e >= E - 8 + log2(M / 1.75), whose smallest integer solution is
    E - 8, plus one when M > 1.75."""
    amax = np.asarray(amax, np.float64)
    m, ex = np.frexp(np.where(amax > 0, amax, 0.0))    # amax = m 2^ex, m in [1/2, 1)
    M, E = 2.0 * m, ex - 1
    e = np.where(amax > 0, E - 8 + (M > 1.75), -126)
    return np.ldexp(1.0, np.maximum(e, -126).astype(np.int64))


def quantize_rows(x) -> tuple:
    """(codes, scales): per-row power-of-two scales and E4M3 codes of x [rows, cols] (codes as the
    float64 values of the E4M3 numbers)."""
    x = vo._f64(x)
    s = pow2_scale(np.abs(x).max(axis=1))
    return round_e4m3(x / s[:, None]), s


def dequantize_rows(codes, scales) -> np.ndarray:
    return np.asarray(codes, np.float64) * np.asarray(scales, np.float64)[:, None]


def quant_dequant_rows(x) -> np.ndarray:
    q, s = quantize_rows(x)
    return dequantize_rows(q, s)


def quantize_weights(weights: Dict) -> Dict:
    """The tower's weights with the four block linears replaced by their dequantised E4M3 values
    (per output channel), everything else unchanged."""
    out = dict(weights)
    out["layers"] = [{k: (quant_dequant_rows(v) if k in FP8_LINEARS else v) for k, v in L.items()}
                     for L in weights["layers"]]
    return out


def layer_norm_f32(x, gamma, beta, eps: float) -> np.ndarray:
    """The same LayerNorm evaluated in float32 throughout (numpy's float32 arithmetic), returned
    as float64: a second exact implementation of the definition that differs only in rounding."""
    x = np.asarray(x, np.float32)
    mu = x.mean(axis=-1, keepdims=True, dtype=np.float32)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True, dtype=np.float32)
    y = (x - mu) / np.sqrt(var + np.float32(eps))
    y = y * vo._f64(gamma).astype(np.float32) + (vo._f64(beta).astype(np.float32) if beta is not None else 0)
    return y.astype(np.float64)


def round_bf16(x) -> np.ndarray:
    """Nearest bfloat16 value (ties to even), as float64."""
    x = np.asarray(x, np.float64)
    _, ex = np.frexp(np.where(x != 0, np.abs(x), 1.0))
    step = np.ldexp(1.0, np.maximum(ex - 1, -126) - 7)   # 8 significant bits
    return np.round(x / step) * step


def vit_block_fp8(x, L, segs, hpos, wpos, eps, ln=vo.layer_norm, store=lambda t: t):
    """The pre-norm block with E4M3 inputs to its four linears (weights L already dequantised).
    ``store`` is applied to the tensors a GPU keeps in memory between kernels (q, k, v, the
    attention output, the MLP hidden layer): the identity for the definition itself."""
    h = quant_dequant_rows(ln(x, L["ln1_w"], L["ln1_b"], eps))
    q, k, v = (store(t) for t in vo.qkv_rope(h, L, hpos, wpos))
    a = store(vo.varlen_attention(q, k, v, segs))
    x = x + vo.linear(quant_dequant_rows(a), L["proj_w"], L["proj_b"])
    h = quant_dequant_rows(ln(x, L["ln2_w"], L["ln2_b"], eps))
    f = store(vo.gelu_erf(vo.linear(h, L["fc1_w"], L["fc1_b"])))
    return x + vo.linear(quant_dequant_rows(f), L["fc2_w"], L["fc2_b"])


def vit_encode_fp8(patches, grids, weights: Dict, depth: int = None, eps: float = 1e-6,
                   patch_order: int = 0, ln_float32: bool = False, bf16_storage: bool = False):
    """The fp8 tower: patches [P, 1176] + grid_thw -> merged tokens [P/4, out_dim] (float64).
    ``weights`` are the bf16 tower's weights; the block linears are quantised here.

    Two switches give further exact implementations of the same definition that differ only in
    rounding, to measure how far such implementations drift apart through the activation
    roundings (each rounding to E4M3 is a step function of its input): ln_float32 evaluates every
    LayerNorm in float32; bf16_storage rounds q, k, v, the attention output and the MLP hidden
    layer to bfloat16, the precision a GPU keeps them in between kernels."""
    g = vo.check_grid(grids)
    segs = vo.segments(g)
    hpos, wpos = vo.patch_positions(g, patch_order)
    wq = quantize_weights(weights)
    depth = len(wq["layers"]) if depth is None else depth
    ln = layer_norm_f32 if ln_float32 else vo.layer_norm
    store = round_bf16 if bf16_storage else (lambda t: t)
    x = vo.patch_embed(patches, wq["pe_w"], wq.get("pe_b"))
    for l in range(depth):
        x = vit_block_fp8(x, wq["layers"][l], segs, hpos, wpos, eps, ln, store)
    return vo.merger(x, g, wq, eps, patch_order)
