"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances, derived from the arithmetic of the CUDA path. bf16 carries 8 significant bits, so
one rounding to bf16 has relative error at most u = 2^-8 (the unit roundoff).
* fp32 outputs of a bf16 x bf16 -> fp32 product: max|err| <= 1e-4 * max|ref| (fp32-accumulate path).
* bf16 outputs: the fp32 result is rounded once to bf16, so |err| <= u * |ref| + 1e-4 * max|ref|.
* attention: every weight of P is rounded to bf16 before P V (relative error <= u, weights sum to
  1 after normalisation) and O is rounded to bf16, so |err| <= u * (max|v| + |O|) <= 2u * max|v|
  (+ the fp32 slack 1e-4 * max|v|).
* whole encoder (bf16 output): max|err| <= 3e-2 * max|ref| and per-token cosine >= 0.999.
"""
import numpy as np
import torch

BF16_REL = 2.0 ** -8          # unit roundoff of bf16 (8 significant bits)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def bf16_bits_to_torch(bits: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16).to(device)


def assert_fp32_close(got, ref, rel=1e-4, what=""):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    scale = np.abs(ref).max()
    err = np.abs(got - ref).max()
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    assert err <= rel * scale, f"{what}: max|err| {err:.3e} > {rel:g} * max|ref| {scale:.3e}"


def assert_bf16_close(got, ref, what="", extra=1e-4):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    bound = BF16_REL * np.abs(ref) + extra * np.abs(ref).max()
    bad = np.abs(got - ref) > bound
    if bad.any():
        i = np.unravel_index(np.argmax(np.abs(got - ref) - bound), got.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {got.size} elements outside the bf16 bound; "
                             f"worst at {i}: got {got[i]:.6g} ref {ref[i]:.6g}")


def assert_attention_close(got, ref, vmax, what=""):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref).max()
    bound = (2 * BF16_REL + 1e-4) * vmax
    assert err <= bound, f"{what}: max|err| {err:.3e} > 2u max|v| = {bound:.3e}"


def assert_encoder_close(got, ref, what=""):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref).max()
    scale = np.abs(ref).max()
    cos = (got * ref).sum(1) / (np.linalg.norm(got, axis=1) * np.linalg.norm(ref, axis=1) + 1e-30)
    assert err <= 3e-2 * scale, f"{what}: max|err| {err:.3e} > 3e-2 * max|ref| {scale:.3e}"
    assert cos.min() >= 0.999, f"{what}: min per-token cosine {cos.min():.6f} < 0.999"
    return err / scale, cos.min()
