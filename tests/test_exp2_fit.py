"""Provenance of the FMA-pipe exponential's polynomial (no GPU needed).

The coefficients in ``csrc/ptx.cuh`` (``exp2_fma2``) must be the float32 rounding of the minimax
fit that ``csrc/fit_exp2_poly.py`` computes (Remez exchange on the relative error of 2^f over
[-1/2, 1/2], degree 3), and that fit must meet the error bound the kernel's documentation states.
The fit itself is checked against properties of the best approximation: its error equioscillates
on degree + 2 points, and the polynomial is close to the Taylor coefficients (ln 2)^k / k!.
"""
import math
import os
import re
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "resolution_vit_vision_b200", "csrc")
sys.path.insert(0, CSRC)
import fit_exp2_poly as fit  # noqa: E402


def _kernel_coefficients():
    src = open(os.path.join(CSRC, "ptx.cuh")).read()
    body = src[src.index("void exp2_fma2"):]
    return [float(re.search(rf"c{i} = ([0-9.eE+-]+)f", body).group(1)) for i in range(4)]


def test_kernel_coefficients_are_the_fit():
    c, E = fit.remez(3)
    np.testing.assert_array_equal(np.float32(_kernel_coefficients()), c.astype(np.float32))
    assert E < 7.5e-5


def test_fit_error_bound_and_equioscillation():
    c, E = fit.remez(3)
    f = np.linspace(-0.5, 0.5, 400001)
    err = np.polyval(c[::-1], f) / 2.0 ** f - 1.0
    assert abs(np.abs(err).max() - E) < 1e-3 * E          # the levelled error is the max error
    # 5 alternating extrema of magnitude E (the Chebyshev alternation of a best approximation)
    s = np.sign(err)
    parts = np.split(np.arange(f.size), np.nonzero(np.diff(s))[0] + 1)
    peaks = [np.abs(err[p]).max() for p in parts]
    assert len(peaks) == 5 and min(peaks) > 0.99 * E
    assert fit.f32_horner_error(c.astype(np.float32)) < 7.5e-5


def test_fit_close_to_taylor_series():
    c, _ = fit.remez(3)
    taylor = [math.log(2) ** k / math.factorial(k) for k in range(4)]
    np.testing.assert_allclose(c, taylor, rtol=0.05, atol=2e-3)
