"""The activation's fast-path sin^2 constants, checked on the CPU.

The kernel evaluates sin(pi f), |f| <= 1/2, as f P(f^2) with the float
coefficients of sin2.cuh (`sin2p::coef`).  These tests read those constants
from the header and check them against the mathematics: the approximation
error in double precision, the error of the same Horner evaluation carried
out in float32, and the exact special values sin(0) = 0, sin(pi/2) = 1.
"""
import os
import re

import numpy as np

HEADER = os.path.join(os.path.dirname(__file__), "..", "bigvgan_waveform_decoder_alias_b200",
                      "csrc", "sin2.cuh")


def coefficients():
    src = open(HEADER).read()
    body = src[src.index("constexpr float coef(int j)"):]
    body = body[:body.index("}")]
    vals = [float(v) for v in re.findall(r"(-?\d+\.\d+(?:e-?\d+)?)f", body)]
    assert len(vals) == 5, vals
    return vals


def horner_f32(c, f):
    f = f.astype(np.float32)
    s = (f * f).astype(np.float32)
    p = np.full_like(s, np.float32(c[4]))
    for j in (3, 2, 1, 0):
        # fused multiply-add: one rounding of the exact product-sum
        p = (p.astype(np.float64) * s.astype(np.float64) + np.float64(np.float32(c[j]))).astype(np.float32)
    return (f * p).astype(np.float32)


def test_polynomial_approximation_error():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 200001)
    approx = f * sum(cj * (f * f) ** j for j, cj in enumerate(c))
    # the fit itself is within 3.4e-9; rounding the coefficients to float adds the rest
    assert np.abs(approx - np.sin(np.pi * f)).max() < 6e-8


def test_float32_evaluation_error():
    c = coefficients()
    f = np.linspace(-0.5, 0.5, 400001).astype(np.float32)
    got = horner_f32(c, f).astype(np.float64)
    exact = np.sin(np.pi * f.astype(np.float64))
    assert np.abs(got - exact).max() < 2.5e-7
    # sin^2 as the kernel forms it (g^2 with g = f P), relative to its size near the top
    assert np.abs(got ** 2 - exact ** 2).max() < 5e-7


def test_special_values():
    c = coefficients()
    g = horner_f32(c, np.array([0.0, 0.5, -0.5, 1e-30], np.float32)).astype(np.float64)
    assert g[0] == 0.0 and g[3] == np.float32(1e-30) * np.float32(c[0])
    assert abs(g[1] - 1.0) < 2.5e-7 and abs(g[2] + 1.0) < 2.5e-7
    # odd symmetry of f P(f^2)
    f = np.linspace(0, 0.5, 1001).astype(np.float32)
    np.testing.assert_array_equal(horner_f32(c, f), -horner_f32(c, -f))
