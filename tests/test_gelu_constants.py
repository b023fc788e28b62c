"""The BF16 GEGLU epilogue evaluates GELU with the rational erf approximation of
Abramowitz and Stegun, Handbook of Mathematical Functions, eq. 7.1.26 (constants
folded with 1/sqrt(2) and 1/2).  This test reads the constants out of the CUDA
source, evaluates the same sequence of float32 operations with numpy (reciprocal
and exp2 exact here, so only the formula and its constants are under test) and
holds it to the bound the source states against the exact erf form from scipy.
"""
import os
import re

import numpy as np
from scipy.special import erf

SRC = os.path.join(os.path.dirname(__file__), "..", "encoder_decision_model_b200", "csrc", "common.cuh")


def _gelu_as_constants():
    src = open(SRC).read()
    body = src[src.index("float gelu_as(float x)"):]
    body = body[:body.index("\n}\n")]
    # float literals in source order: p/sqrt2, 1.0, a5/2, a4/2, a3/2, a2/2, a1/2, -log2(e)/2
    return [float(v[:-1]) for v in re.findall(r"-?\d+\.\d+(?:e-?\d+)?f", body)]


def test_gelu_as_constants_match_the_published_formula():
    c = _gelu_as_constants()
    p, a5, a4, a3, a2, a1, k = c[0], c[2], c[3], c[4], c[5], c[6], c[7]
    # the folded constants are the handbook's times exact scalars
    np.testing.assert_allclose(p, 0.3275911 / np.sqrt(2), rtol=1e-7)
    np.testing.assert_allclose([a1, a2, a3, a4, a5],
                               0.5 * np.array([0.254829592, -0.284496736, 1.421413741, -1.453152027, 1.061405429]),
                               rtol=1e-7)
    np.testing.assert_allclose(k, -0.5 / np.log(2), rtol=1e-7)


def test_gelu_as_error_bound():
    c = _gelu_as_constants()
    f = np.float32
    p, a5, a4, a3, a2, a1, k = (f(v) for v in (c[0], c[2], c[3], c[4], c[5], c[6], c[7]))
    x = np.linspace(-12, 12, 400_001).astype(f)
    t = (f(1) / (p * np.abs(x) + f(1))).astype(f)
    q = (a5 * t + a4).astype(f)
    q = (q * t + a3).astype(f)
    q = (q * t + a2).astype(f)
    q = (q * t + a1).astype(f)
    e = np.exp2((x * (x * k)).astype(f)).astype(f)
    xh = (x * ((q * t).astype(f) * e).astype(f)).astype(f)
    g = np.where(x >= 0, x - xh, xh).astype(np.float64)
    xd = x.astype(np.float64)
    ref = 0.5 * xd * (1.0 + erf(xd / np.sqrt(2.0)))
    assert np.abs(g - ref).max() <= 4e-7
