"""The BF16 GEGLU epilogue's GELU (csrc/gemm.cu, `geglu_pair`), emulated in float32
from the constants in the source.

GELU(x) = x Phi(x) = max(x, 0) - |x| Phi(-|x|), with the normal tail
Phi(-a) = 2^(P(a / 6) - a^2 log2(e) / 2) and P the degree-7 polynomial of least
maximum error against log2 Phi(-6 s) + 18 s^2 log2(e) on s in [0, 1] (Remez
exchange), held at s = 1 past |x| = 6.  The exact reference is scipy's log_ndtr
and erf in float64.  ex2 is taken exact here (the instruction's own relative
error, about 2^-22, adds at most 2.4e-7 relative to the tail); the output is
rounded to bf16 afterwards (relative half-ulp 2^-9), so the bounds held here are
far inside what reaches the next GEMM.
"""
import os
import re

import numpy as np
from scipy.special import erf, log_ndtr

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "encoder_decision_model_b200",
                   "csrc", "gemm.cu")
LOG2E = np.log2(np.e)


def _constants():
    txt = open(SRC).read()
    c = [float(re.search(rf"GT_C{k} = ([0-9.eE+-]+)f", txt).group(1)) for k in range(8)]
    g = float(re.search(r"GT_G = ([0-9.eE+-]+)f", txt).group(1))
    return [np.float32(v) for v in c], np.float32(g)


def _target(s):
    return log_ndtr(-6.0 * s) / np.log(2) + 18.0 * s * s * LOG2E


def _f32(v):
    return np.asarray(v, np.float64).astype(np.float32)


def _gelu_pair(x, g):
    """geglu_pair step by step: every f32x2 multiply and fma rounded once to float32."""
    c, G = _constants()
    x = _f32(x)
    g = _f32(g)
    na = -np.abs(x)
    s = _f32(na.astype(np.float64) * np.float64(np.float32(-1.0 / 6.0)))
    sc = np.minimum(s, np.float32(1.0))
    p = _f32(sc.astype(np.float64) * c[7] + c[6])
    for k in (5, 4, 3, 2, 1, 0):
        p = _f32(p.astype(np.float64) * sc + c[k])
    s2 = _f32(s.astype(np.float64) * s)
    arg = _f32(s2.astype(np.float64) * G + p)
    t = _f32(np.exp2(arg.astype(np.float64)))
    t = np.where(arg < -126.0, np.float32(0.0), t)  # .ftz: results below 2^-126 flush to zero
    y = _f32(na.astype(np.float64) * t + np.maximum(x, np.float32(0.0)))
    return _f32(y.astype(np.float64) * g)


def _gelu_exact(x):
    x = np.asarray(x, np.float64)
    return 0.5 * x * (1.0 + erf(x / np.sqrt(2.0)))


def test_constants_are_the_stated_scalars():
    _, G = _constants()
    np.testing.assert_allclose(float(G), -36.0 * LOG2E / 2.0, rtol=1e-7)


def test_tail_polynomial_bound():
    c, _ = _constants()
    s = np.linspace(0.0, 1.0, 400001)
    p = np.polyval([float(v) for v in c[::-1]], s)
    err = p - _target(s)
    assert np.abs(err).max() <= 4.8e-6, float(np.abs(err).max())
    # a minimax fit equioscillates: both ends and an interior point reach the bound
    assert abs(err[0]) > 4.5e-6 and abs(err[-1]) > 4.5e-6
    assert np.abs(err[150000:250000]).max() > 4.5e-6


def test_whole_routine_against_erf_gelu():
    x = np.concatenate([np.linspace(-40.0, 40.0, 800001), np.array([0.0, -0.0, 1e-30, -1e-30, 6.0, -6.0])])
    y = _gelu_pair(x, np.ones_like(x)).astype(np.float64)
    ref = _gelu_exact(_f32(x).astype(np.float64))
    err = np.abs(y - ref)
    # absolute error below 1e-6 plus the float32 rounding of the result
    assert np.all(err <= 1e-6 + 2.0 ** -23 * np.abs(ref)), float((err - 2.0 ** -23 * np.abs(ref)).max())
    # the negative side, where GELU is the tail itself: relative error
    neg = (x < -1e-3) & (x > -6.0)
    rel = np.abs(y[neg] / ref[neg] - 1.0)
    assert rel.max() <= 1e-5, float(rel.max())
    assert y[-6] == 0.0 and y[-5] == 0.0  # GELU(0) = 0 for both zeros


def test_gate_multiplies_and_special_points():
    x = np.array([-3.0, -1.0, -0.5, 0.5, 1.0, 3.0, 8.0, -8.0], np.float32)
    g = np.array([2.0, -1.5, 0.25, 4.0, -3.0, 1.0, 0.5, 7.0], np.float32)
    y = _gelu_pair(x, g).astype(np.float64)
    np.testing.assert_allclose(y, _gelu_exact(x) * g, rtol=2e-6, atol=1e-7)
    # GELU(x) - GELU(-x) = x, so the two halves meet without a seam at 0 and at |x| = 6
    xs = np.linspace(0.0, 10.0, 20001)
    d = _gelu_pair(xs, np.ones_like(xs)).astype(np.float64) - _gelu_pair(-xs, np.ones_like(xs)).astype(np.float64)
    np.testing.assert_allclose(d, _f32(xs), rtol=1e-6, atol=1e-6)
