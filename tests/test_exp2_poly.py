"""The FMA-pipe 2^x of the global attention softmax (csrc/attention_tc.cu,
`ex2_poly2`), emulated in float32 from the constants in the source.

x = j + f with j = round(x) and f in [-1/2, 1/2]; 2^f by a degree-3 polynomial
fitted for the least maximum relative error on [-1/2, 1/2] (Remez exchange);
2^j added into the exponent field.  The attention probabilities it produces
are rounded to bf16 (relative half-ulp 2^-9), so the bound that matters is
far looser than the one held here (7.6e-5).
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "encoder_decision_model_b200",
                   "csrc", "attention_tc.cu")


def _coeffs():
    txt = open(SRC).read()
    return [np.float32(float(re.search(rf"EX2_C{k} = ([0-9.eE+-]+)f", txt).group(1))) for k in range(4)]


def _ex2_poly(x):
    """The routine step by step in float32 (round to nearest even, as add.rn)."""
    c0, c1, c2, c3 = _coeffs()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-126.0))
    magic = np.float32(12582912.0)
    t = (x + magic).astype(np.float32)
    j = (t - magic).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = (f * c3 + c2).astype(np.float32)   # fma: one rounding; the product is exact enough in float64 here
    p = (p.astype(np.float64) * f + c1).astype(np.float32)
    p = (p.astype(np.float64) * f + c0).astype(np.float32)
    bits = p.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_fraction_polynomial_bound():
    c = [float(v) for v in _coeffs()]
    f = np.linspace(-0.5, 0.5, 200001)
    p = c[0] + f * (c[1] + f * (c[2] + f * c[3]))
    rel = np.abs(p / np.exp2(f) - 1.0)
    assert rel.max() <= 7.6e-5
    # minimax: the error equioscillates, so both ends and the interior reach the bound
    assert rel[0] > 5e-5 and rel[-1] > 5e-5


def test_whole_routine_over_the_softmax_range():
    # the softmax feeds x = s / 8 * log2(e) - m <= 8 (lazy maximum) and as low as -inf (masked keys)
    x = np.concatenate([np.linspace(-125.9, 8.5, 400001), -np.arange(0, 126, 0.5)]).astype(np.float32)
    y = _ex2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 7.6e-5, float(rel.max())
    # integers come out as 2^j times p(0) ~ 1 - 7.2e-5
    np.testing.assert_allclose(_ex2_poly(np.array([0.0, 1.0, -3.0, 8.0], np.float32)), [1, 2, 0.125, 256], rtol=8e-5)


def test_masked_keys_give_a_negligible_normal_number():
    y = _ex2_poly(np.array([-np.inf, -1e30, -126.0, -200.0], np.float32))
    assert np.all(y > 0) and np.all(y < 2.0 ** -125) and np.all(np.isfinite(y))
