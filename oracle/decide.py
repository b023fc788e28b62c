"""Per-question read-outs (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

"Julia-1: one score per mask token", § "Three modes through one head": the
probabilities are a softmax across the options at temperature 1 with nothing
fitted; choice reads the argmax, score the expected index sum_i i * p_i, noul
p(true) where the options are always [false, true].  Readings: the argmax
takes the lowest index among equal maxima; score is reported for every row
(the caller reads it for score rows); noul is NaN for rows that are not noul.
Parity: pinned by closed forms (sum p = 1, two equal logits -> 0.5 / choice 0,
score range [0, K-1]) in tests/test_oracle_decide.py.
"""
from __future__ import annotations

import numpy as np


def softmax(z):
    z = np.asarray(z, dtype=np.float64)
    e = np.exp(z - z.max())
    return e / e.sum()


def readouts(z, qtype):
    """Return dict(probs, choice, score, noul, max_p) for one row's logits z [K]."""
    p = softmax(z)
    choice = int(np.argmax(p))  # first index of the maximum
    score = float(np.sum(np.arange(len(p)) * p))
    noul = float(p[1]) if qtype == 2 else float("nan")
    return dict(probs=p, choice=choice, score=score, noul=noul, max_p=float(p.max()))
