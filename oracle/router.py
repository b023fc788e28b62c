"""The router's narrowing tournament (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

"Julia-1: one score per mask token", § "More than 20 options: the Router":
split the candidates in order into consecutive groups of at most 20, score all
groups in one batch, keep a group's winner alone when its probability is above
0.95 and every other option is below 0.045, otherwise keep its top two; repeat
until 20 or fewer remain, then make one final call.  The page's arithmetic
(60 options -> 3 + 1 calls, 72 -> 4 + 1) pins the call counts.

Readings: the inequalities are strict; the top two are the two highest
probabilities, the lower index first on ties; survivors keep their original
relative order; a group of one candidate passes through without a call.
Parity: pinned by the call counts above and synthetic-probability cases in
tests/test_oracle_router.py.
"""
from __future__ import annotations

import numpy as np

GROUP = 20


def survivors(p):
    """Indices (ascending) kept from one group with probabilities p."""
    p = np.asarray(p, dtype=np.float64)
    order = sorted(range(len(p)), key=lambda i: (-p[i], i))
    best = order[0]
    if p[best] > 0.95 and all(p[i] < 0.045 for i in range(len(p)) if i != best):
        return [best]
    return sorted(order[:2])


def route(n_candidates, score_groups):
    """Run the tournament.

    score_groups(list of candidate-index lists) -> list of probability arrays,
    one batch per round.  Returns (final candidate indices, final probs,
    winner index, number of rows scored per round).
    """
    cands = list(range(n_candidates))
    calls = []
    while len(cands) > GROUP:
        groups = [cands[i:i + GROUP] for i in range(0, len(cands), GROUP)]
        scored = [g for g in groups if len(g) > 1]
        probs = iter(score_groups(scored)) if scored else iter(())
        calls.append(len(scored))
        nxt = []
        for g in groups:
            if len(g) == 1:
                nxt += g
                continue
            keep = survivors(next(probs))
            nxt += [g[i] for i in keep]
        cands = nxt
    if len(cands) == 1:
        return cands, np.ones(1), cands[0], calls
    (p,) = score_groups([cands])
    calls.append(1)
    p = np.asarray(p, dtype=np.float64)
    return cands, p, cands[int(np.argmax(p))], calls
