"""Pins of the oracle read-outs and the router's narrowing rule."""
import os

import numpy as np
import pytest

from oracle import readouts, softmax, route, survivors

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_softmax_sums_to_one_and_is_shift_invariant():
    rng = np.random.default_rng(0)
    for k in (2, 7, 20):
        z = rng.normal(size=k) * 5
        p = softmax(z)
        assert abs(p.sum() - 1) < 1e-15 and (p > 0).all()
        np.testing.assert_allclose(softmax(z + 1000.0), p, rtol=1e-12)


def test_two_equal_logits():
    r = readouts(np.array([0.3, 0.3]), qtype=2)
    assert r["probs"].tolist() == [0.5, 0.5] and r["choice"] == 0
    assert r["noul"] == 0.5 and r["score"] == 0.5 and r["max_p"] == 0.5


def test_readouts_closed_forms():
    z = np.log(np.array([1.0, 2.0, 7.0]))       # p = [0.1, 0.2, 0.7]
    r = readouts(z, qtype=1)
    np.testing.assert_allclose(r["probs"], [0.1, 0.2, 0.7], atol=1e-15)
    assert r["choice"] == 2 and abs(r["score"] - (0.2 + 1.4)) < 1e-14
    assert np.isnan(r["noul"]) and abs(r["max_p"] - 0.7) < 1e-15
    r = readouts(np.log(np.array([3.0, 1.0])), qtype=2)
    assert abs(r["noul"] - 0.25) < 1e-15 and r["choice"] == 0


def test_score_range():
    rng = np.random.default_rng(1)
    for _ in range(100):
        k = int(rng.integers(2, 21))
        s = readouts(rng.normal(size=k) * 10, 1)["score"]
        assert 0.0 <= s <= k - 1


def test_argmax_tie_lowest_index():
    assert readouts(np.array([0.0, 2.0, 2.0, 1.0]), 0)["choice"] == 1


def test_survivor_rule():
    assert survivors([0.96, 0.02, 0.02]) == [0]
    assert survivors([0.96, 0.039, 0.001]) == [0]
    assert survivors([0.95, 0.025, 0.025]) == [0, 1]          # not strictly above 0.95
    assert survivors([0.951, 0.045, 0.004]) == [0, 1]         # an other not below 0.045
    assert survivors([0.1, 0.5, 0.4]) == [1, 2]               # top two, original order
    assert survivors([0.3, 0.3, 0.4]) == [0, 2]               # tie -> lower index


def _golden_calls():
    out = []
    for line in open(os.path.join(GOLD, "router_calls.txt")):
        if line.startswith("#") or not line.strip():
            continue
        n, *calls = map(int, line.split())
        out.append((n, calls))
    return out


@pytest.mark.parametrize("n,calls", _golden_calls())
def test_router_call_counts(n, calls):
    rng = np.random.default_rng(n)

    def score(groups):
        return [softmax(rng.normal(size=len(g))) for g in groups]

    _, _, _, got = route(n, score)
    assert got == calls


def test_router_keeps_confident_winner_and_ordering():
    # candidate 45 wins its group decisively, others lose: it must survive and win
    def score(groups):
        out = []
        for g in groups:
            z = np.zeros(len(g))
            if 45 in g:
                z[g.index(45)] = 10.0
            else:
                z[:] = -np.arange(len(g))
            out.append(softmax(z))
        return out

    cands, p, win, calls = route(60, score)
    assert win == 45 and calls == [3, 1]
    assert cands == sorted(cands) and 45 in cands and len(cands) == 5  # 2 + 1 + 2


def test_router_group_of_one_passes_without_call():
    seen = []

    def score(groups):
        seen.extend(len(g) for g in groups)
        return [softmax(np.zeros(len(g))) for g in groups]

    _, _, _, calls = route(41, score)        # 20 + 20 + 1
    assert 1 not in seen[:2] and calls[0] == 2


def _closed_form_calls(n):
    """Calls per round when no group ever keeps a single winner: a round over n > 20
    candidates scores floor(n/20) full groups plus the tail group if it holds two or
    more (a tail of one passes unscored), and leaves 2 floor(n/20) + min(n mod 20, 2);
    at 20 or fewer, one final call if two or more remain."""
    calls = []
    while n > 20:
        q, r = divmod(n, 20)
        calls.append(q + (1 if r >= 2 else 0))
        n = 2 * q + min(r, 2)
    if n >= 2:
        calls.append(1)
    return calls


@pytest.mark.parametrize("n", [1, 2, 20, 21, 22, 40, 41, 60, 72, 399, 400, 401, 1000, 4095, 4096])
def test_router_call_counts_closed_form(n):
    """Uniform probabilities in every group (p = 1/size <= 1/2 < 0.95): never a single
    winner, so the counts follow the closed form; 4,096 is the pages' maximum."""
    _, _, _, got = route(n, lambda groups: [np.full(len(g), 1.0 / len(g)) for g in groups])
    assert got == _closed_form_calls(n)


def test_router_closed_form_spot_values():
    # worked by hand: 4096 -> 205 calls, 410 left -> 21 calls, 42 left -> 3 calls, 6 left -> final
    assert _closed_form_calls(4096) == [205, 21, 3, 1]
    assert _closed_form_calls(41) == [2, 1]
    assert _closed_form_calls(1) == []
