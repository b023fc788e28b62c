"""The library's Router tournament ("Julia-1: one score per mask token", "More
than 20 options: the Router") on the CPU: jd_route_scored runs the same
grouping, survivor rule and final call as jd_route_host with the scoring left
to a callback.  Driven here and in the oracle's tournament by the same float32
probabilities, the two must agree exactly: winners, final candidates and their
probabilities, and the rows scored per round (the library batches all requests
of a round together, so it scores the sum of the oracle's per-request calls).

A label's logit is a hash of its first id times a scale; large scales give
groups with one confident winner (the single-survivor branch), small ones keep
the top two.  Label i of every request starts with id 10 + i.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from oracle import route
from workloads import RouterRequest

N_LABELS = [1, 2, 3, 20, 21, 22, 40, 41, 60, 72, 399, 400, 1000, 4095, 4096]
SCALES = [0.5, 4.0, 12.0, 40.0]


def _unit(first_id):
    return ((int(first_id) * 2654435761) % (1 << 32)) / float(1 << 32)


def _probs(first_ids, scale):
    z = np.array([scale * _unit(i) for i in first_ids], np.float64)
    e = np.exp(z - z.max())
    return (e / e.sum()).astype(np.float32)


def _request(rng, n):
    labels = [np.concatenate([[10 + i], rng.integers(10, 1000, size=int(rng.integers(0, 5)))]).astype(np.int32)
              for i in range(n)]
    return RouterRequest(state=np.array([7, 8, 9], np.int32), question=np.array([5, 6], np.int32), labels=labels)


def _lib_scorer(scale):
    return lambda rows: [_probs([opt[0] for opt in row], scale) for row in rows]


def _oracle_scorer(scale):
    return lambda groups: [_probs([10 + i for i in g], scale) for g in groups]


def _top2_final_count(n):
    """Candidates left for the final call when every group keeps two."""
    while n > 20:
        q, r = divmod(n, 20)
        n = 2 * q + min(r, 2)
    return n


@pytest.fixture(scope="module")
def lib_built():
    from encoder_decision_model_b200.build import build
    build()
    return jl.lib()


@pytest.mark.parametrize("scale", SCALES)
def test_scored_router_matches_oracle(lib_built, scale):
    rng = np.random.default_rng(int(scale * 10))
    reqs = [_request(rng, n) for n in N_LABELS]
    got = jl.jd_route_scored(reqs, _lib_scorer(scale))
    grouped, finals = [], 0
    single_winner_seen = False
    for r, q in enumerate(reqs):
        cands, p, winner, calls = route(len(q.labels), _oracle_scorer(scale))
        fc = got["final_candidates"][r]
        assert fc[fc >= 0].tolist() == cands, (len(q.labels), scale)
        np.testing.assert_array_equal(got["final_probs"][r][:len(cands)], np.asarray(p, np.float32))
        assert got["winner"][r] == winner
        # the oracle's calls: grouped rounds, then one final call when two or more remain
        final = 1 if len(cands) >= 2 else 0
        for i, c in enumerate(calls[:len(calls) - final]):
            if i == len(grouped):
                grouped.append(0)
            grouped[i] += c
        finals += final
        if len(cands) < _top2_final_count(len(q.labels)):
            single_winner_seen = True
    # the library scores each grouped round for all requests still above 20 candidates, then
    # every request's final row together once the last grouped round is done
    assert got["rows_per_round"].tolist() == grouped + ([finals] if finals else [])
    if scale >= 12.0:
        assert single_winner_seen, "the single-survivor branch was not exercised"


def test_scored_router_errors(lib_built):
    q = RouterRequest(state=np.array([1], np.int32), question=np.array([2], np.int32),
                      labels=[np.array([10 + i], np.int32) for i in range(30)])

    def failing(rows):
        raise RuntimeError("scorer failed")

    with pytest.raises(RuntimeError, match="scorer failed"):
        jl.jd_route_scored([q], failing)

    def short(rows):
        return [np.ones(1, np.float32) for _ in rows]

    with pytest.raises(ValueError):
        jl.jd_route_scored([q], short)
