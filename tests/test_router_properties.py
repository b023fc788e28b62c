"""Property-based check of the library's Router tournament against the oracle's
("More than 20 options: the Router"): every label carries a float32 value drawn
from a set around the rule's thresholds (exactly 0.95 and 0.045 as float32,
their float32 neighbours, ties), used as its probability in every call.  The
library and the oracle must keep the same survivors in the same order and pick
the same winner (lowest index among equal maxima)."""
import numpy as np
from hypothesis import HealthCheck, given, settings, strategies as st

from encoder_decision_model_b200 import _lib as jl
from oracle import route
from workloads import RouterRequest

F = np.float32
VALUES = [F(0.95), np.nextafter(F(0.95), F(1)), np.nextafter(F(0.95), F(0)), F(0.045),
          np.nextafter(F(0.045), F(0)), np.nextafter(F(0.045), F(1)), F(0.5), F(0.0), F(1.0), F(0.3), F(0.3)]


@settings(max_examples=200, deadline=None, suppress_health_check=[HealthCheck.too_slow, HealthCheck.data_too_large])
@given(table=st.lists(st.sampled_from(range(len(VALUES))), min_size=1, max_size=130))
def test_router_thresholds_and_ties(table):
    from encoder_decision_model_b200.build import build
    build()
    val = np.array([VALUES[i] for i in table], np.float32)
    n = len(val)
    labels = [np.array([10 + i], np.int32) for i in range(n)]
    req = RouterRequest(state=np.array([7], np.int32), question=np.array([5], np.int32), labels=labels)
    got = jl.jd_route_scored([req], lambda rows: [val[[int(o[0]) - 10 for o in row]] for row in rows])
    cands, p, winner, calls = route(n, lambda groups: [val[list(g)] for g in groups])
    fc = got["final_candidates"][0]
    assert fc[fc >= 0].tolist() == cands
    assert got["winner"][0] == winner
    np.testing.assert_array_equal(got["final_probs"][0][:len(cands)], np.asarray(p, np.float32))
    assert got["rows_per_round"].tolist() == calls
