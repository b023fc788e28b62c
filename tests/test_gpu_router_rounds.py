"""Router tournaments of several rounds ("Julia-1: one score per mask token",
"More than 20 options: the Router"): jd_route_host against the oracle's
tournament rule driven by the same device probabilities.

A row's result does not depend on the other rows of its packed batch, so scoring
each round's groups through jd_decide_host gives exactly the probabilities
jd_route_host sees; the survivors, the rows per round and the winner must then
agree exactly.  1000 labels take three calls (1000 -> 50 groups -> <= 100 ->
5 groups -> <= 10 -> final call), 333 labels too (17 groups, 2 groups, final).
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from oracle import route
from workloads import Row, requests_config4

pytestmark = pytest.mark.gpu


def test_multi_round_tournaments(weights_file):
    from encoder_decision_model_b200.build import build
    build()
    reqs = requests_config4(1, seed=7, n_labels=1000) + requests_config4(1, seed=8, n_labels=333)
    opts = jl.encode_opts(1024, 512, True)
    model = jl.Model(weights_file, 1 << 18, 256, 256 * 20)
    out = model.jd_route_host(reqs, opts)

    per_round = []
    for r, q in enumerate(reqs):
        def score_groups(groups, q=q):
            rows = [Row(state=q.state, question=q.question, options=[q.labels[i] for i in g], qtype=0)
                    for g in groups]
            ho = model.jd_decide_host(rows, opts)
            off = np.cumsum([0] + [len(g) for g in groups])
            return [ho["probs"][off[i]:off[i + 1]] for i in range(len(groups))]

        cands, p, winner, calls = route(len(q.labels), score_groups)
        fc = out["final_candidates"][r]
        assert fc[fc >= 0].tolist() == cands
        np.testing.assert_array_equal(out["final_probs"][r][:len(cands)], np.asarray(p, dtype=np.float32))
        assert out["winner"][r] == winner
        for i, c in enumerate(calls):
            if i == len(per_round):
                per_round.append(0)
            per_round[i] += c
    # rounds are batched across requests in jd_route_host: compare the row counts per round
    assert out["rows_per_round"].tolist() == per_round
    assert len(per_round) == 3
    model.close()
