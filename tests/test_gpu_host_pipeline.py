"""jd_decide_host_submit / jd_decide_host_collect: two host calls in flight on one
handle ("Julia-1 MLX", "Performance": a server scoring a stream of requests).

The outputs of pipelined calls must equal those of jd_decide_host on the same
rows bit for bit (the same kernels on the same packed batches; each call keeps
its own pinned staging slot and its own copy of the status word).  The rules:
at most two calls in flight, tickets collected in order, no synchronous host
call while a submitted one is uncollected; graph mode works through the
pipeline too.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import rows_config1, rows_config2

pytestmark = pytest.mark.gpu

KEYS = ("logits", "probs", "choice", "score", "noul", "max_p")


def _same(a, b):
    for k in KEYS:
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)


def test_two_calls_in_flight(weights_file):
    from encoder_decision_model_b200.build import build
    build()
    m = jl.Model(weights_file, 1 << 17, 256, 4096)
    opts = jl.encode_opts(1024, 512, True)
    batches = [rows_config2(48, seed=s) for s in (31, 32, 33)]
    ref = [m.jd_decide_host(b, opts) for b in batches]

    t0 = m.jd_decide_host_submit(batches[0], opts)
    t1 = m.jd_decide_host_submit(batches[1], opts)
    assert (t0, t1) == (0, 1)
    with pytest.raises(jl.JDError) as ei:  # a third call in flight
        m.jd_decide_host_submit(batches[2], opts)
    assert ei.value.code == jl.JD_ERR_INVALID_ARG
    with pytest.raises(jl.JDError):  # no synchronous call meanwhile
        m.jd_decide_host(batches[2], opts)
    _same(m.jd_decide_host_collect(t0), ref[0])
    t2 = m.jd_decide_host_submit(batches[2], opts)
    _same(m.jd_decide_host_collect(t1), ref[1])
    _same(m.jd_decide_host_collect(t2), ref[2])
    # a long stream through the two slots
    out = []
    inflight = []
    for k in range(7):
        inflight.append((k % 3, m.jd_decide_host_submit(batches[k % 3], opts)))
        if len(inflight) == 2:
            i, t = inflight.pop(0)
            out.append((i, m.jd_decide_host_collect(t)))
    for i, t in inflight:
        out.append((i, m.jd_decide_host_collect(t)))
    for i, o in out:
        _same(o, ref[i])
    # synchronous calls work again once nothing is in flight
    _same(m.jd_decide_host(batches[0], opts), ref[0])

    # graph mode (bucketed graphs) through the pipeline
    reqs = [rows_config1(seed=101 + k) for k in range(4)]
    eager = [m.jd_decide_host(r, opts) for r in reqs]
    m.jd_set_graph_mode(True)
    try:
        ts = []
        got = []
        for r in reqs:
            ts.append(m.jd_decide_host_submit(r, opts))
            if len(ts) == 2:
                got.append(m.jd_decide_host_collect(ts.pop(0)))
        got += [m.jd_decide_host_collect(t) for t in ts]
    finally:
        m.jd_set_graph_mode(False)
    for a, b in zip(got, eager):
        _same(a, b)
    m.close()
