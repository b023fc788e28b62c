"""Router rounds on the device (jd_route_device) against jd_route_host ("Julia-1: one
score per mask token", "More than 20 options: the Router").

jd_route_device forms, encodes and packs every round's rows with kernels and applies
the survivor rule on the device.  A row's result does not depend on the other rows
of its batch, and the device encoding follows the host serializer's layout and
budget rules, so every output must equal jd_route_host's bit for bit: winners,
their probabilities, the final candidates and probabilities, the rows per round.
jd_route_host itself is held to the oracle's tournament in
tests/test_gpu_router_rounds.py.

Cases: the router workload (72 labels, two rounds); one and three-round
tournaments (1, 2, 20, 21, 333 and 1000 labels in one call); non-strict encoding
with labels over 48 ids and a head budget that forces the common option cap and
the question clip; strict overflow; a round beyond the capacity.
"""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import RouterRequest, requests_config4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def model(weights_file):
    from encoder_decision_model_b200.build import build
    build()
    m = jl.Model(weights_file, 1 << 18, 1024, 1024 * 20)
    yield m
    m.close()


def _same(a, b):
    for k in ("winner", "winner_p", "final_candidates", "final_probs", "rows_per_round"):
        np.testing.assert_array_equal(np.asarray(a[k]), np.asarray(b[k]), err_msg=k)


def test_router_workload_matches_host_rounds(model):
    reqs = requests_config4(96, seed=211)
    opts = jl.encode_opts(1024, 512, True)
    host = model.jd_route_host(reqs, opts)
    dev = model.jd_route_device(reqs, opts)
    _same(dev, host)
    assert dev["rows_per_round"].tolist() == [96 * 4, 96]
    # a second call reuses the workspace and gives the same bits
    _same(model.jd_route_device(reqs, opts), host)


def test_mixed_label_counts_and_three_rounds(model):
    rng = np.random.Generator(np.random.PCG64(5))
    ids = lambda n: rng.integers(10, 256000, size=n).astype(np.int32)
    reqs = []
    for n in (1000, 1, 2, 20, 21, 333, 40):
        reqs.append(RouterRequest(state=ids(200), question=ids(int(rng.integers(8, 25))),
                                  labels=[ids(int(rng.integers(1, 13))) for _ in range(n)]))
    opts = jl.encode_opts(1024, 512, True)
    host = model.jd_route_host(reqs, opts)
    dev = model.jd_route_device(reqs, opts)
    _same(dev, host)
    assert len(dev["rows_per_round"]) == 3
    assert dev["winner"][1] == 0 and dev["winner_p"][1] == 1.0


def test_non_strict_truncation_rules(model):
    rng = np.random.Generator(np.random.PCG64(9))
    ids = lambda n: rng.integers(10, 256000, size=n).astype(np.int32)
    reqs = [
        # options over 48 ids, clipped to 48
        RouterRequest(state=ids(300), question=ids(20), labels=[ids(int(rng.integers(30, 70))) for _ in range(45)]),
        # a head budget of 160 forces one common cap on the options
        RouterRequest(state=ids(900), question=ids(24), labels=[ids(int(rng.integers(5, 40))) for _ in range(30)]),
        # long question: with 20 options the cap falls to one id and the question is clipped
        RouterRequest(state=ids(50), question=ids(150), labels=[ids(int(rng.integers(2, 9))) for _ in range(26)]),
    ]
    opts = jl.encode_opts(512, 160, False)
    host = model.jd_route_host(reqs, opts)
    dev = model.jd_route_device(reqs, opts)
    _same(dev, host)


def test_strict_overflow_and_capacity(model, weights_file):
    rng = np.random.Generator(np.random.PCG64(3))
    ids = lambda n: rng.integers(10, 256000, size=n).astype(np.int32)
    long_label = RouterRequest(state=ids(100), question=ids(10), labels=[ids(60)] + [ids(5) for _ in range(24)])
    opts = jl.encode_opts(1024, 512, True)
    for call in (model.jd_route_host, model.jd_route_device):
        with pytest.raises(jl.JDError) as ei:
            call([long_label], opts)
        assert ei.value.code == jl.JD_ERR_OVERFLOW
    # the model still serves after the error
    ok = requests_config4(4, seed=3)
    _same(model.jd_route_device(ok, opts), model.jd_route_host(ok, opts))
    # a round beyond the capacity of a small model: an error, no device work past the counts
    small = jl.Model(weights_file, 4096, 8, 160)
    with pytest.raises(jl.JDError) as ei:
        small.jd_route_device(requests_config4(8, seed=4), opts)
    assert ei.value.code == jl.JD_ERR_CAPACITY
    small.close()
