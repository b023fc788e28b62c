"""Concurrent serving ("Julia-1 MLX", "Performance": single requests scored from
several threads, each on its own stream): handles made with jd_model_create_shared
share one copy of the weights, run on their own streams from their own host
threads, and give the same outputs as serial calls on the base handle."""
import threading

import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from workloads import rows_config1, rows_config2

pytestmark = pytest.mark.gpu


def test_shared_handles_on_concurrent_streams(weights_file):
    import torch
    from encoder_decision_model_b200.build import build
    build()
    base = jl.Model(weights_file, 16384, 32, 640)
    opts = jl.encode_opts(1024, 512, True)
    requests = [rows_config1(seed=101 + i) for i in range(6)] + [rows_config2(16, seed=300 + i) for i in range(2)]
    serial = [base.jd_decide_host(r, opts) for r in requests]

    shared = [jl.Model.shared(base, 16384, 32, 640) for _ in range(2)]
    assert all(s.device_bytes() < base.device_bytes() for s in shared)  # no second copy of the weights
    results = [[None] * len(requests) for _ in shared]
    errors = []

    def serve(k):
        try:
            st = torch.cuda.Stream()
            for rep in range(3):
                for i, r in enumerate(requests):
                    results[k][i] = shared[k].jd_decide_host(r, opts, stream=st)
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=serve, args=(k,)) for k in range(len(shared))]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for k in range(len(shared)):
        for i in range(len(requests)):
            for key in ("logits", "probs", "choice", "score", "max_p"):
                np.testing.assert_array_equal(results[k][i][key], serial[i][key], err_msg=f"handle {k} request {i} {key}")
    for s in shared:
        s.jd_check_status()
        s.close()
    base.close()
