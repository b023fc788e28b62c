"""The multi-GPU protocol of bench.py on CPU: two gloo ranks, each with its own
shard of rows (independent decisions, no collective on the data path), the
barrier and the max-over-ranks timing, and the reference arm on rank 0 only."""
import json
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import torch.distributed as dist
    import bench
    from encoder_decision_model_b200 import _lib as jl

    dist.init_process_group("gloo", rank=rank, world_size=world)
    class A:  # the fields bench.workload reads
        workload = "throughput"
        rows = 8
    rows, opts, _ = bench.workload(A, rank)
    hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
    ranks = bench.Ranks(world, "cpu")
    ranks.barrier()
    seconds = 1.0 + rank  # rank 1 is the slow one
    rate = bench.whole_job_rate(hb.n_rows, seconds, ranks)
    tmax = ranks.max(seconds)
    json.dump(dict(rank=rank, tokens=hb.tokens[:16].tolist(), n_tokens=hb.n_tokens, rate=rate, tmax=tmax),
              open(os.path.join(out_dir, f"r{rank}.json"), "w"))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks(tmp_path):
    import torch.multiprocessing as mp
    from encoder_decision_model_b200.build import build
    build()
    port = _free_port()
    mp.start_processes(_worker, args=(2, port, str(tmp_path)), nprocs=2, start_method="spawn", join=True)
    r0 = json.load(open(tmp_path / "r0.json"))
    r1 = json.load(open(tmp_path / "r1.json"))
    # each rank has its own rows (different seeds), deterministic per rank
    assert r0["tokens"] != r1["tokens"]
    sys.path.insert(0, ROOT)
    import bench
    class A:
        workload = "throughput"
        rows = 8
    from encoder_decision_model_b200 import _lib as jl
    for r, rec in ((0, r0), (1, r1)):
        rows, opts, _ = bench.workload(A, r)
        hb = jl.jd_serialize(rows, jl.encode_opts(**opts))
        assert hb.tokens[:16].tolist() == rec["tokens"]
    # whole-job value: all ranks' units over the slowest rank's time
    assert r0["tmax"] == r1["tmax"] == 2.0
    assert r0["rate"] == r1["rate"] == pytest.approx((8 + 8) / 2.0)


def test_reference_arm_runs_on_rank0_only(capsys, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    class A:
        workload = "throughput"
        rows = 8
        steps = 1
        warmup = 0
        gpus = 2
    bench.run_reference(A)
    assert capsys.readouterr().out == ""


def test_four_thread_oracle_leg():
    """The cpu_baseline's 4-thread figure runs the same oracle with NumPy's BLAS
    held to 4 threads, and reports that count."""
    import bench
    sys_argv = sys.argv
    sys.argv = ["bench.py", "--rows", "4"]
    try:
        args = bench.parse()
    finally:
        sys.argv = sys_argv
    rows, opts, _ = bench.workload(args, 0)
    before = bench.blas_threads()
    r = bench.oracle_four_threads(rows[:2], opts, 0.0)
    assert r is not None and r["value"] > 0 and r["unit"] == bench.UNIT
    assert r["cores"] == 4
    assert bench.blas_threads() == before  # the limit is lifted afterwards
