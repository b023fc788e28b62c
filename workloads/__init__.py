"""Seeded synthetic inputs shared by the oracle, the tests and the benchmark.

This package draws random numbers and lays them out; it performs none of the
model's arithmetic (no norms, no projections, no serialisation).  Both the
oracle and the CUDA library consume what it writes, each with its own reader.
"""
from .gen import (  # noqa: F401
    ARCH,
    Row,
    RouterRequest,
    weight_specs,
    write_weights,
    weights_path,
    read_weight_index,
    rows_config0,
    rows_config1,
    rows_config2,
    rows_config3,
    requests_config4,
    worked_example_rows,
    SPECIAL,
)
