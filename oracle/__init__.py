"""CPU oracle for the Julia-1 decision-model forward pass.

TEST INFRASTRUCTURE ONLY.  This package is the plain, slow, obviously correct
statement of what the library computes: the marker serialiser with its
budgets, the encoder and decision-head forward pass in float64 NumPy (dense
per-row attention, no packing, no fusion), the per-question read-outs and the
router's narrowing rule.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import it; the library never does, and it shares no code
with the CUDA path.

Sources (page title, section):
  * "Julia-1: one score per mask token" -- "From a state to one decision"
    (layout, budgets, strict mode), "The decision head" (forward steps 1-4),
    "Three modes through one head" (read-outs), "More than 20 options: the
    Router" (tournament rule).
  * "Julia-1 MLX" -- "Performance" (alternating global / +-64 local attention,
    FP32 residual stream), "Fine-tuning and export" (head layers are PyTorch
    TransformerEncoderLayers).
  * "julia1 -- Rust runtime for Julia-1" -- "Why it is faster" (GEGLU,
    bias / ReLU epilogues, marker-only last head layer).

Parity status per function is listed in the module docstrings; every function
here has at least one pin in tests/test_oracle_*.py, and the whole chain of
"The decision head" (encoder, final norm, type row, both head layers, gather,
scorer) has a closed-form pin on tiny structured weights.  Logits of the
trained model are not pinned: no page provides a checkpoint or its outputs.
"""
from .serialize import (  # noqa: F401
    EncodeOptions, EncodingError, Encoded, serialize_row, serialize_rows,
    ERR_OK, ERR_INVALID_ARG, ERR_OPTION_COUNT, ERR_OVERFLOW, ERR_TOKEN_RANGE,
    TRUNC_OPTION_48, TRUNC_OPTION_CAP, TRUNC_QUESTION, TRUNC_STATE,
)
from .model import OracleModel, ModelOptions  # noqa: F401
from .decide import readouts, softmax  # noqa: F401
from .router import route, survivors  # noqa: F401
