"""Write the oracle's outputs for sampled rows of the long-context workload.

The float64 oracle needs minutes per 8192-token row, so the GPU parity test
compares against values stored here.  This script calls only the oracle and
the seeded input generators:

    python tests/golden/make_long_context_golden.py

Output: tests/golden/long_context_rows.npz with, per sampled row i,
  logits_i [20], marker_state_i [20, 384], enc_pos_i [P], encoder_out_i [P, 384]
(encoder output after the final norm at P sampled positions, float32).
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

from oracle import EncodeOptions, OracleModel, serialize_row  # noqa: E402
from workloads import rows_config3, weights_path  # noqa: E402

ROWS = (0, 9)


def main():
    m = OracleModel(weights_path(0))
    rows = rows_config3(16)
    eo = EncodeOptions(max_length=8192, head_budget=256, strict=False)
    out = {}
    rng = np.random.default_rng(1234)
    for i in ROWS:
        e = serialize_row(rows[i], eo)
        r = m.forward_all(e)
        pos = np.unique(np.concatenate([np.arange(0, 8), e.mask_pos, rng.integers(0, len(e.ids), 48),
                                        np.arange(len(e.ids) - 8, len(e.ids))])).astype(np.int32)
        out[f"logits_{i}"] = r["logits"]
        out[f"marker_state_{i}"] = r["marker_state"].astype(np.float32)
        out[f"enc_pos_{i}"] = pos
        out[f"encoder_out_{i}"] = r["encoder_out"][pos].astype(np.float32)
        print(f"row {i}: {len(e.ids)} tokens, logits {r['logits'][:3]}", flush=True)
    np.savez_compressed(os.path.join(HERE, "long_context_rows.npz"), rows=np.asarray(ROWS), **out)


if __name__ == "__main__":
    main()
