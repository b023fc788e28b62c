"""Row sharding across ranks (host logic): every row in exactly one shard, the
load bound of longest-first greedy assignment, per-shard serialization equal to
the whole batch's row by row, and results merged back into row order."""
import numpy as np
import pytest

from encoder_decision_model_b200 import _lib as jl
from encoder_decision_model_b200.shard import merge_shards, shard_rows
from workloads import rows_config2


@pytest.mark.parametrize("n_shards", [1, 2, 3, 8, 50])
def test_shards_cover_rows_once_and_balance(n_shards):
    rng = np.random.default_rng(n_shards)
    lengths = rng.integers(64, 1025, size=37)
    parts = shard_rows(lengths, n_shards)
    assert len(parts) == n_shards
    flat = sorted(i for p in parts for i in p)
    assert flat == list(range(len(lengths)))
    assert all(p == sorted(p) for p in parts)
    loads = [int(lengths[p].sum()) if p else 0 for p in parts]
    # list scheduling: the last row placed on the fullest shard went to the least-loaded one
    assert max(loads) <= lengths.sum() / n_shards + lengths.max()


def test_shard_rows_rejects_zero_shards():
    with pytest.raises(ValueError):
        shard_rows([1, 2], 0)


def test_sharded_serialization_equals_whole_batch():
    rows = rows_config2(24)
    opts = jl.encode_opts(1024, 512, True)
    info = jl.jd_rows_encoding_info(rows, opts)
    whole = jl.jd_serialize(rows, opts)
    for part in shard_rows(info["length"], 3):
        hb = jl.jd_serialize([rows[i] for i in part], opts)
        for j, i in enumerate(part):
            a = whole.tokens[whole.cu_seqlens[i]:whole.cu_seqlens[i + 1]]
            b = hb.tokens[hb.cu_seqlens[j]:hb.cu_seqlens[j + 1]]
            np.testing.assert_array_equal(a, b)
            ma = whole.mask_pos[whole.opt_off[i]:whole.opt_off[i + 1]] - whole.cu_seqlens[i]
            mb = hb.mask_pos[hb.opt_off[j]:hb.opt_off[j + 1]] - hb.cu_seqlens[j]
            np.testing.assert_array_equal(ma, mb)


def test_merge_restores_row_order():
    rng = np.random.default_rng(3)
    n = 29
    k = rng.integers(2, 21, size=n)
    off = np.concatenate([[0], np.cumsum(k)])
    full = dict(choice=np.arange(n, dtype=np.int32) * 7, score=rng.random(n).astype(np.float32),
                logits=rng.normal(size=int(off[-1])).astype(np.float32))
    parts = shard_rows(rng.integers(1, 100, size=n), 4)
    results = []
    for p in parts:
        opt = np.concatenate([np.arange(off[i], off[i + 1]) for i in p]) if p else np.zeros(0, np.int64)
        results.append(dict(choice=full["choice"][p], score=full["score"][p], logits=full["logits"][opt]))
    out = merge_shards(parts, results, n, k)
    for key in full:
        np.testing.assert_array_equal(out[key], full[key])
