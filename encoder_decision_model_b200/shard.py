"""Row sharding across GPUs (host logic, no device work).

Rows are independent decisions ("Julia-1 MLX", "API": every row is scored on
its own; the packed batch gives each row the result it gets alone), so a row
list spreads over ranks with no exchange on the data path: each rank
serializes and scores its own shard, and the results are put back in row
order afterwards.  Shards are balanced by serialized token count, longest row
first onto the least-loaded shard, since a forward pass costs in proportion to
its tokens (and more for long rows under global attention).
"""
from __future__ import annotations

import heapq

import numpy as np


def shard_rows(lengths, n_shards: int):
    """Row indices per shard, balanced by token count.

    `lengths`: serialized tokens per row (e.g. the `length` field of
    `jd_rows_encoding_info`).  Rows go longest first to the shard with the fewest
    tokens so far (ties: lower shard index); each shard's indices come back in
    ascending order.  No shard exceeds the mean load by more than the longest row.
    """
    if n_shards < 1:
        raise ValueError("n_shards must be >= 1")
    lengths = np.asarray(lengths, dtype=np.int64)
    order = np.argsort(-lengths, kind="stable")
    heap = [(0, s) for s in range(n_shards)]
    parts = [[] for _ in range(n_shards)]
    for i in order:
        load, s = heapq.heappop(heap)
        parts[s].append(int(i))
        heapq.heappush(heap, (load + int(lengths[i]), s))
    return [sorted(p) for p in parts]


def merge_shards(parts, results, n_rows: int, n_options):
    """Put per-shard results back in row order.

    `parts`: the row indices of each shard (from `shard_rows`); `results`: per
    shard, a dict of arrays in that shard's row order: per-row arrays (choice,
    score, noul, max_p) of the shard's length and per-option arrays (logits,
    probs) of its total option count; `n_options`: options per row of the
    whole list.  Returns the same keys over all rows.
    """
    n_options = np.asarray(n_options, dtype=np.int64)
    off = np.concatenate([[0], np.cumsum(n_options)])
    out = {}
    for idx, res in zip(parts, results):
        if not idx:
            continue
        idx = np.asarray(idx, dtype=np.int64)
        k = n_options[idx]
        opt_idx = np.concatenate([np.arange(off[i], off[i] + n) for i, n in zip(idx, k)])
        for key, val in res.items():
            val = np.asarray(val)
            if len(val) == len(idx):
                dst = out.setdefault(key, np.zeros(n_rows, val.dtype))
                dst[idx] = val
            elif len(val) == len(opt_idx):
                dst = out.setdefault(key, np.zeros(int(off[-1]), val.dtype))
                dst[opt_idx] = val
            else:
                raise ValueError(f"{key}: {len(val)} values for {len(idx)} rows / {len(opt_idx)} options")
    return out
