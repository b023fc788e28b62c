"""The algorithmic bytes and FLOPs that `bench.py` divides by measured time.

Each roofline fraction the bench reports is (algorithmic bytes or FLOPs per
launch) / (measured duration) / (peak), so the accounting is pinned here: the
per-token bytes against the compulsory traffic of each step (BF16 activations
of width 384 = 768 B, the FP32 residual = 1,536 B, the QKV output 2,304 B, the
GEGLU output 2,304 B, the head FFN output 3,072 B), the GEMM FLOPs against
2 * K * N per token, and the attention FLOPs against a brute-force count of the
(query, key) pairs each layer kind lets through (4 * 64 FLOPs per pair and head:
q.k and p.v).
"""
import numpy as np
import pytest

import bench

D, FF, HFF, H, DH = 384, 1152, 1536, 6, 64
LENS = [1, 2, 63, 64, 65, 129, 130, 257, 1000]


@pytest.mark.parametrize("name,bytes_per_token,k,n", [
    ("embed_ln", 4 + 1536 + 1536 + 768, None, None),
    ("gemm_qkv_rope", 768 + 2304, D, 3 * D),
    ("gemm_wo_res_ln", 768 + 1536 + 1536 + 768, D, D),
    ("gemm_wi_geglu", 768 + 2304, D, 2 * FF),
    ("gemm_wo2_res_ln", 2304 + 1536 + 1536 + 768, FF, D),
    ("head0_gemm_ffn1", 768 + 3072, D, HFF),
    ("head0_gemm_ffn2", 3072 + 1536 + 1536 + 768, HFF, D),
    ("head1_gemm_kv", 768 + 1536, D, 2 * D),
])
def test_per_token_costs(name, bytes_per_token, k, n):
    T = sum(LENS)
    b, f = bench.algorithmic_cost(name, LENS, 0)
    assert b == T * bytes_per_token
    if k is not None:
        assert f == T * 2 * k * n


def _pairs(lens, window):
    total = 0
    for L in lens:
        for i in range(L):
            for j in range(L):
                if window is None or abs(i - j) <= window:
                    total += 1
    return total


def test_attention_flops_count_visible_pairs():
    T = sum(LENS)
    for name, window in (("attn_global", None), ("head0_attn", None), ("attn_local", 64)):
        b, f = bench.algorithmic_cost(name, LENS, 0)
        assert b == T * (3 * 768 + 768)
        assert f == 4 * DH * H * _pairs(LENS, window), name


def test_marker_attention_cost():
    lens, kper = [100, 300], [3, 20]
    M = sum(kper)
    b, f = bench.algorithmic_cost("head1_marker_attn", lens, M, kper)
    # K and V of every token read once, each marker's q read and o written (BF16)
    assert b == sum(lens) * 2 * 768 + M * 2 * 768
    # every marker attends to every key of its row
    assert f == 4 * DH * H * sum(k * L for k, L in zip(kper, lens))


def test_embedding_reads_count_distinct_ids():
    """The gather's compulsory reads are one FP32 embedding row per distinct id (a
    repeated id is served from L2); its writes are one FP32 and one BF16 row per token."""
    T = sum(LENS)
    b, _ = bench.algorithmic_cost("embed_ln", LENS, 0, n_unique_ids=100)
    assert b == T * 4 + 100 * 1536 + T * (1536 + 768)
    b_all, _ = bench.algorithmic_cost("embed_ln", LENS, 0, n_unique_ids=T)
    assert b_all == T * (4 + 1536 + 1536 + 768)
