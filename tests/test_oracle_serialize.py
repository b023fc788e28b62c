"""Pins of the oracle serialiser against the pages' layout, limits and error rules."""
import os

import numpy as np
import pytest

from oracle import (EncodeOptions, EncodingError, serialize_row, ERR_OPTION_COUNT, ERR_OVERFLOW,
                    ERR_TOKEN_RANGE, ERR_INVALID_ARG, TRUNC_OPTION_48, TRUNC_OPTION_CAP,
                    TRUNC_QUESTION, TRUNC_STATE)
from workloads import Row, rows_config0, worked_example_rows, rows_config3, rows_config2

GOLD = os.path.join(os.path.dirname(__file__), "golden")
BOS, EOS, MASK = 2, 1, 4


def _golden(name):
    out = {}
    for line in open(os.path.join(GOLD, name)):
        if line.startswith("#") or not line.strip():
            continue
        k, *v = line.split()
        out[k] = [int(x) for x in v]
    return out


def ids(n, start=100):
    return np.arange(start, start + n, dtype=np.int32)


def row(nq, olens, ns, qtype=0):
    return Row(state=ids(ns, 5000), question=ids(nq, 100), options=[ids(n, 1000 + 100 * i) for i, n in enumerate(olens)], qtype=qtype)


def test_worked_example_positions():
    g = _golden("worked_example_layout.txt")
    (r,) = worked_example_rows()
    assert len(r.question) == g["question_len"][0]
    assert [len(o) for o in r.options] == g["option_lens"]
    assert len(r.state) == g["state_len"][0]
    e = serialize_row(r, EncodeOptions(max_length=1024, head_budget=512))
    assert list(e.mask_pos) == g["mask_positions"]
    assert len(e.ids) == g["total_tokens"][0]
    assert e.trunc == 0


def test_layout_order():
    r = row(3, [2, 1], 4)
    e = serialize_row(r, EncodeOptions())
    expect = [BOS, 100, 101, 102, EOS, MASK, 1000, 1001, MASK, 1100, EOS, 5000, 5001, 5002, 5003, EOS]
    assert e.ids.tolist() == expect
    assert e.mask_pos.tolist() == [5, 8]
    assert e.head_len == 11


def test_config0_layout():
    (r,) = rows_config0()
    e = serialize_row(r, EncodeOptions(max_length=8192, head_budget=256))
    # 1 + 12 + 1 + 3 * (1 + 4) + 1 + 16 + 1 = 47 tokens; markers after bos+question+eos
    assert len(e.ids) == 47
    assert e.mask_pos.tolist() == [14, 19, 24]


@pytest.mark.parametrize("k", [0, 1, 21, 25])
def test_option_count_errors(k):
    r = row(4, [2] * k, 5)
    for strict in (True, False):
        with pytest.raises(EncodingError) as ei:
            serialize_row(r, EncodeOptions(strict=strict))
        assert ei.value.code == ERR_OPTION_COUNT


def test_option_count_bounds_ok():
    for k in (2, 20):
        serialize_row(row(4, [1] * k, 5), EncodeOptions(head_budget=512))


def test_noul_needs_two():
    with pytest.raises(EncodingError) as ei:
        serialize_row(row(4, [2, 2, 2], 5, qtype=2), EncodeOptions(strict=False))
    assert ei.value.code == ERR_OPTION_COUNT
    serialize_row(row(4, [2, 2], 5, qtype=2), EncodeOptions())


def test_token_range():
    r = row(4, [2, 2], 5)
    r.state = r.state.copy()
    r.state[2] = 256000
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions(strict=False))
    assert ei.value.code == ERR_TOKEN_RANGE
    r.state[2] = -1
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions())
    assert ei.value.code == ERR_TOKEN_RANGE


def test_invalid_opts():
    with pytest.raises(EncodingError) as ei:
        serialize_row(row(2, [1, 1], 1), EncodeOptions(max_length=8193))
    assert ei.value.code == ERR_INVALID_ARG


def test_strict_option_49():
    r = row(4, [49, 2], 5)
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions(strict=True, head_budget=512))
    assert ei.value.code == ERR_OVERFLOW
    serialize_row(row(4, [48, 2], 5), EncodeOptions(strict=True, head_budget=512))


def test_strict_head_budget_edge():
    # head = 3 + nq + K + sum = 3 + 10 + 2 + 3 + 4 = 22
    r = row(10, [3, 4], 5)
    e = serialize_row(r, EncodeOptions(strict=True, head_budget=22))
    assert e.head_len == 22
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions(strict=True, head_budget=21))
    assert ei.value.code == ERR_OVERFLOW


def test_strict_total_edge():
    r = row(10, [3, 4], 5)  # total = 22 + 5 + 1 = 28
    assert len(serialize_row(r, EncodeOptions(max_length=28)).ids) == 28
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions(max_length=27))
    assert ei.value.code == ERR_OVERFLOW


def test_nonstrict_clip_48():
    r = row(4, [60, 2], 5)
    e = serialize_row(r, EncodeOptions(strict=False, head_budget=512))
    assert e.trunc == TRUNC_OPTION_48
    assert e.mask_pos.tolist() == [6, 6 + 49]
    assert e.ids[7:7 + 48].tolist() == list(range(1000, 1048))


def test_nonstrict_cap():
    # fixed = 3 + 5 + 3 = 11; lens 10, 2, 7; budget 25 -> sum(min(len, c)) <= 14
    # c=5: 5+2+5 = 12 ok; c=6: 6+2+6 = 14 ok; c=7: 7+2+7 = 16 no -> c = 6
    r = row(5, [10, 2, 7], 3)
    e = serialize_row(r, EncodeOptions(strict=False, head_budget=25))
    assert e.trunc == TRUNC_OPTION_CAP
    assert e.head_len == 25
    assert e.mask_pos.tolist() == [7, 14, 17]
    assert e.ids[18:24].tolist() == list(range(1200, 1206))


def test_nonstrict_question_clip():
    # fixed without question: 3 + K = 5; options capped to 1 -> 2; budget 9 -> 2 question ids
    r = row(10, [4, 4], 3)
    e = serialize_row(r, EncodeOptions(strict=False, head_budget=9))
    assert e.trunc == TRUNC_OPTION_CAP | TRUNC_QUESTION
    assert e.ids[:4].tolist() == [BOS, 100, 101, EOS]
    assert e.head_len == 9


def test_nonstrict_impossible():
    r = row(10, [4, 4], 3)
    with pytest.raises(EncodingError) as ei:
        serialize_row(r, EncodeOptions(strict=False, head_budget=6))
    assert ei.value.code == ERR_OVERFLOW


def test_nonstrict_state_clip():
    r = row(4, [2, 2], 100)
    e = serialize_row(r, EncodeOptions(strict=False, max_length=40))
    assert e.trunc == TRUNC_STATE
    assert len(e.ids) == 40
    assert e.ids[-1] == EOS
    assert e.ids[e.head_len:-1].tolist() == list(range(5000, 5000 + 40 - e.head_len - 1))


def test_empty_state_and_options():
    r = row(0, [0, 0], 0)
    e = serialize_row(r, EncodeOptions())
    assert e.ids.tolist() == [BOS, EOS, MASK, MASK, EOS, EOS]
    assert e.mask_pos.tolist() == [2, 3]


def test_config3_fills_8192():
    for r in rows_config3(4):
        e = serialize_row(r, EncodeOptions(max_length=8192, head_budget=256, strict=False))
        assert len(e.ids) == 8192
        assert e.head_len <= 256 and e.trunc & TRUNC_OPTION_CAP and e.trunc & TRUNC_STATE
        assert len(e.mask_pos) == 20


def test_config2_rows_valid_strict():
    rs = rows_config2(64)
    for r in rs:
        e = serialize_row(r, EncodeOptions(max_length=1024, head_budget=512, strict=True))
        assert 64 <= len(e.ids) <= 1024 and e.trunc == 0
        assert (r.qtype == 2) == (len(r.options) == 2) or r.qtype != 2
