"""Marker serialisation with the documented budgets (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows "Julia-1: one score per mask token", § "From a state to one decision":
the question comes first, each option follows its own <mask> marker, the state
comes last, and the sequence reads

    <bos> question <eos> (<mask> option_k)_k <eos> state <eos>

with 2 to 20 options, each at most 48 tokens, question plus options within a
head budget (256 by default, 512 in the card's example) and 8,192 tokens in
all; with strict encoding any overflow raises.  "Julia-1 MLX", § "API" adds
that the encoder reports whether anything was truncated, and § "Three modes
through one head" fixes noul to exactly two options [false, true].

Readings where the page is silent (stated, not quoted):
  * the type prefix ("choice question:") is part of the caller's question ids;
  * the 48-token limit counts an option's ids without its marker;
  * "head" is every token before the state (bos, question, eos, markers,
    option ids, eos); total = head + state + final eos <= max_length;
  * always errors: option count outside [2, 20], noul with K != 2, an id
    outside [0, vocab); strict-only errors: an option over 48 ids, head over
    budget, total over max_length;
  * non-strict truncation: (1) clip every option to its first 48 ids; (2) if
    the head is still over budget, cap every option at the largest c >= 1
    that fits, and if even c = 1 does not fit, clip the question from its end
    (an error if nothing fits); (3) clip the state to its first
    max_length - head - 1 ids.
Parity: pinned by the card's worked example (markers 12, 17, 21 in 37 tokens)
and hand-built rows for every branch (tests/test_oracle_serialize.py).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

ERR_OK = 0
ERR_INVALID_ARG = 1
ERR_OPTION_COUNT = 2
ERR_OVERFLOW = 3
ERR_TOKEN_RANGE = 4

TRUNC_OPTION_48 = 1     # an option was clipped to 48 ids
TRUNC_OPTION_CAP = 2    # options were capped to fit the head budget
TRUNC_QUESTION = 4      # the question was clipped from its end
TRUNC_STATE = 8         # the state was clipped to fit max_length

MAX_OPTION_IDS = 48
MIN_OPTIONS, MAX_OPTIONS = 2, 20
MAX_LENGTH_LIMIT = 8192


class EncodingError(ValueError):
    def __init__(self, code, msg):
        super().__init__(msg)
        self.code = code


@dataclass
class EncodeOptions:
    max_length: int = 8192
    head_budget: int = 256
    strict: bool = True
    bos: int = 2
    eos: int = 1
    mask: int = 4
    vocab: int = 256000


@dataclass
class Encoded:
    ids: np.ndarray        # int32 [L]
    mask_pos: np.ndarray   # int32 [K], positions within the row
    qtype: int
    trunc: int             # TRUNC_* bit set
    head_len: int


def _check_ids(arr, vocab, what):
    a = np.asarray(arr, dtype=np.int64)
    if a.size and (a.min() < 0 or a.max() >= vocab):
        raise EncodingError(ERR_TOKEN_RANGE, f"{what}: token id outside [0, {vocab})")


def serialize_row(row, opt: EncodeOptions) -> Encoded:
    if not (1 <= opt.max_length <= MAX_LENGTH_LIMIT) or opt.head_budget < 1:
        raise EncodingError(ERR_INVALID_ARG, "max_length must be in [1, 8192] and head_budget >= 1")
    _check_ids([opt.bos, opt.eos, opt.mask], opt.vocab, "bos/eos/mask")
    if row.qtype not in (0, 1, 2):
        raise EncodingError(ERR_INVALID_ARG, "type must be choice (0), score (1) or noul (2)")
    k = len(row.options)
    if not (MIN_OPTIONS <= k <= MAX_OPTIONS):
        raise EncodingError(ERR_OPTION_COUNT, f"{k} options: a question takes 2 to 20")
    if row.qtype == 2 and k != 2:
        raise EncodingError(ERR_OPTION_COUNT, "a noul question takes exactly two options [false, true]")
    _check_ids(row.question, opt.vocab, "question")
    for i, o in enumerate(row.options):
        _check_ids(o, opt.vocab, f"option {i}")
    _check_ids(row.state, opt.vocab, "state")

    q = list(np.asarray(row.question, dtype=np.int64))
    opts = [list(np.asarray(o, dtype=np.int64)) for o in row.options]
    st = list(np.asarray(row.state, dtype=np.int64))
    trunc = 0

    if opt.strict:
        if any(len(o) > MAX_OPTION_IDS for o in opts):
            raise EncodingError(ERR_OVERFLOW, "an option is longer than 48 tokens")
        head = 3 + len(q) + k + sum(len(o) for o in opts)
        if head > opt.head_budget:
            raise EncodingError(ERR_OVERFLOW, f"question plus options take {head} tokens, over the head budget")
        if head + len(st) + 1 > opt.max_length:
            raise EncodingError(ERR_OVERFLOW, "sequence longer than max_length")
    else:
        # (1) clip each option to 48 ids
        if any(len(o) > MAX_OPTION_IDS for o in opts):
            trunc |= TRUNC_OPTION_48
            opts = [o[:MAX_OPTION_IDS] for o in opts]
        fixed = 3 + len(q) + k
        lens = [len(o) for o in opts]
        if fixed + sum(lens) > opt.head_budget:
            # (2) largest common cap c >= 1 that fits the budget
            cap = None
            for c in range(max(lens), 0, -1):
                if fixed + sum(min(n, c) for n in lens) <= opt.head_budget:
                    cap = c
                    break
            if cap is not None:
                opts = [o[:cap] for o in opts]
                trunc |= TRUNC_OPTION_CAP
            else:
                if any(n > 1 for n in lens):
                    trunc |= TRUNC_OPTION_CAP
                opts = [o[:1] for o in opts]
                room = opt.head_budget - (3 + k + sum(len(o) for o in opts))
                if room < 0:
                    raise EncodingError(ERR_OVERFLOW, "head budget too small for the markers alone")
                q = q[:room]
                trunc |= TRUNC_QUESTION
        head = 3 + len(q) + k + sum(len(o) for o in opts)
        room_state = opt.max_length - head - 1
        if room_state < 0:
            raise EncodingError(ERR_OVERFLOW, "max_length too small for the head")
        if len(st) > room_state:
            st = st[:room_state]
            trunc |= TRUNC_STATE

    seq = [opt.bos] + q + [opt.eos]
    marks = []
    for o in opts:
        marks.append(len(seq))
        seq.append(opt.mask)
        seq.extend(o)
    seq.append(opt.eos)
    head_len = len(seq)
    seq.extend(st)
    seq.append(opt.eos)
    return Encoded(ids=np.asarray(seq, np.int32), mask_pos=np.asarray(marks, np.int32),
                   qtype=int(row.qtype), trunc=trunc, head_len=head_len)


def serialize_rows(rows, opt: EncodeOptions):
    return [serialize_row(r, opt) for r in rows]
