"""Seeded weights and synthetic request rows for the Julia-1 decision model.

Weights: the tensors of the architecture described on "Julia-1: one score per
mask token" (§ "The decision head": an mmBERT-small / ModernBERT encoder of 22
layers, width 384, 6 heads, then a 3x384 type table, two pre-norm transformer
layers with feed-forward 1536 and a LayerNorm -> Linear(384,384) -> GELU ->
Linear(384,1) scorer).  Every non-norm tensor (weights and biases) is drawn
N(0, 0.02); norm gains are 1 and norm biases 0.  One numpy PCG64 stream (seed
0) fills the tensors in the fixed order of `weight_specs()`.

File format (".jdw", little endian):
    8 bytes   magic b"JDWGT001"
    u32       number of tensors n
    n records of 96 bytes: name (64 bytes, NUL padded ASCII), u32 ndim,
              u32 shape[4] (unused dims 1), u64 byte offset of the tensor
              within the data section
    zero padding to a multiple of 256 bytes, then the data section:
    every tensor in float32, C order, each starting on a 256-byte boundary.

Rows: pre-tokenized requests whose ids are uniform in [10, 256000) (ids 0..9
are reserved for special tokens).  The five workload recipes are stated on
each function.
"""
from __future__ import annotations

import os
import struct
from dataclasses import dataclass, field
from pathlib import Path

import numpy as np

# Architecture constants (mmBERT-small encoder + Julia-1 head).
ARCH = dict(
    vocab=256000,
    d=384,
    n_heads=6,
    head_dim=64,
    n_layers=22,
    ffn=1152,          # GEGLU half width: Wi maps 384 -> 2*1152
    head_ffn=1536,     # feed-forward width of the two head layers
    n_head_layers=2,
    n_types=3,         # 0 = choice, 1 = score, 2 = noul
    global_every=3,    # layer l is global iff l % 3 == 0
    window=64,         # local layers see keys with |i - j| <= 64
    theta_global=160000.0,
    theta_local=10000.0,
    eps=1e-5,
)

# Special token ids (any id below 10 is free with random weights).
SPECIAL = dict(pad=0, eos=1, bos=2, mask=4)

ID_LO, ID_HI = 10, ARCH["vocab"]
MAGIC = b"JDWGT001"
REC = struct.Struct("<64sI4IQ")  # 64 + 4 + 16 + 8 = 92 -> padded to 96 below
REC_SIZE = 96
ALIGN = 256


def weight_specs():
    """Ordered (name, shape, kind) list; kind is 'normal', 'ones' or 'zeros'."""
    a = ARCH
    d, f, hf = a["d"], a["ffn"], a["head_ffn"]
    s = [("embed.E", (a["vocab"], d), "normal"), ("embed.norm.g", (d,), "ones")]
    for l in range(a["n_layers"]):
        p = f"enc.{l}."
        if l != 0:  # layer 0 has no pre-attention norm (the embedding norm precedes it)
            s.append((p + "attn_norm.g", (d,), "ones"))
        s += [
            (p + "Wqkv", (3 * d, d), "normal"),
            (p + "Wo", (d, d), "normal"),
            (p + "mlp_norm.g", (d,), "ones"),
            (p + "Wi", (2 * f, d), "normal"),
            (p + "Wo2", (d, f), "normal"),
        ]
    s.append(("enc.final_norm.g", (d,), "ones"))
    s.append(("head.type_table", (a["n_types"], d), "normal"))
    for i in range(a["n_head_layers"]):
        p = f"head.{i}."
        s += [
            (p + "norm1.g", (d,), "ones"), (p + "norm1.b", (d,), "zeros"),
            (p + "in_proj.W", (3 * d, d), "normal"), (p + "in_proj.b", (3 * d,), "normal"),
            (p + "out_proj.W", (d, d), "normal"), (p + "out_proj.b", (d,), "normal"),
            (p + "norm2.g", (d,), "ones"), (p + "norm2.b", (d,), "zeros"),
            (p + "linear1.W", (hf, d), "normal"), (p + "linear1.b", (hf,), "normal"),
            (p + "linear2.W", (d, hf), "normal"), (p + "linear2.b", (d,), "normal"),
        ]
    s += [
        ("scorer.norm.g", (d,), "ones"), ("scorer.norm.b", (d,), "zeros"),
        ("scorer.linear1.W", (d, d), "normal"), ("scorer.linear1.b", (d,), "normal"),
        ("scorer.linear2.W", (1, d), "normal"), ("scorer.linear2.b", (1,), "normal"),
        # single-linear scorer variant (LayerNorm -> Linear(384 -> 1)); shares scorer.norm
        ("scorer_lin.W", (1, d), "normal"), ("scorer_lin.b", (1,), "normal"),
    ]
    return s


def _cache_dir() -> Path:
    p = Path(os.environ.get("JD_CACHE_DIR", Path(__file__).resolve().parent.parent / ".cache"))
    p.mkdir(parents=True, exist_ok=True)
    return p


def weights_path(seed: int = 0, std: float = 0.02, tag: str = "") -> Path:
    """Path of the seeded weights file, generating it on first use."""
    name = f"weights_seed{seed}{tag}.jdw"
    path = _cache_dir() / name
    if not path.exists():
        write_weights(path, seed=seed, std=std)
    return path


def write_weights(path, seed: int = 0, std: float = 0.02, overrides=None):
    """Draw every tensor from one PCG64 stream in spec order and write a .jdw file.

    `overrides` maps tensor name -> callable(array) -> array applied after the
    draw (used by tests that scale a tensor); it does not change the stream.
    """
    specs = weight_specs()
    rng = np.random.Generator(np.random.PCG64(seed))
    header_len = 8 + 4 + REC_SIZE * len(specs)
    data_start = (header_len + ALIGN - 1) // ALIGN * ALIGN
    offsets, off = [], 0
    for _, shape, _ in specs:
        offsets.append(off)
        nbytes = int(np.prod(shape)) * 4
        off += (nbytes + ALIGN - 1) // ALIGN * ALIGN
    tmp = Path(str(path) + ".tmp")
    with open(tmp, "wb") as fh:
        fh.write(MAGIC)
        fh.write(struct.pack("<I", len(specs)))
        for (name, shape, _), o in zip(specs, offsets):
            dims = list(shape) + [1] * (4 - len(shape))
            rec = REC.pack(name.encode().ljust(64, b"\0"), len(shape), *dims, o)
            fh.write(rec.ljust(REC_SIZE, b"\0"))
        fh.write(b"\0" * (data_start - header_len))
        for (name, shape, kind), o in zip(specs, offsets):
            n = int(np.prod(shape))
            if kind == "normal":
                arr = rng.standard_normal(n, dtype=np.float32) * np.float32(std)
            elif kind == "ones":
                arr = np.ones(n, np.float32)
            else:
                arr = np.zeros(n, np.float32)
            if overrides and name in overrides:
                arr = np.ascontiguousarray(overrides[name](arr.reshape(shape)), np.float32).reshape(-1)
            assert fh.tell() == data_start + o
            fh.write(arr.astype("<f4").tobytes())
            pad = (-(n * 4)) % ALIGN
            fh.write(b"\0" * pad)
    os.replace(tmp, path)
    return Path(path)


def read_weight_index(path):
    """Return {name: (shape, absolute byte offset)} for a .jdw file."""
    with open(path, "rb") as fh:
        if fh.read(8) != MAGIC:
            raise ValueError(f"{path}: not a .jdw weights file")
        (n,) = struct.unpack("<I", fh.read(4))
        recs = [fh.read(REC_SIZE) for _ in range(n)]
    header_len = 8 + 4 + REC_SIZE * n
    data_start = (header_len + ALIGN - 1) // ALIGN * ALIGN
    out = {}
    for r in recs:
        name, ndim, s0, s1, s2, s3, o = REC.unpack(r[: REC.size])
        shape = (s0, s1, s2, s3)[:ndim]
        out[name.rstrip(b"\0").decode()] = (shape, data_start + o)
    return out


# --------------------------------------------------------------------------- rows


@dataclass
class Row:
    """One pre-tokenized decision request: state, question, 2..20 options, type."""

    state: np.ndarray
    question: np.ndarray
    options: list = field(default_factory=list)
    qtype: int = 0  # 0 choice, 1 score, 2 noul


@dataclass
class RouterRequest:
    """A choice question over more candidates than one call takes (router input)."""

    state: np.ndarray
    question: np.ndarray
    labels: list


def _ids(rng, n):
    return rng.integers(ID_LO, ID_HI, size=int(n), dtype=np.int64).astype(np.int32)


def worked_example_rows():
    """Token-count skeleton of the card's routing example.

    "Julia-1: one score per mask token", § "From a state to one decision": a
    question of 10 tokens ("choice question: Which team should handle this
    request?"), three options of 4, 3 and 4 tokens and a 9-token state give
    marker positions 12, 17, 21 in a 37-token sequence.  Ids are placeholders.
    """
    rng = np.random.Generator(np.random.PCG64(7))
    return [Row(state=_ids(rng, 9), question=_ids(rng, 10),
                options=[_ids(rng, 4), _ids(rng, 3), _ids(rng, 4)], qtype=0)]


def rows_config0(seed: int = 100):
    """One choice row: 12 question ids, 3 options of 4 ids, a 16-id state (47 tokens)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    q = _ids(rng, 12)
    opts = [_ids(rng, 4) for _ in range(3)]
    st = _ids(rng, 16)
    return [Row(state=st, question=q, options=opts, qtype=0)]


def rows_config1(seed: int = 101):
    """Latency request: 3 questions (choice/4, score/3, noul/2) on one 200-id state.

    Options have 3..20 ids, questions 8..24 ids.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    st = _ids(rng, 200)
    rows = []
    for qtype, k in ((0, 4), (1, 3), (2, 2)):
        q = _ids(rng, rng.integers(8, 25))
        opts = [_ids(rng, rng.integers(3, 21)) for _ in range(k)]
        rows.append(Row(state=st, question=q, options=opts, qtype=qtype))
    return rows


def rows_config2(n_rows: int, seed: int = 102, head_budget: int = 512):
    """Batched throughput rows.

    Per row: total length L ~ U[64, 1024]; type uniform over choice/score/noul;
    K ~ U{2..20} (noul rows take K = 2); option lengths ~ U{1..48}; question
    length ~ U{8..24}.  A draw is redrawn (same stream) while its head part
    (bos + question + eos + K markers + option ids + eos) exceeds the head
    budget or leaves fewer than one state id before the final eos.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = []
    while len(rows) < n_rows:
        L = int(rng.integers(64, 1025))
        qtype = int(rng.integers(0, 3))
        k = 2 if qtype == 2 else int(rng.integers(2, 21))
        olens = rng.integers(1, 49, size=k)
        nq = int(rng.integers(8, 25))
        head = 3 + nq + k + int(olens.sum())
        n_state = L - head - 1
        if head > head_budget or n_state < 1:
            continue
        q = _ids(rng, nq)
        opts = [_ids(rng, n) for n in olens]
        st = _ids(rng, n_state)
        rows.append(Row(state=st, question=q, options=opts, qtype=qtype))
    return rows


def rows_config3(n_rows: int = 16, seed: int = 103, state_ids: int = 8192):
    """Long-context rows: 20 options of 48 ids, question ~U{8..24}, a state longer
    than the 8192-token limit, types choice/score.  Encoded non-strict with a
    256-token head budget, the options are capped and the state clipped so every
    row is exactly 8192 tokens.
    """
    rng = np.random.Generator(np.random.PCG64(seed))
    rows = []
    for _ in range(n_rows):
        qtype = int(rng.integers(0, 2))
        q = _ids(rng, rng.integers(8, 25))
        opts = [_ids(rng, 48) for _ in range(20)]
        st = _ids(rng, state_ids)
        rows.append(Row(state=st, question=q, options=opts, qtype=qtype))
    return rows


def requests_config4(n_requests: int = 512, seed: int = 104, n_labels: int = 72):
    """Router workload: per request a 256-id state, a question ~U{8..24} ids and
    72 candidate labels of 3..12 ids each (choice)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    reqs = []
    for _ in range(n_requests):
        st = _ids(rng, 256)
        q = _ids(rng, rng.integers(8, 25))
        labels = [_ids(rng, rng.integers(3, 13)) for _ in range(n_labels)]
        reqs.append(RouterRequest(state=st, question=q, labels=labels))
    return reqs
