"""Julia-1 forward pass, one row at a time, in float64 NumPy (oracle).

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

What it computes, in the pages' order ("Julia-1: one score per mask token",
§ "The decision head"):
  encoder   mmBERT-small with ModernBERT's block: 22 layers, width 384, 6
            heads; every third layer attends globally, the rest within a
            128-token sliding window ("Julia-1 MLX", § "Performance": +-64
            tokens); GEGLU feed-forward ("julia1 -- Rust runtime", § "Why it
            is faster"); RoPE with theta 160000 (global) / 10000 (local).
  step 1    add the type-table row (0 choice, 1 score, 2 noul) to every position
  step 2    two pre-norm transformer layers (6 heads, feed-forward 1536) over
            the whole row; they are PyTorch TransformerEncoderLayers ("Julia-1
            MLX", § "Fine-tuning and export"): biased projections, biased
            LayerNorms, ReLU feed-forward by default
  step 3    gather the hidden state at each <mask> position
  step 4    LayerNorm -> Linear(384,384) -> GELU -> Linear(384,1) per option

Readings where the pages are silent (each a flag where the alternative is
plausible):
  * global layers are l % 3 == 0 (8 global, 14 local); key j is visible to
    query i in a local layer iff |i - j| <= 64;
  * RoPE pairs dim i with i + 32 inside each 64-dim head ("rotate half"),
    inv_freq_i = theta^(-2i/64), position = index within the row;
  * layer 0 has no pre-attention norm (the embedding norm precedes it);
    encoder norms have a gain and no bias; head and scorer norms have both;
    eps = 1e-5; a final encoder norm precedes the type-row add;
  * GEGLU: the first 1152 outputs of Wi feed GELU, the last 1152 are the gate;
    GELU is the exact erf form everywhere;
  * attention scale 1/sqrt(64); head attention has no positional encoding;
  * head feed-forward activation ReLU (flag "gelu"); scorer "mlp" (flag
    "linear": LayerNorm -> Linear(384 -> 1)).
Arithmetic is float64 end to end; weights are the float32 values of the file.
Parity: each function is pinned in tests/test_oracle_model.py by closed forms,
brute force on tiny inputs and invariants, and the whole chain (encoder ->
final norm -> type row -> head layer 0 -> head layer 1 -> gather -> scorer) by
a closed form on tiny structured weights.  Logits of the trained model have
no printed value to pin against (no checkpoint offline).
"""
from __future__ import annotations

import math
import struct
from dataclasses import dataclass

import numpy as np
from scipy.special import erf

F = np.float64


# ---------------------------------------------------------------- weight file


def _read_index(path):
    """Own reader of the .jdw container: {name: (shape, byte offset)}."""
    with open(path, "rb") as fh:
        magic = fh.read(8)
        if magic != b"JDWGT001":
            raise ValueError("not a .jdw weights file")
        (n,) = struct.unpack("<I", fh.read(4))
        body = fh.read(96 * n)
    header = 12 + 96 * n
    data0 = (header + 255) // 256 * 256
    idx = {}
    for i in range(n):
        rec = body[96 * i: 96 * i + 92]
        name = rec[:64].rstrip(b"\0").decode()
        ndim, d0, d1, d2, d3, off = struct.unpack("<I4IQ", rec[64:92])
        idx[name] = ((d0, d1, d2, d3)[:ndim], data0 + off)
    return idx


class Weights:
    """Lazy float64 view of a .jdw file (the embedding table stays float32 on disk)."""

    def __init__(self, path):
        self.path = str(path)
        self.index = _read_index(path)
        self._mm = np.memmap(self.path, dtype=np.uint8, mode="r")
        self._cache = {}

    def raw(self, name):
        shape, off = self.index[name]
        n = int(np.prod(shape))
        return np.frombuffer(self._mm, dtype="<f4", count=n, offset=off).reshape(shape)

    def __getitem__(self, name):
        if name not in self._cache:
            self._cache[name] = self.raw(name).astype(F)
        return self._cache[name]

    def embed_rows(self, ids):
        return self.raw("embed.E")[np.asarray(ids, dtype=np.int64)].astype(F)


# ---------------------------------------------------------------- components


def layer_norm(x, g, b=None, eps=1e-5):
    """LayerNorm over the last axis: (x - mean) / sqrt(biased var + eps) * g (+ b)."""
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    y = (x - mu) / np.sqrt(var + eps) * g
    return y if b is None else y + b


def gelu(x):
    """Exact GELU, x * Phi(x) with Phi the standard normal CDF."""
    return 0.5 * x * (1.0 + erf(x / math.sqrt(2.0)))


def rope(x, theta):
    """Rotary embedding of x [L, H, dh]; pairs (i, i + dh/2), positions 0..L-1."""
    L, _, dh = x.shape
    half = dh // 2
    inv_freq = theta ** (-np.arange(0, dh, 2, dtype=F) / dh)          # [half]
    ang = np.arange(L, dtype=F)[:, None] * inv_freq[None, :]          # [L, half]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half], x[..., half:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def softmax_rows(s):
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def attention(q, k, v, window=None):
    """Bidirectional multi-head attention inside one row.

    q, k, v: [L, H, dh].  Scores q.k / sqrt(dh); with `window` = w the key j is
    visible to query i iff |i - j| <= w (a dense mask, as the plain definition).
    """
    L, H, dh = q.shape
    out = np.empty_like(q)
    if window is not None:
        i = np.arange(L)
        hidden = np.abs(i[:, None] - i[None, :]) > window
    for h in range(H):
        s = (q[:, h, :] @ k[:, h, :].T) / math.sqrt(dh)
        if window is not None:
            s = np.where(hidden, -np.inf, s)
        out[:, h, :] = softmax_rows(s) @ v[:, h, :]
    return out


@dataclass
class ModelOptions:
    scorer: str = "mlp"        # "mlp" | "linear"
    head_act: str = "relu"     # "relu" | "gelu"
    n_layers: int = 22
    n_heads: int = 6
    global_every: int = 3
    window: int = 64
    theta_global: float = 160000.0
    theta_local: float = 10000.0
    eps: float = 1e-5


def encoder_layer(x, W, l, mo: ModelOptions):
    """One ModernBERT block: x += Wo.attn(rope(Wqkv.norm(x))); x += Wo2.GEGLU(Wi.norm(x))."""
    L, d = x.shape
    H = mo.n_heads
    dh = d // H
    p = f"enc.{l}."
    h = x if l == 0 else layer_norm(x, W[p + "attn_norm.g"], eps=mo.eps)
    qkv = h @ W[p + "Wqkv"].T
    q, k, v = (qkv[:, i * d:(i + 1) * d].reshape(L, H, dh) for i in range(3))
    is_global = (l % mo.global_every) == 0
    theta = mo.theta_global if is_global else mo.theta_local
    q, k = rope(q, theta), rope(k, theta)
    o = attention(q, k, v, window=None if is_global else mo.window)
    x = x + o.reshape(L, d) @ W[p + "Wo"].T
    ug = layer_norm(x, W[p + "mlp_norm.g"], eps=mo.eps) @ W[p + "Wi"].T
    f = ug.shape[1] // 2
    y = gelu(ug[:, :f]) * ug[:, f:]
    return x + y @ W[p + "Wo2"].T


def head_layer(h, W, i, mo: ModelOptions):
    """Pre-norm TransformerEncoderLayer: h += MHA(LN1 h); h += W2 act(W1 LN2 h + b1) + b2."""
    L, d = h.shape
    H = mo.n_heads
    dh = d // H
    p = f"head.{i}."
    a = layer_norm(h, W[p + "norm1.g"], W[p + "norm1.b"], mo.eps)
    qkv = a @ W[p + "in_proj.W"].T + W[p + "in_proj.b"]
    q, k, v = (qkv[:, j * d:(j + 1) * d].reshape(L, H, dh) for j in range(3))
    o = attention(q, k, v)
    h = h + o.reshape(L, d) @ W[p + "out_proj.W"].T + W[p + "out_proj.b"]
    f = layer_norm(h, W[p + "norm2.g"], W[p + "norm2.b"], mo.eps)
    z = f @ W[p + "linear1.W"].T + W[p + "linear1.b"]
    z = np.maximum(z, 0.0) if mo.head_act == "relu" else gelu(z)
    return h + z @ W[p + "linear2.W"].T + W[p + "linear2.b"]


def scorer(hm, W, mo: ModelOptions):
    """Per-option logit from the marker states hm [K, d]."""
    n = layer_norm(hm, W["scorer.norm.g"], W["scorer.norm.b"], mo.eps)
    if mo.scorer == "linear":
        return (n @ W["scorer_lin.W"].T + W["scorer_lin.b"])[:, 0]
    z = gelu(n @ W["scorer.linear1.W"].T + W["scorer.linear1.b"])
    return (z @ W["scorer.linear2.W"].T + W["scorer.linear2.b"])[:, 0]


class OracleModel:
    """Forward pass of one serialised row at a time.

    `weights` is a .jdw path, or any mapping of tensor names to arrays that
    also has `embed_rows(ids)` (the tests build tiny structured ones)."""

    def __init__(self, weights, options: ModelOptions | None = None):
        self.W = weights if hasattr(weights, "embed_rows") else Weights(weights)
        self.mo = options or ModelOptions()

    def encode(self, ids):
        """Encoder output after the final norm, [L, d]."""
        W, mo = self.W, self.mo
        x = layer_norm(W.embed_rows(ids), W["embed.norm.g"], eps=mo.eps)
        for l in range(mo.n_layers):
            x = encoder_layer(x, W, l, mo)
        return layer_norm(x, W["enc.final_norm.g"], eps=mo.eps)

    def head(self, e, qtype):
        """"The decision head", steps 1-2: the type-table row added to every
        position of the encoder output e, then both head layers, [L, d]."""
        h = e + self.W["head.type_table"][qtype]
        for i in range(2):
            h = head_layer(h, self.W, i, self.mo)
        return h

    def hidden(self, ids, qtype):
        """State after the type-row add and both head layers, [L, d]."""
        return self.head(self.encode(ids), qtype)

    def forward_all(self, enc):
        """The whole pass for one serialised row (oracle.serialize.Encoded):
        encoder -> final norm -> steps 1-2 (head) -> step 3 (gather at the
        <mask> positions) -> step 4 (scorer).  Returns the encoder output
        (after the final norm), the marker states after both head layers,
        and the raw option logits."""
        e = self.encode(enc.ids)
        hm = self.head(e, enc.qtype)[np.asarray(enc.mask_pos, dtype=np.int64)]
        return dict(encoder_out=e, marker_state=hm, logits=scorer(hm, self.W, self.mo))

    def logits(self, enc):
        """Raw option logits for one serialised row (the same chain as forward_all)."""
        return self.forward_all(enc)["logits"]
