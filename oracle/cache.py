"""Layer-level semantics of the quantized cache: anchors, effective bits, decode.

Anchors ("Fourier Magnitude KV Cache Quantization" post 6: "Corrected semantics" -- every
layer is quantized and anchors only add protection; "Minimal recipe" -- fp16 anchors on layer 0
only, 48 tokens; "The winning recipe" -- the first decoded tokens stay high precision on
selected layers; a 64-token sliding window is also reported).  Every row is quantized; a row in
the anchor set is additionally kept as its original fp16 row, and attention reads that fp16 row
instead of the quantized one.  Rules, for layers in
the anchor layer set:
  first_n(n): tokens t < n
  window(w):  tokens t >= L - w, L = the sequence's stored length
  all:        every token of the layer

Per-layer formats ("E21W" "What I tested": a per-layer K/V bit allocation, 2 to 4 bits in groups
of 128, under a 3.2-bit average; "Result": 2-bit K in layers 2 and 7, 4-bit V in layers 1, 3
and 4, 3 bits elsewhere, 3.19 bits on average).  A Spec may give one Side per layer for K and for
V; layers are numbered from 0 (the same result calls layer 7 the last of the 8).

Anchor precision (post 6, "The winning recipe" item 4, the anchor-precision dial: fp16, int8
or int4 anchors; "Best results" rows "ternboth_a8" and "signboth_a8" use int8 anchors).  Reading
taken here: an int8 or int4 anchor row is the original fp16 row on the same signed absmax grid as
the int format (largest-magnitude element at -2^(b-1), first index on ties), in groups of 32
channels with one fp16 scale each, no pre-transform; attention reads its dequantized values.

Key mean subtraction (llama.cpp #21385, the later comment on a per-head shared key mean that
carries about half of the key energy: the running mean is subtracted before quantization and
restored after).  Reading taken here: the mean of one (layer, sequence, kv-head) is the running
mean of its keys at the end of the sequence's first append (normally the prefill), frozen for
the tokens that follow, so that every stored key row of the sequence shares it.  It is exact
before one rounding: mu = fp16(fp64(S) / n * 2^-24) with S the exact integer sum of the n fp16
keys times 2^24.  Rows are quantized as fp32(k - mu); dequantized rows get mu added back (the
attention logits of the sequence's quantized rows all shift by q . mu).  Anchored rows keep the
raw key.

Effective bits ("E21W" "Result" counts group scales in the totals, 3.5 b for 3-bit g32 and
4.5 b for 4-bit g32; "E22L" "What I tested" averages over K and V with scales included; post 6
"Corrected semantics" reports anchored configurations in effective bits): (code bits + 16 per
scale + 16 per zero point + 16 D per anchored row + 16 D per channel-scale vector) / values,
averaged over K and V.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import attention as A
from .quant import F64
from .quant import Side, bits_per_value, quantize_rows, to_original_f64


@dataclass
class Spec:
    n_layers: int
    batch: int
    n_kv: int
    n_q: int
    D: int
    k: Side
    v: Side
    anchor_layers: frozenset = field(default_factory=frozenset)
    anchor_rule: str = "none"  # none | first_n | window | all
    anchor_n: int = 0
    sm_scale: float | None = None
    layer_k: tuple = ()  # one Side per layer, or empty: k on every layer
    layer_v: tuple = ()
    anchor_bits: int = 16  # 16 (fp16 rows), 8 or 4 (signed absmax grid, groups of 32)
    head_k: tuple = ()  # per (layer, kv-head): n_layers tuples of n_kv Sides, or empty
    head_v: tuple = ()


def side_of(spec: Spec, layer: int, is_k: bool, head: int = 0) -> Side:
    ph = spec.head_k if is_k else spec.head_v
    if ph:
        return ph[layer][head]
    per = spec.layer_k if is_k else spec.layer_v
    return per[layer] if per else (spec.k if is_k else spec.v)


def anchored(spec: Spec, layer: int, tokens: np.ndarray, seq_len: int) -> np.ndarray:
    t = np.asarray(tokens)
    if spec.anchor_rule == "none" or layer not in spec.anchor_layers:
        return np.zeros(t.shape, dtype=bool)
    if spec.anchor_rule == "first_n":
        return t < spec.anchor_n
    if spec.anchor_rule == "window":
        return (t >= seq_len - spec.anchor_n) & (t < seq_len)
    if spec.anchor_rule == "all":
        return t < seq_len
    raise ValueError(spec.anchor_rule)


def anchor_side(spec: Spec) -> Side:
    return Side("int", spec.anchor_bits, group=32)


def anchor_rows(spec: Spec, X16: np.ndarray) -> dict:
    """The stored anchor form of fp16 rows X16 [n, D]: for int anchors the quantize_rows dict of
    the anchor grid, for fp16 anchors the rows themselves (as 'exact')."""
    X16 = np.asarray(X16, dtype=np.float16)
    if spec.anchor_bits == 16:
        return {"exact": X16.astype(F64)}
    return quantize_rows(X16, anchor_side(spec))


def key_mean(K16: np.ndarray) -> np.ndarray:
    """fp16 mean over the rows of K16 [n, D]: the exact sum rounded once (see the module text)."""
    k = np.asarray(K16, dtype=np.float16).astype(F64)
    S = np.round(k * 2.0 ** 24).astype(np.int64).sum(axis=0)  # fp16 values are multiples of 2^-24
    return ((S.astype(F64) / F64(k.shape[0])) * 2.0 ** -24).astype(np.float16)


def quantize_unit(spec: Spec, K16: np.ndarray, V16: np.ndarray, c16=None, layer: int = 0, first_rows=None,
                  head: int = 0):
    """Quantize one (layer, sequence, kv-head) unit: K16, V16 [T, D]; c16 [D] or None;
    first_rows: rows of the sequence's first append (the key mean's rows; default all)."""
    ks = side_of(spec, layer, True, head)
    mu = key_mean(K16[:first_rows or K16.shape[0]]) if ks.mean_sub else None
    kq = quantize_rows(K16, ks, None if c16 is None else np.broadcast_to(c16, K16.shape),
                       None if mu is None else np.broadcast_to(mu, K16.shape))
    kq["mu"] = mu
    kq["side"] = ks
    vq = quantize_rows(V16, side_of(spec, layer, False, head), None)
    vq["side"] = side_of(spec, layer, False, head)
    return kq, vq


def reconstruct_unit(spec: Spec, layer: int, K16, V16, kq, vq, seq_len: int, c16=None):
    """Keys and values attention sees for one unit (fp64 [T, D]); anchors override."""
    T = K16.shape[0]
    cK = None if c16 is None else np.broadcast_to(c16, K16.shape)
    mu = kq.get("mu")
    Kh = to_original_f64(kq["exact"], kq.get("side") or side_of(spec, layer, True), cK,
                         None if mu is None else np.broadcast_to(mu, K16.shape))
    Vh = to_original_f64(vq["exact"], vq.get("side") or side_of(spec, layer, False), None)
    an = anchored(spec, layer, np.arange(T), seq_len)
    if an.any():
        Kh[an] = anchor_rows(spec, np.asarray(K16)[an])["exact"]
        Vh[an] = anchor_rows(spec, np.asarray(V16)[an])["exact"]
    return Kh, Vh


def decode_query(spec: Spec, layer: int, q16: np.ndarray, Kh: np.ndarray, Vh: np.ndarray, kv_len: int):
    """q16 [Hq, D]; Kh, Vh [Hkv, T, D] reconstructed; returns (o, lse, p)."""
    return A.attention(np.asarray(q16, np.float16), Kh, Vh, kv_len, spec.sm_scale)


def effective_bits(spec: Spec, seq_len: int) -> float:
    """Average stored bits per K/V value over all layers (and kv-heads) of one sequence of length
    seq_len."""
    D = spec.D
    heads = spec.n_kv if (spec.head_k or spec.head_v) else 1
    tot = 0.0
    for layer in range(spec.n_layers):
        an = anchored(spec, layer, np.arange(seq_len), seq_len).sum()
        a_row = 16 * D if spec.anchor_bits == 16 else bits_per_value(anchor_side(spec), D) * D
        for h in range(heads):
            for side, is_k in ((side_of(spec, layer, True, h), True), (side_of(spec, layer, False, h), False)):
                per_row = bits_per_value(side, D) * D
                bits = (seq_len - an) * per_row + an * a_row
                if is_k and side.chan_scale:
                    bits += 16 * D
                if is_k and side.mean_sub:
                    bits += 16 * D
                tot += bits
    return tot / (spec.n_layers * heads * 2 * seq_len * D)
