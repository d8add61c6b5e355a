"""Decode attention over a (partly) quantized KV cache, and the pages' error metrics; fp64.

Attention is the textbook definition: query head h reads kv-head floor(h / G) (contiguous
GQA groups), s_t = sm_scale * (q . k_t) for t < kv_len with sm_scale = 1/sqrt(D),
p = softmax(s), o = sum_t p_t v_t.  The keys and values are the oracle's own reconstruction
of the stored rows in the original domain; rows kept as fp16 anchors are used as stored.

Metrics, as defined in "E21W" "What I tested" (K/V error as squared error relative to the
signal energy, attention error as the relative error of the attention output, KL of the
attention distribution against the fp16 one) and averaged as in "E22L" "Result":
  X1 = sum (x - x_hat)^2 / sum x^2
  X2 = ||o - o_f16||_2 / ||o_f16||_2
  X3 = sum_t p_f16(t) ln(p_f16(t) / p_q(t))
"""
from __future__ import annotations

import math

import numpy as np

F64 = np.float64


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, kv_len: int, sm_scale: float | None = None):
    """One query position.  q [Hq, D]; K, V [Hkv, T, D] (any float); returns (o [Hq, D],
    lse [Hq] natural-log, p [Hq, kv_len]) in fp64."""
    q = np.asarray(q, dtype=F64)
    K = np.asarray(K, dtype=F64)
    V = np.asarray(V, dtype=F64)
    Hq, D = q.shape
    Hkv = K.shape[0]
    G = Hq // Hkv
    if sm_scale is None:
        sm_scale = 1.0 / math.sqrt(D)
    o = np.zeros((Hq, D))
    lse = np.full(Hq, -np.inf)
    P = np.zeros((Hq, kv_len))
    for h in range(Hq):
        j = h // G
        if kv_len == 0:
            continue
        s = sm_scale * (K[j, :kv_len] @ q[h])
        m = s.max()
        e = np.exp(s - m)
        l = e.sum()
        p = e / l
        o[h] = p @ V[j, :kv_len]
        lse[h] = m + math.log(l)
        P[h] = p
    return o, lse, P


def rel_sq_error(x, x_hat) -> float:
    x = np.asarray(x, dtype=F64)
    x_hat = np.asarray(x_hat, dtype=F64)
    return float(((x - x_hat) ** 2).sum() / (x ** 2).sum())


def rel_l2(o, o_ref) -> float:
    o = np.asarray(o, dtype=F64)
    o_ref = np.asarray(o_ref, dtype=F64)
    return float(np.linalg.norm(o - o_ref) / np.linalg.norm(o_ref))


def kl(p_ref, p) -> float:
    p_ref = np.asarray(p_ref, dtype=F64)
    p = np.asarray(p, dtype=F64)
    mask = p_ref > 0
    return float((p_ref[mask] * np.log(p_ref[mask] / p[mask])).sum())


def rel_inf(o, o_ref) -> float:
    """Max-abs error over max-abs reference, the per-vector decode tolerance measure."""
    o = np.asarray(o, dtype=F64)
    o_ref = np.asarray(o_ref, dtype=F64)
    return float(np.abs(o - o_ref).max() / np.abs(o_ref).max())
