"""Per-head bit allocation from attention entropy (llama.cpp issue #21385, "Finding 2").

The page allocates bits per attention head by the Renyi entropy of the head's attention
distribution, b_h = b_avg + 0.25 (H_avg - H_2(h)), where H_avg is the mean over heads, and keeps
the lowest-entropy ~2% of heads ("sink heads": 3 of GPT-2's 144) out of quantization entirely
("Feature Request: Per-Head KV Cache Types": sink heads at f16 or q8_0, standard heads at q4_0,
diffuse heads lower).

Readings taken here: H_2(p) = -log2 sum_t p_t^2 (in bits) for one query's attention over its
keys, and a head's entropy is the mean over its calibration queries (and over the query heads
that share the kv-head); b_h is rounded to the nearest integer (halves up) and clipped to the
grid's range; the sink count is round(0.02 x heads), the lowest entropies (ties to the lower
index), and those heads keep fp16 K and V.
"""
from __future__ import annotations

import math

import numpy as np


def renyi2(p: np.ndarray) -> float:
    """Renyi entropy of order 2 of one distribution, in bits."""
    p = np.asarray(p, dtype=np.float64)
    return float(-math.log2((p * p).sum()))


def head_bits(H2: np.ndarray, b_avg: float, lo: int = 2, hi: int = 8) -> np.ndarray:
    """Integer bits per head from the rule b_avg + 0.25 (mean(H2) - H2)."""
    H2 = np.asarray(H2, dtype=np.float64)
    b = b_avg + 0.25 * (H2.mean() - H2)
    return np.clip(np.floor(b + 0.5), lo, hi).astype(np.int64)


def sink_heads(H2: np.ndarray, frac: float = 0.02) -> np.ndarray:
    """Indices of the round(frac x heads) lowest-entropy heads."""
    H2 = np.asarray(H2, dtype=np.float64)
    n = int(math.floor(frac * H2.size + 0.5))
    return np.sort(np.argsort(H2, kind="stable")[:n])
