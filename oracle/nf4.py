"""NF4 (4-bit NormalFloat) level table.

The pages use NF4 as a K-cache grid ("Fourier Magnitude KV Cache Quantization", post 6:
"Corrected semantics" lists NF4 with groups of 64 at 4.25 b, the "Milestone" table pairs NF4 K
with int4-g64 V, and "Mechanism findings" credits fixed non-uniform codebooks that keep the
full range) but print no table.  This follows
the published NormalFloat construction (Dettmers et al., QLoRA, 2023): normal quantiles, 8
levels above zero and 7 below, an exact zero, extremes normalised to +-1.  The outer
probability is delta = 1 - (1/(2*15) + 1/(2*16)) / 2, the mean of the 15- and 16-level
half-offsets.

Reading taken here: levels are stored at fp16 precision (rounded from the fp64
construction).  That makes every level times an fp16 scale exact in fp32 and lets decode
feed levels to fp16 tensor-core operands without rounding.

Parity unpinned as to the exact values (no table on the pages); the tests pin the
construction's own properties (count, order, exact 0 and +-1, quantile spacing via erf).
"""
from __future__ import annotations

import statistics

import numpy as np

DELTA = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0)


def nf4_levels_f64() -> np.ndarray:
    nd = statistics.NormalDist()
    pos_p = np.linspace(DELTA, 0.5, 9)[:-1]
    neg_p = np.linspace(DELTA, 0.5, 8)[:-1]
    pos = [nd.inv_cdf(float(p)) for p in pos_p]
    neg = [-nd.inv_cdf(float(p)) for p in neg_p]
    vals = np.array(sorted(pos + neg + [0.0]), dtype=np.float64)
    return vals / np.max(np.abs(vals))


def nf4_levels() -> np.ndarray:
    """The 16 sorted levels as fp16-representable float64 values."""
    return nf4_levels_f64().astype(np.float16).astype(np.float64)
