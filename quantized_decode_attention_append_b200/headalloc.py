"""Per-head KV formats from attention entropy: the calibration pass of llama.cpp issue #21385.

"Finding 2" allocates bits per attention head from the Renyi entropy of the head's attention,
b_h = b_avg + 0.25 (H_avg - H_2(h)), and skips quantization for the lowest-entropy ~2% of heads
(the "sink heads", 3 of GPT-2's 144); "Feature Request: Per-Head KV Cache Types" asks for a
calibration pass computing per-head entropy, per-head type selection and per-head dequantization.
The last two are the library's (kvq_create_heads); this module is the calibration, run once on
fp16 keys and calibration queries.

Conventions: H_2 = -log2 sum_t p_t^2 in bits, per query and query head, averaged over the
calibration queries and the query heads that share a kv-head; H_avg is the mean over every
(layer, kv-head); b_h is rounded to the nearest integer (halves up) and clipped to [lo, hi]; the
round(0.02 x heads) lowest-entropy heads (ties to the lower index) take the sink format.
"""
from __future__ import annotations

import math

import torch

from .kvq import Side


def head_entropy(q: torch.Tensor, K: torch.Tensor, kv_len=None, sm_scale: float | None = None) -> torch.Tensor:
    """Mean Renyi-2 entropy (bits) of each kv-head's attention.

    q: [n, Hq, D] queries; K: [Hkv, T, D] keys (fp16 or fp32, any device); kv_len: per-query key
    counts (keys t < kv_len[i]; default all T).  Returns [Hkv] float64."""
    n, Hq, D = q.shape
    Hkv, T, _ = K.shape
    G = Hq // Hkv
    scale = sm_scale or 1.0 / math.sqrt(D)
    qf = q.double().view(n, Hkv, G, D)
    kf = K.double()
    s = torch.einsum("nhgd,htd->nhgt", qf, kf) * scale
    if kv_len is not None:
        kl = torch.as_tensor(kv_len, device=s.device).view(n, 1, 1, 1)
        s = s.masked_fill(torch.arange(T, device=s.device).view(1, 1, 1, T) >= kl, float("-inf"))
    p = torch.softmax(s, dim=-1)
    h2 = -torch.log2((p * p).sum(dim=-1))  # [n, Hkv, G]
    return h2.mean(dim=(0, 2))


def allocate(H2, b_avg: float = 4.0, side_of_bits=None, sink: Side | None = None, sink_frac: float = 0.02,
             lo: int = 2, hi: int = 8):
    """Per-(layer, kv-head) sides from entropies H2 [n_layers, n_kv_heads].

    side_of_bits(b) -> Side gives the format of a b-bit head (default: absmax int, groups of 32);
    sink (default fp16) is the sink heads' format.  Returns (head_k, head_v, bits) with bits the
    [n_layers, n_kv_heads] integer allocation (16 for sinks)."""
    H2 = torch.as_tensor(H2, dtype=torch.float64).cpu()
    side_of_bits = side_of_bits or (lambda b: Side("int", b, group=32))
    sink = sink or Side("fp16")
    L, H = H2.shape
    flat = H2.reshape(-1)
    b = torch.clamp(torch.floor(b_avg + 0.25 * (flat.mean() - flat) + 0.5), lo, hi).to(torch.int64)
    n_sink = int(math.floor(sink_frac * flat.numel() + 0.5))
    order = sorted(range(flat.numel()), key=lambda i: (float(flat[i]), i))
    sinks = set(order[:n_sink])
    bits = [[16 if l * H + h in sinks else int(b[l * H + h]) for h in range(H)] for l in range(L)]
    head = tuple(tuple(sink if bits[l][h] == 16 else side_of_bits(bits[l][h]) for h in range(H)) for l in range(L))
    return head, head, bits
