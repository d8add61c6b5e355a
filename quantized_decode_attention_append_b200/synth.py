"""Seeded synthetic KV-cache inputs (shared by the tests, the benchmark and the oracle checks).

This module holds none of the quantization or attention arithmetic: it only draws inputs.
It stands in for the real caches the source pages measured on (the "wikiA/wikiB/mathA"
f16 slot dumps of "E21W: 3-bit cache variants, proxy queries" and the 64K spans of
"E22L: 2-bit value cache for a 1M budget"), which are not available.

Law (the same for every workload):
  * K, V ~ N(0, 1) in fp16.  Samples come from a 65536-entry table of standard-normal
    quantiles (built in float64, rounded to fp16) indexed by a counter-based 32-bit hash of
    (seed, side, layer, sequence, kv-head, token, channel).  The hash uses only exact integer
    arithmetic, so a slice drawn on the GPU is bit-identical to the same slice drawn on the CPU.
  * 4 outlier channels per (layer, kv-head) and side, picked by the hash, scaled x20.
  * token 0 scaled x50 (attention sink) in K and V.
  * K gets RoPE (base 1e4, rotate-half pairing j <-> j + D/2, theta_j = 1e4^(-2j/D),
    position = token index).  The cos/sin table is built in float64 and rounded to fp32;
    the rotation is evaluated as separate fp32 multiplies and a subtraction/addition (no
    fused multiply-add), then rounded to fp16.
  * queries: the same law with their own seed, RoPE'd at the decode position.

All functions return torch tensors on the requested device; generation on "cuda" and "cpu"
gives identical bits.
"""
from __future__ import annotations

import functools
import statistics

import numpy as np
import torch

M32 = 0xFFFFFFFF

# stream tags keep the K, V, query and outlier draws independent
TAG_K, TAG_V, TAG_Q, TAG_OUT_K, TAG_OUT_V, TAG_PROXY = 1, 2, 3, 4, 5, 6

N_OUTLIERS = 4
OUTLIER_GAIN = 20.0
SINK_GAIN = 50.0
ROPE_BASE = 1.0e4


@functools.lru_cache(maxsize=1)
def normal_table_np() -> np.ndarray:
    """65536 standard-normal quantiles at probabilities (i + 1/2) / 65536, as fp16."""
    nd = statistics.NormalDist()
    vals = np.array([nd.inv_cdf((i + 0.5) / 65536.0) for i in range(65536)], dtype=np.float64)
    return vals.astype(np.float16)


_TABLE_CACHE: dict = {}


def normal_table(device) -> torch.Tensor:
    key = str(device)
    if key not in _TABLE_CACHE:
        _TABLE_CACHE[key] = torch.from_numpy(normal_table_np().copy()).to(device)
    return _TABLE_CACHE[key]


def _mulmod32(x: torch.Tensor, c: int) -> torch.Tensor:
    """(x * c) mod 2^32 for int64 tensors holding values in [0, 2^32), without int64 overflow."""
    lo = x & 0xFFFF
    hi = x >> 16
    return (lo * c + (((hi * c) & 0xFFFF) << 16)) & M32


def _mix(x: torch.Tensor) -> torch.Tensor:
    """32-bit integer finaliser (xor-shift / multiply rounds); a bijection on [0, 2^32)."""
    x = x ^ (x >> 16)
    x = _mulmod32(x, 0x7FEB352D)
    x = x ^ (x >> 15)
    x = _mulmod32(x, 0x846CA68B)
    x = x ^ (x >> 16)
    return x


def _mix_int(x: int) -> int:
    x &= M32
    x ^= x >> 16
    x = (x * 0x7FEB352D) & M32
    x ^= x >> 15
    x = (x * 0x846CA68B) & M32
    x ^= x >> 16
    return x


def _chain(h: torch.Tensor, v) -> torch.Tensor:
    return _mix((h ^ (v & M32)) & M32)


def _prefix(seed: int, tag: int, layer: int) -> int:
    h = _mix_int(seed * 0x9E3779B1 + 0x632BE5AB)
    h = _mix_int(h ^ tag)
    h = _mix_int(h ^ (layer & M32))
    return h


def gaussian_rows(seed: int, tag: int, layer: int, seqs, heads, tokens, D: int, device="cpu") -> torch.Tensor:
    """N(0,1) fp16 draws of shape [len(seqs), len(heads), len(tokens), D]."""
    dev = torch.device(device)
    s = torch.as_tensor(seqs, dtype=torch.int64, device=dev).view(-1, 1, 1)
    hh = torch.as_tensor(heads, dtype=torch.int64, device=dev).view(1, -1, 1)
    tt = torch.as_tensor(tokens, dtype=torch.int64, device=dev).view(1, 1, -1)
    base = torch.full((1, 1, 1), _prefix(seed, tag, layer), dtype=torch.int64, device=dev)
    h = _chain(base, s)
    h = _chain(h, hh)
    h = _chain(h, tt)  # [S, H, T]
    ch = torch.arange(D, dtype=torch.int64, device=dev)
    e = _mix((_mulmod32(h.unsqueeze(-1), 0x9E3779B1) + ch + 0x7F4A7C15) & M32)
    idx = e >> 16
    tab = normal_table(dev)
    return tab[idx]


def outlier_channels(seed: int, side_tag: int, layer: int, head: int, D: int) -> np.ndarray:
    """The 4 outlier channels of one (layer, kv-head): the channels with the largest hash."""
    hs = []
    base = _prefix(seed, side_tag, layer)
    base = _mix_int(base ^ head)
    for j in range(D):
        hs.append((_mix_int(base ^ (j * 0x01000193)), -j))
    order = sorted(range(D), key=lambda j: hs[j], reverse=True)
    return np.array(sorted(order[:N_OUTLIERS]), dtype=np.int64)


def outlier_mask(seed: int, side_tag: int, layer: int, heads, D: int, device="cpu") -> torch.Tensor:
    m = torch.zeros(len(heads), D, dtype=torch.bool)
    for i, h in enumerate(heads):
        m[i, torch.from_numpy(outlier_channels(seed, side_tag, layer, int(h), D))] = True
    return m.to(device)


@functools.lru_cache(maxsize=8)
def rope_table_np(max_pos: int, D: int):
    """fp32 cos/sin of pos * theta_j for pos in [0, max_pos), j in [0, D/2)."""
    half = D // 2
    theta = ROPE_BASE ** (-2.0 * np.arange(half, dtype=np.float64) / D)
    ang = np.arange(max_pos, dtype=np.float64)[:, None] * theta[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope_positions(x16: torch.Tensor, positions) -> torch.Tensor:
    """Rotate-half RoPE of fp16 rows x16 [..., T, D] at the given token positions; fp16 out."""
    D = x16.shape[-1]
    half = D // 2
    pos = np.asarray(positions, dtype=np.int64)
    cos_np, sin_np = rope_table_np(int(pos.max()) + 1, D)
    dev = x16.device
    c = torch.from_numpy(cos_np[pos]).to(dev)
    s = torch.from_numpy(sin_np[pos]).to(dev)
    x = x16.float()
    a, b = x[..., :half], x[..., half:]
    ra = a * c - b * s
    rb = b * c + a * s
    return torch.cat([ra, rb], dim=-1).to(torch.float16)


def kv_rows(seed: int, side: str, layer: int, seqs, heads, tokens, D: int, device="cpu",
            outlier_seed: int | None = None) -> torch.Tensor:
    """Synthetic K or V rows [S, H, T, D] (fp16) following the module law.  The outlier channels
    are a property of the (layer, kv-head): `outlier_seed` (default `seed`) picks them."""
    tag = TAG_K if side == "k" else TAG_V
    otag = TAG_OUT_K if side == "k" else TAG_OUT_V
    x = gaussian_rows(seed, tag, layer, seqs, heads, tokens, D, device)
    om = outlier_mask(seed if outlier_seed is None else outlier_seed, otag, layer, heads, D, device)  # [H, D]
    gain = torch.where(om, torch.tensor(OUTLIER_GAIN, dtype=torch.float16, device=om.device),
                       torch.tensor(1.0, dtype=torch.float16, device=om.device))
    x = x * gain.view(1, len(heads), 1, D)
    tt = torch.as_tensor(tokens, dtype=torch.int64, device=x.device)
    sink = (tt == 0).view(1, 1, -1, 1)
    x = torch.where(sink, x * torch.tensor(SINK_GAIN, dtype=torch.float16, device=x.device), x)
    if side == "k":
        x = rope_positions(x, np.asarray(tokens, dtype=np.int64))
    return x


def queries(seed: int, layer: int, n: int, n_heads: int, D: int, position: int, device="cpu") -> torch.Tensor:
    """Decode queries [n, Hq, D] fp16 ~ N(0,1), RoPE'd at `position`."""
    x = gaussian_rows(seed, TAG_Q, layer, list(range(n)), list(range(n_heads)), [0], D, device)
    x = x[:, :, 0, :]  # [n, Hq, D]
    x = x.unsqueeze(2)  # [n, Hq, 1, D]
    return rope_positions(x, np.array([position])).squeeze(2)


def proxy_positions(seed: int, n: int, lo: int, hi: int) -> np.ndarray:
    """n distinct positions drawn uniformly from [lo, hi) (proxy-query recipe of "E21W")."""
    keys = [(_mix_int(_prefix(seed, TAG_PROXY, 0) ^ p), p) for p in range(lo, hi)]
    keys.sort(reverse=True)
    return np.array(sorted(p for _, p in keys[:n]), dtype=np.int64)


def channel_scale(seed: int, layer: int, n_kv_heads: int, T: int, D: int) -> torch.Tensor:
    """Per-channel K scale c [Hkv, D] fp16: RMS over tokens of a calibration cache.

    The calibration cache follows the same law with seed + 1000 (one sequence) and the same
    outlier channels (those belong to the layer and head, not to the text).  RMS rather than
    absmax because the x50 sink token would otherwise set every channel's scale.
    """
    k = kv_rows(seed + 1000, "k", layer, [0], list(range(n_kv_heads)), list(range(T)), D, "cpu", outlier_seed=seed)
    k64 = k[0].double()  # [H, T, D]
    rms = torch.sqrt((k64 * k64).mean(dim=1))
    return rms.to(torch.float16)
