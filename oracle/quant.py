"""Group quantizers, code packing and stored-domain dequantization (one K or V row at a time).

Every code is the nearest grid level of the scaled value in exact arithmetic, ties toward
the larger code.  The decision is taken by exact fp64 comparisons against thresholds that
are exact in fp64 (small odd integers times an fp16 scale, plus an fp16 zero point), so
rounding in a division can never flip a code.

Grids and scales (sources by page title and section):
  * signed absmax int b, ggml-style: "E22L" "What I tested" (absmax scaling, one fp16 scale
    per group) and "Result" (the 2-bit grid is the ggml signed one, levels -2..1 times the
    scale, one level fewer on the positive side); q4_0 in llama.cpp #21385 "Finding 1".  The group's largest-magnitude element m (first index on ties)
    maps to -2^(b-1): d = fp16(m / -2^(b-1)), q = clamp(round(x/d), -2^(b-1), 2^(b-1)-1),
    stored as the unsigned code q + 2^(b-1).
  * per-token min-max (asymmetric): "E21W" "What I tested", variant A.  z = fp16(min), d = fp16(fp32(max - min) / (2^b - 1)),
    q = clamp(round((x - z)/d), 0, 2^b - 1).  The minimum orders -0 below +0 (IEEE 754
    minimum), so a group whose smallest value is zero stores z = -0 if it holds a -0.
  * NF4: "Fourier Magnitude KV Cache Quantization" post 6 (NF4 in groups of 64); s = fp16(max|x|),
    code = nearest level of x/s (see oracle.nf4).
  * ternary {-s, 0, +s}: post 6 "Milestone" table (ternary in groups of 8 and 4);
    s = fp16(max|x|), t = nearest of {-1, 0, 1} to x/s.
  * sign {-s, +s}: post 6 "Minimal recipe" (one-bit sign KV with a scale);
    s = fp16(fp32 sum of |x| in channel order / g) (least-squares scale for fixed signs),
    t = +1 if x >= 0 else -1.
  * symmetric int b: "E22L" "Result" (the ggml grid has one level fewer on its positive side;
    the page names a symmetric grid as the next value grid to try).  Levels (q - (2^b - 1)/2) d for q = 0 .. 2^b - 1, so
    the outermost level is the group's largest magnitude m: d = fp16(fp32(m / (2^(b-1) - 1/2))),
    q = clamp(floor(x/d) + 2^(b-1), 0, 2^b - 1) (nearest level, ties up); d = 0 gives q = 2^(b-1).
  * Gaussian Lloyd-Max b: "E22L" "Result" (the other next candidate, "Gaussian Lloyd-Max levels
    on rotated values"); levels from oracle.lloyd in units of the group's RMS,
    s = fp16(sqrt(fp32(fp32 sum of x^2 in channel order / g))), code = nearest level of x/s
    (ties up); s = 0 gives the level just above zero, 2^(b-1).
  * sorted groups: post 6, "The winning recipe" item 1 (titled magnitude-sorted grouping: each
    row is sorted in descending order and quantized in groups, so the outliers end up together in
    one wide group; g = 8 for K and 4 for V, with 2-bit codes).  Reading taken here: a row is ordered by value, descending (equal values
    keep channel order), and consecutive g values of that order form a group on the per-token
    min-max grid (so the top group, where large outliers gather, gets its own wide range); the row
    stores each channel's rank (its position in the order) in ceil(log2 D) bits -- the permutation
    the page's bit counts leave out -- after the codes.
  * rFFT polar: the reply, "Fixed-rate magnitude/phase allocation" (mag/phase splits
    4+8 .. 8+4 at 12 bits per coefficient) and "The finite-phase implementation and the
    physical codec may be worth separating" (a magnitude index and one phase-angle index per
    rFFT coefficient).  Magnitude uniform over [0, max] with one fp16 scale per row:
    s = fp16(fp32(max_f |X_f|) / (2^bm - 1)); phase uniform over [-pi, pi):
    code = round((atan2 + pi) 2^bp / 2pi) mod 2^bp.
  * FFT Cartesian control: the reply, "The three controls I would try first" item 2 (real and
    imaginary parts instead of polar): the n folded spectrum reals, signed absmax int-b, one
    scale.

Packing: per row an LSB-first bit stream (element j at bits [b j, b j + b)); ternary packs
5 trits per byte (byte = sum_m d_m 3^m, d = t + 1, pad digits 0); polar stores the
magnitude stream then the phase stream.  Scales (and min-max zero points) are fp16, one per
group, in separate arrays.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

from . import transforms as T
from .lloyd import lloyd_max_levels
from .nf4 import nf4_levels

F32 = np.float32
F64 = np.float64


@dataclass(frozen=True)
class Side:
    fmt: str = "int"          # int | nf4 | ternary | sign | polar | cart | lloyd | sorted | fp16
    bits: int = 4             # code bits (magnitude bits for polar)
    bits2: int = 0            # phase bits (polar only)
    scale: str = "absmax"     # absmax | minmax | sym   (int only)
    group: int = 32           # channels per scale (polar/cart: the whole row)
    rot: int = 0              # 0 | 128 | 256 (Walsh-Hadamard block size)
    chan_scale: bool = False  # divide by a per-channel scale first (K only)
    mean_sub: bool = False    # subtract the sequence's key mean first (K only; oracle.cache)

    def n_groups(self, D: int) -> int:
        if self.fmt in ("polar", "cart"):
            return 1
        if self.fmt == "fp16":
            return 0
        return D // self.group

    def row_bytes(self, D: int) -> int:
        if self.fmt == "fp16":
            return 2 * D
        if self.fmt == "ternary":
            return -(-D // 5)
        if self.fmt == "sign":
            return -(-D // 8)
        if self.fmt == "polar":
            return (D // 2) * (self.bits + self.bits2) // 8
        if self.fmt == "nf4":
            return D // 2
        if self.fmt == "sorted":
            return -(-(D * self.bits + D * rank_bits(D)) // 8)
        return -(-D * self.bits // 8)  # int (absmax, minmax, sym), lloyd, cart

    def has_zero(self) -> bool:
        return (self.fmt == "int" and self.scale == "minmax") or self.fmt == "sorted"


def rank_bits(D: int) -> int:
    """Bits of one stored rank (channel position in the magnitude order): ceil(log2 D)."""
    return max(1, (D - 1).bit_length())


def f16(x) -> np.ndarray:
    """Round to IEEE binary16, nearest-even; returned as the fp16 value in fp64."""
    return np.asarray(x, dtype=F64).astype(np.float16).astype(F64)


def round_half_up_exact(x: np.ndarray, d: np.ndarray, z=0.0) -> np.ndarray:
    """k = floor((x - z) / d + 1/2) in exact arithmetic (d != 0; 0 where d == 0).

    Requires z + (k +- 1/2) d to be exact in fp64 (true for fp16 z and d and |k| < 2^12)
    and x exact in fp64 (true for fp32 x).  An fp64 estimate is corrected by comparing x
    with those exact thresholds.
    """
    x = np.asarray(x, dtype=F64)
    d = np.broadcast_to(np.asarray(d, dtype=F64), x.shape)
    z = np.broadcast_to(np.asarray(z, dtype=F64), x.shape)
    nz = d != 0
    with np.errstate(divide="ignore", invalid="ignore"):
        k = np.floor(np.where(nz, (x - z) / np.where(nz, d, 1.0), 0.0) + 0.5)
    pos = d > 0
    lo = z + (k - 0.5) * d
    below = np.where(pos, x < lo, x > lo) & nz
    k = np.where(below, k - 1, k)
    hi = z + (k + 0.5) * d
    above = np.where(pos, x >= hi, x <= hi) & nz & ~below
    k = np.where(above, k + 1, k)
    return np.where(nz, k, 0.0)


# ----------------------------------------------------------------------------- packing
def pack_bits(codes: np.ndarray, b: int) -> np.ndarray:
    codes = np.asarray(codes, dtype=np.int64)
    R, n = codes.shape
    nbytes = -(-n * b // 8)
    bits = ((codes[:, :, None] >> np.arange(b)) & 1).reshape(R, n * b)
    pad = nbytes * 8 - n * b
    if pad:
        bits = np.concatenate([bits, np.zeros((R, pad), dtype=np.int64)], axis=1)
    bits = bits.reshape(R, nbytes, 8)
    return (bits << np.arange(8)).sum(axis=-1).astype(np.uint8)


def unpack_bits(data: np.ndarray, b: int, n: int) -> np.ndarray:
    data = np.asarray(data, dtype=np.int64)
    R = data.shape[0]
    bits = ((data[:, :, None] >> np.arange(8)) & 1).reshape(R, -1)[:, : n * b]
    return (bits.reshape(R, n, b) << np.arange(b)).sum(axis=-1)


def pack_trits(digits: np.ndarray) -> np.ndarray:
    digits = np.asarray(digits, dtype=np.int64)
    R, n = digits.shape
    nb = -(-n // 5)
    pad = nb * 5 - n
    if pad:
        digits = np.concatenate([digits, np.zeros((R, pad), dtype=np.int64)], axis=1)
    digits = digits.reshape(R, nb, 5)
    return (digits * (3 ** np.arange(5))).sum(axis=-1).astype(np.uint8)


def unpack_trits(data: np.ndarray, n: int) -> np.ndarray:
    v = np.asarray(data, dtype=np.int64)
    out = np.stack([(v // (3 ** m)) % 3 for m in range(5)], axis=-1)
    return out.reshape(v.shape[0], -1)[:, :n]


# ----------------------------------------------------------------------------- quantizers
def quant_int_absmax(x32: np.ndarray, b: int, g: int):
    """Signed ggml-style grid -2^(b-1) .. 2^(b-1)-1; returns (q signed, d fp16 as f64)."""
    R, D = x32.shape
    xg = x32.reshape(R, D // g, g).astype(F64)
    idx = np.argmax(np.abs(xg), axis=-1)  # first index on ties
    m = np.take_along_axis(xg, idx[..., None], axis=-1)[..., 0]
    d = f16(m / -(2 ** (b - 1)))
    q = round_half_up_exact(xg, d[..., None])
    q = np.clip(q, -(2 ** (b - 1)), 2 ** (b - 1) - 1)
    return q.reshape(R, D).astype(np.int64), d


def quant_int_minmax(x32: np.ndarray, b: int, g: int):
    """Asymmetric grid 0 .. 2^b - 1 over [min, max]; returns (q, d, z)."""
    R, D = x32.shape
    xg = x32.reshape(R, D // g, g).astype(F32)
    mn = xg.min(axis=-1)
    mx = xg.max(axis=-1)
    # a zero minimum is -0 when the group holds a -0 (IEEE 754 minimum: -0 orders below +0)
    negz = np.any((xg == 0) & np.signbit(xg), axis=-1)
    mn = np.where(mn == 0, np.where(negz, F32(-0.0), F32(0.0)), mn).astype(F32)
    z = f16(mn)
    d = f16((mx - mn).astype(F32) / F32(2 ** b - 1))
    q = round_half_up_exact(xg.astype(F64), d[..., None], z[..., None])
    q = np.clip(q, 0, 2 ** b - 1)
    return q.reshape(R, D).astype(np.int64), d, z


def quant_nf4(x32: np.ndarray, g: int):
    R, D = x32.shape
    L = nf4_levels()
    mids = (L[:-1] + L[1:]) / 2.0
    xg = x32.reshape(R, D // g, g).astype(F64)
    s = f16(np.abs(xg).max(axis=-1))
    thr = mids[None, None, None, :] * s[..., None, None]
    code = (xg[..., None] >= thr).sum(axis=-1)
    zero_code = int(np.nonzero(L == 0.0)[0][0])
    code = np.where(s[..., None] == 0, zero_code, code)
    return code.reshape(R, D).astype(np.int64), s


def quant_ternary(x32: np.ndarray, g: int):
    R, D = x32.shape
    xg = x32.reshape(R, D // g, g).astype(F64)
    s = f16(np.abs(xg).max(axis=-1))
    h = s[..., None] / 2.0
    t = np.where(xg >= h, 1, np.where(xg < -h, -1, 0))
    t = np.where(s[..., None] == 0, 0, t)
    return t.reshape(R, D).astype(np.int64), s


def floor_exact(x: np.ndarray, d: np.ndarray) -> np.ndarray:
    """k = floor(x / d) in exact arithmetic for d > 0 (x fp32, d fp16, |k| < 2^12): an fp64
    estimate corrected by comparing x with the exact products k d and (k + 1) d."""
    x = np.asarray(x, dtype=F64)
    d = np.broadcast_to(np.asarray(d, dtype=F64), x.shape)
    pos = d > 0
    with np.errstate(divide="ignore", invalid="ignore"):
        k = np.floor(np.where(pos, x / np.where(pos, d, 1.0), 0.0))
    k = np.where(pos & (x < k * d), k - 1, k)
    k = np.where(pos & (x >= (k + 1) * d), k + 1, k)
    return np.where(pos, k, 0.0)


def quant_int_sym(x32: np.ndarray, b: int, g: int):
    """Symmetric grid (q - (2^b - 1)/2) d, q = 0 .. 2^b - 1; returns (q, d)."""
    R, D = x32.shape
    xg = x32.reshape(R, D // g, g).astype(F32)
    m = np.abs(xg).max(axis=-1).astype(F32)
    d = f16((m / F32(2 ** (b - 1) - 0.5)).astype(F32))
    q = floor_exact(xg.astype(F64), d[..., None]) + 2 ** (b - 1)
    q = np.clip(q, 0, 2 ** b - 1)
    q = np.where(d[..., None] == 0, 2 ** (b - 1), q)
    return q.reshape(R, D).astype(np.int64), d


def quant_lloyd(x32: np.ndarray, b: int, g: int):
    """Gaussian Lloyd-Max levels times the group RMS; returns (code, s)."""
    R, D = x32.shape
    L = lloyd_max_levels(b)
    mids = (L[:-1] + L[1:]) / 2.0
    xg = x32.reshape(R, D // g, g).astype(F32)
    acc = np.zeros(xg.shape[:-1], dtype=F32)
    for j in range(g):  # fp32 sum of the rounded squares, in channel order
        acc = (acc + (xg[..., j] * xg[..., j]).astype(F32)).astype(F32)
    s = f16(np.sqrt((acc / F32(g)).astype(F32)).astype(F32))
    thr = mids[None, None, None, :] * s[..., None, None]
    code = (xg.astype(F64)[..., None] >= thr).sum(axis=-1)
    code = np.where(s[..., None] == 0, 2 ** (b - 1), code)
    return code.reshape(R, D).astype(np.int64), s


def quant_sorted(x32: np.ndarray, b: int, g: int):
    """Sorted groups: returns (q at sorted positions, d and z per sorted group, rank per channel)."""
    R, D = x32.shape
    x = np.asarray(x32, dtype=F32)
    order = np.argsort(-x, axis=1, kind="stable")  # channel at each sorted position (descending)
    rank = np.empty_like(order)
    rank[np.arange(R)[:, None], order] = np.arange(D)[None, :]
    q, d, z = quant_int_minmax(np.take_along_axis(x, order, axis=1), b, g)
    return q, d, z, rank


def quant_sign(x32: np.ndarray, g: int):
    R, D = x32.shape
    xg = x32.reshape(R, D // g, g).astype(F32)
    acc = np.zeros(xg.shape[:-1], dtype=F32)
    for j in range(g):  # fp32 sum in channel order
        acc = (acc + np.abs(xg[..., j])).astype(F32)
    s = f16((acc / F32(g)).astype(F32))
    t = np.where(xg >= 0, 1, -1)
    return t.reshape(R, D).astype(np.int64), s


def phase_angles_f64(bp: int) -> np.ndarray:
    return -math.pi + 2.0 * math.pi * np.arange(2 ** bp) / (2 ** bp)


def quant_polar(x32: np.ndarray, bm: int, bp: int):
    """rFFT polar codec; returns (mag codes, phase codes, s) with n/2 slots per row."""
    re, im = T.dft_dit_f32(x32)
    a, b = T.fold_spectrum(re, im)
    mag = np.sqrt(((a * a).astype(F32) + (b * b).astype(F32)).astype(F32)).astype(F32)
    mmax = mag.max(axis=-1)
    s = f16((mmax / F32(2 ** bm - 1)).astype(F32))
    mc = round_half_up_exact(mag.astype(F64), s[:, None])
    mc = np.clip(mc, 0, 2 ** bm - 1).astype(np.int64)
    a64 = a.astype(F64)
    b64 = b.astype(F64)
    theta = np.arctan2(b64, a64)
    theta = np.where((a64 == 0) & (b64 == 0), 0.0, theta)
    v = (theta + math.pi) * (2 ** bp) / (2.0 * math.pi)
    pc = np.mod(np.floor(v + 0.5), 2 ** bp).astype(np.int64)
    return mc, pc, s


def interleave_slots(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    out = np.empty(a.shape[:-1] + (2 * a.shape[-1],), dtype=a.dtype)
    out[..., 0::2] = a
    out[..., 1::2] = b
    return out


# ----------------------------------------------------------------------------- rows
def transform_rows(x16: np.ndarray, side: Side, c16=None, mu16=None) -> np.ndarray:
    """fp16 rows -> fp32 rows in the domain the grid sees (key mean subtracted, then channel
    scale, then rotation)."""
    x = np.asarray(x16, dtype=np.float16).astype(F32)
    if side.mean_sub:
        x = (x - np.asarray(mu16, dtype=np.float16).astype(F32)).astype(F32)
    if side.chan_scale:
        x = T.channel_divide(x, np.asarray(c16, dtype=np.float16))
    if side.rot:
        x = T.fwht_f32(x, side.rot)
    return x


def quantize_rows(x16: np.ndarray, side: Side, c16=None, mu16=None) -> dict:
    """Quantize fp16 rows [R, D] of one side (mu16: the key mean, with side.mean_sub).  Returns
    a dict with
    bytes  uint8 [R, row_bytes]  logical packed codes
    scales float16 [R, G]         (min-max also: zeros float16 [R, G])
    stored float32 [R, D]         stored-domain dequantization (bit-exact definition)
    exact  float64 [R, D]         stored-domain dequantization in exact arithmetic
    """
    x16 = np.asarray(x16, dtype=np.float16)
    R, D = x16.shape
    out = {}
    if side.fmt == "fp16":
        out["bytes"] = x16.view(np.uint8).reshape(R, 2 * D).copy()
        out["scales"] = np.zeros((R, 0), np.float16)
        out["stored"] = x16.astype(F32)
        out["exact"] = x16.astype(F64)
        return out
    x = transform_rows(x16, side, c16, mu16)
    g = side.group
    if side.fmt == "int" and side.scale == "sym":
        q, d = quant_int_sym(x, side.bits, g)
        out["bytes"] = pack_bits(q, side.bits)
        dd = np.repeat(d, g, axis=1)
        lv = q - (2 ** side.bits - 1) / 2.0
        out["stored"] = (lv * dd).astype(F32)
        out["exact"] = lv * dd
        out["scales"] = d.astype(np.float16)
        out["q"] = q
    elif side.fmt == "lloyd":
        code, s = quant_lloyd(x, side.bits, g)
        L = lloyd_max_levels(side.bits)
        out["bytes"] = pack_bits(code, side.bits)
        val = L[code] * np.repeat(s, g, axis=1)
        out["stored"] = val.astype(F32)
        out["exact"] = val
        out["scales"] = s.astype(np.float16)
        out["q"] = code
    elif side.fmt == "sorted":
        q, d, z, rank = quant_sorted(x, side.bits, g)
        out["bytes"] = np.concatenate([pack_bits(q, side.bits), pack_bits(rank, rank_bits(D))], axis=1)
        rows = np.arange(R)[:, None]
        qq, dd, zz = q[rows, rank], d[rows, rank // g], z[rows, rank // g]  # channel order
        out["stored"] = (zz.astype(F32) + (qq * dd).astype(F32)).astype(F32)
        out["exact"] = zz + qq * dd
        out["scales"] = d.astype(np.float16)
        out["zeros"] = z.astype(np.float16)
        out["q"] = q
        out["rank"] = rank
    elif side.fmt == "int" and side.scale == "absmax":
        q, d = quant_int_absmax(x, side.bits, g)
        out["bytes"] = pack_bits(q + 2 ** (side.bits - 1), side.bits)
        dd = np.repeat(d, g, axis=1)
        out["stored"] = (q * dd).astype(F32)
        out["exact"] = q * dd
        out["scales"] = d.astype(np.float16)
        out["q"] = q
    elif side.fmt == "int" and side.scale == "minmax":
        q, d, z = quant_int_minmax(x, side.bits, g)
        out["bytes"] = pack_bits(q, side.bits)
        dd = np.repeat(d, g, axis=1)
        zz = np.repeat(z, g, axis=1)
        out["stored"] = (zz.astype(F32) + (q * dd).astype(F32)).astype(F32)
        out["exact"] = zz + q * dd
        out["scales"] = d.astype(np.float16)
        out["zeros"] = z.astype(np.float16)
        out["q"] = q
    elif side.fmt == "nf4":
        code, s = quant_nf4(x, g)
        L = nf4_levels()
        out["bytes"] = pack_bits(code, 4)
        val = L[code] * np.repeat(s, g, axis=1)
        out["stored"] = val.astype(F32)
        out["exact"] = val
        out["scales"] = s.astype(np.float16)
        out["q"] = code
    elif side.fmt == "ternary":
        t, s = quant_ternary(x, g)
        out["bytes"] = pack_trits(t + 1)
        val = t * np.repeat(s, g, axis=1)
        out["stored"] = val.astype(F32)
        out["exact"] = val
        out["scales"] = s.astype(np.float16)
        out["q"] = t
    elif side.fmt == "sign":
        t, s = quant_sign(x, g)
        out["bytes"] = pack_bits((t > 0).astype(np.int64), 1)
        val = t * np.repeat(s, g, axis=1)
        out["stored"] = val.astype(F32)
        out["exact"] = val
        out["scales"] = s.astype(np.float16)
        out["q"] = t
    elif side.fmt == "polar":
        bm, bp = side.bits, side.bits2
        mc, pc, s = quant_polar(x, bm, bp)
        out["bytes"] = np.concatenate([pack_bits(mc, bm), pack_bits(pc, bp)], axis=1)
        phi = phase_angles_f64(bp)
        cos32 = np.array([math.cos(v) for v in phi], dtype=F64).astype(F32)  # libm, per entry
        sin32 = np.array([math.sin(v) for v in phi], dtype=F64).astype(F32)
        m = (mc * s[:, None]).astype(F32)  # exact
        a32 = (m * cos32[pc]).astype(F32)
        b32 = (m * sin32[pc]).astype(F32)
        out["stored"] = interleave_slots(a32, b32)
        m64 = mc * s[:, None]
        out["exact"] = interleave_slots(m64 * np.cos(phi[pc]), m64 * np.sin(phi[pc]))
        out["scales"] = s[:, None].astype(np.float16)
        out["q"] = np.concatenate([mc, pc], axis=1)
    elif side.fmt == "cart":
        re, im = T.dft_dit_f32(x)
        a, b = T.fold_spectrum(re, im)
        y = interleave_slots(a, b)
        q, d = quant_int_absmax(y, side.bits, D)
        out["bytes"] = pack_bits(q + 2 ** (side.bits - 1), side.bits)
        out["stored"] = (q * d).astype(F32)
        out["exact"] = q * d
        out["scales"] = d.astype(np.float16)
        out["q"] = q
    else:
        raise ValueError(side)
    return out


def to_original_f64(stored64: np.ndarray, side: Side, c16=None, mu16=None) -> np.ndarray:
    """Undo the pre-transform of stored-domain rows, fp64: (i)DFT, then rotation, then x c,
    then + the key mean."""
    y = np.asarray(stored64, dtype=F64)
    if side.fmt in ("polar", "cart"):
        y = T.unfold_idft_f64(y[..., 0::2], y[..., 1::2])
    if side.rot:
        y = T.hadamard_inverse_f64(y, side.rot)
    if side.chan_scale:
        y = y * np.asarray(c16, dtype=np.float16).astype(F64)
    if side.mean_sub:
        y = y + np.asarray(mu16, dtype=np.float16).astype(F64)
    return y


def bits_per_value(side: Side, D: int) -> float:
    """Storage bits per value of one quantized row: codes + fp16 scales (+ fp16 zeros)."""
    if side.fmt == "fp16":
        return 16.0
    code_bits = side.row_bytes(D) * 8 if side.fmt in ("ternary", "sorted") else (
        (D // 2) * (side.bits + side.bits2) if side.fmt == "polar" else
        D * (1 if side.fmt == "sign" else (4 if side.fmt == "nf4" else side.bits)))
    meta = 16 * side.n_groups(D) * (2 if side.has_zero() else 1)
    return (code_bits + meta) / D
