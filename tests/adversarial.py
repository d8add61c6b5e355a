"""Seeded fp16 K/V rows built to sit on the quantizers' decision boundaries (test inputs only).

Four row kinds, by token index mod 4:
  0  power-of-two grids: x = s j / 2 (j in -16..16), the first channel of every 4-channel block
     at +-8 s, so every group's largest magnitude is 8 s, often with both signs present (the
     first-index rule decides), and x / d lands exactly on half-integers for 2-, 3- and 4-bit
     absmax grids and on +-s/2 for ternary;
  1  NF4 boundaries: the first channel of every 16-channel block at +-s (so the group scale is
     s) and the others at the smallest fp16 at or above a level midpoint times s, or the fp16
     just below it;
  2  min-max grids: x = z + s j / 2 over j in 0..30 with the ends present in every 16-channel
     block, so the 4-bit step is exactly s and (x - z) / d hits half-integers;
  3  zero blocks: 8-channel blocks of +0 / -0 among Gaussian values.
"""
from __future__ import annotations

import numpy as np

from oracle.nf4 import nf4_levels


def _pred16(x: np.ndarray) -> np.ndarray:
    return np.nextafter(x.astype(np.float16), np.float16(-np.inf))


def _up16(x64: np.ndarray) -> np.ndarray:
    """Smallest fp16 >= x (x in fp64)."""
    h = x64.astype(np.float16)
    lo = h.astype(np.float64) < x64
    h[lo] = np.nextafter(h[lo], np.float16(np.inf))
    return h


def rows(seed: int, B: int, H: int, T: int, D: int) -> np.ndarray:
    rng = np.random.default_rng(seed)
    out = np.zeros((B, H, T, D), dtype=np.float16)
    lev = nf4_levels()
    mids = (lev[:-1] + lev[1:]) / 2.0
    for b in range(B):
        for h in range(H):
            for t in range(T):
                kind = t % 4
                s = 2.0 ** int(rng.integers(-4, 3))
                if kind == 0:
                    j = rng.integers(-16, 17, size=D).astype(np.float64)
                    j[::4] = 16.0 * rng.choice([-1.0, 1.0], size=D // 4)
                    r = s * j / 2.0
                elif kind == 1:
                    k = rng.integers(0, 15, size=D)
                    up = _up16(mids[k] * s)
                    r = np.where(rng.random(D) < 0.5, up, _pred16(up)).astype(np.float64)
                    r[::16] = s * rng.choice([-1.0, 1.0], size=D // 16)
                elif kind == 2:
                    z = -4.0 * s
                    j = rng.integers(0, 31, size=D).astype(np.float64)
                    j[::16] = 0.0
                    j[1::16] = 30.0
                    r = z + s * j / 2.0
                else:
                    r = rng.standard_normal(D)
                    for c0 in range(0, D, 8):
                        if rng.random() < 0.5:
                            r[c0:c0 + 8] = np.where(rng.random(8) < 0.5, 0.0, -0.0)
                out[b, h, t] = r.astype(np.float16)
    return out


def spike_rows(seed: int, B: int, H: int, T: int, D: int, n: int) -> np.ndarray:
    """Rows whose orthonormal Hadamard image (blocks of n) lands on absmax ties.

    Each n-channel block holds three spikes (2^(b-1), 2^(b-1) - 1/2, 1/2) x u at random channels,
    b in {2, 3, 4} and u a power of two drawn per row.  The block's image is
    (+-2^(b-1) +- (2^(b-1) - 1/2) +- 1/2) u / sqrt(n): magnitudes 2^b u, (2^b - 1) u, u and 0
    (over sqrt n), so a group's largest magnitude usually occurs with both signs (the first-index
    rule decides) and the b-bit grid's x/d hits half-integers exactly when 1/sqrt(n) is exact
    (n = 256) and within one rounding otherwise (n = 128).  A quarter of the rows add small
    Gaussian noise so that near-ties are reached from both sides."""
    rng = np.random.default_rng(seed)
    out = np.zeros((B, H, T, D), dtype=np.float16)
    for b_ in range(B):
        for h in range(H):
            for t in range(T):
                r = np.zeros(D)
                for blk in range(0, D, n):
                    b = int(rng.integers(2, 5))
                    u = 2.0 ** int(rng.integers(-3, 3))
                    ch = blk + rng.choice(n, size=3, replace=False)
                    r[ch] = np.array([2.0 ** (b - 1), 2.0 ** (b - 1) - 0.5, 0.5]) * u * rng.choice([-1.0, 1.0], 3)
                if t % 4 == 3:
                    r += rng.standard_normal(D) * 2.0 ** -12
                out[b_, h, t] = r.astype(np.float16)
    return out


def polar_boundary_rows(seed: int, n_rows: int, bp: int, pool: int = 40000) -> np.ndarray:
    """fp16 rows (head_dim 128) chosen from a seeded pool so that some folded-spectrum slot's angle
    sits next to a phase-code boundary (k + 1/2) 2 pi / 2^bp.  The oracle's own fp32 FFT decides
    where the angle is; half of the rows are the pool's closest cases (within the GPU's fp64
    fallback band), the other half sit just outside that band (where fp32 atan2 decides)."""
    from oracle import transforms as OT
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((pool, 128)) * 2.0).astype(np.float16)
    a, b = OT.fold_spectrum(*OT.dft_dit_f32(x.astype(np.float32)))
    th = np.arctan2(b.astype(np.float64), a.astype(np.float64))
    v = (th + np.pi) * (2 ** bp) / (2.0 * np.pi) + 0.5
    dist = np.abs(v - np.round(v))            # distance (in code steps) to a rounding boundary
    dist[(a == 0) & (b == 0)] = 1.0
    near = dist.min(axis=1)
    edge = np.abs(dist - 1.05e-3).min(axis=1)  # just outside a 1e-3 guard band
    k = n_rows // 2
    pick = np.concatenate([np.argsort(near)[:k], np.argsort(edge)[:n_rows - k]])
    return x[pick]
