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
