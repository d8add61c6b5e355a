"""Pre-transforms applied to a K/V row before group quantization, and their fp64 inverses.

Forward transforms run in fp32 in a fixed evaluation order, because their outputs decide
integer codes; the inverses (used only for reconstruction and attention) run in fp64.

* Per-channel K scale: "E21W" "What I tested", variants C and D (keys divided by calibrated
  per-channel scales, multiplied back after dequantization).  x_j <- x_j / c_j (IEEE fp32
  division).
* Walsh-Hadamard rotation: "E21W" variant B and "E22L" "What I tested" (a 256-wide Hadamard
  applied before quantizing).  Sylvester order, no random signs, orthonormal (1/sqrt(n));
  block-diagonal when n < D.
* rFFT polar / Cartesian split: "Fourier Magnitude KV Cache Quantization" reply, "The
  finite-phase implementation and the physical codec may be worth separating" (magnitude and
  phase-angle indices per rFFT coefficient, inverted by an irFFT) and "The three controls I
  would try first" (the real/imaginary control).
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32


def channel_divide(x32: np.ndarray, c16: np.ndarray) -> np.ndarray:
    """x / c in fp32 (c broadcast over the last axis)."""
    return (x32.astype(F32) / c16.astype(F32)).astype(F32)


def hadamard_scale(n: int) -> np.float32:
    """fp32 nearest to 1/sqrt(n) for n = 128 (sqrt(2)/16) or 256 (1/16)."""
    if n == 256:
        return F32(1.0 / 16.0)
    if n == 128:
        return F32(np.sqrt(F32(2.0)) / F32(16.0))
    raise ValueError(n)


def fwht_f32(x: np.ndarray, n: int) -> np.ndarray:
    """Orthonormal Sylvester Hadamard over blocks of n channels, fp32.

    Stages h = 1, 2, 4, ..., n/2 in that order; stage h maps the pair (i, i+h) with bit h of
    i clear to (y_i + y_{i+h}, y_i - y_{i+h}); then every entry is multiplied by fp32(1/sqrt n).
    """
    x = np.asarray(x, dtype=F32)
    shape = x.shape
    D = shape[-1]
    assert D % n == 0
    y = x.reshape(-1, D // n, n).copy()
    h = 1
    while h < n:
        y = y.reshape(y.shape[0], D // n, n // (2 * h), 2, h)
        a = y[..., 0, :]
        b = y[..., 1, :]
        y = np.stack([a + b, a - b], axis=-2).astype(F32)
        h *= 2
    y = y.reshape(-1, D // n, n) * hadamard_scale(n)
    return y.astype(F32).reshape(shape)


def sylvester(n: int) -> np.ndarray:
    """The n x n Sylvester Hadamard matrix (entries +-1), fp64, by the doubling construction."""
    H = np.array([[1.0]])
    while H.shape[0] < n:
        H = np.block([[H, H], [H, -H]])
    return H


def hadamard_inverse_f64(y: np.ndarray, n: int) -> np.ndarray:
    """Inverse of the orthonormal block rotation (it is its own inverse), fp64."""
    y = np.asarray(y, dtype=np.float64)
    D = y.shape[-1]
    Hn = sylvester(n) / math.sqrt(n)
    yb = y.reshape(y.shape[:-1] + (D // n, n))
    return (yb @ Hn.T).reshape(y.shape)


def _bitrev(n: int) -> np.ndarray:
    bits = n.bit_length() - 1
    return np.array([int(format(i, f"0{bits}b")[::-1], 2) for i in range(n)], dtype=np.int64)


def twiddles_f32(n: int):
    """W_n^k = exp(-2 pi i k / n) for k < n/2: fp64 libm cos/sin rounded to fp32."""
    wr = np.array([math.cos(2.0 * math.pi * k / n) for k in range(n // 2)], dtype=np.float64).astype(F32)
    wi = np.array([-math.sin(2.0 * math.pi * k / n) for k in range(n // 2)], dtype=np.float64).astype(F32)
    return wr, wi


def dft_dit_f32(x: np.ndarray):
    """Length-n DFT of real rows by the radix-2 decimation-in-time FFT, fp32.

    Bit-reversed input order; stages of span 2, 4, ..., n; butterfly
      t = w * b (t.re = wr*br - wi*bi, t.im = wr*bi + wi*br, each product rounded),
      (a, b) <- (a + t, a - t)
    with w = W_n^(j * n / span) for the j-th pair of a span.  Returns (re, im), fp32 [.., n].
    """
    x = np.asarray(x, dtype=F32)
    rows = x.reshape(-1, x.shape[-1])
    n = rows.shape[-1]
    wr_all, wi_all = twiddles_f32(n)
    re = rows[:, _bitrev(n)].astype(F32)
    im = np.zeros_like(re)
    span = 2
    while span <= n:
        half = span // 2
        step = n // span
        wr = wr_all[np.arange(half) * step]
        wi = wi_all[np.arange(half) * step]
        re = re.reshape(rows.shape[0], n // span, span)
        im = im.reshape(rows.shape[0], n // span, span)
        ar, ai = re[..., :half], im[..., :half]
        br, bi = re[..., half:], im[..., half:]
        tr = (wr * br).astype(F32) - (wi * bi).astype(F32)
        ti = (wr * bi).astype(F32) + (wi * br).astype(F32)
        re = np.concatenate([ar + tr, ar - tr], axis=-1).astype(F32)
        im = np.concatenate([ai + ti, ai - ti], axis=-1).astype(F32)
        span *= 2
    return re.reshape(x.shape), im.reshape(x.shape)


def fold_spectrum(re: np.ndarray, im: np.ndarray):
    """The n/2 complex slots of a real row's spectrum.

    Slot 0 carries the two real bins: (X_0, X_{n/2}); slots f = 1 .. n/2-1 carry X_f.  This
    keeps exactly n reals (n/2 slots), the limit the reply's one-sided-spectrum bit count
    approaches for long rows (12 bits x (n/2 + 1) / n -> 6 bits).
    Returns (a, b) fp32 [.., n/2]: slot real and imaginary parts.
    """
    n = re.shape[-1]
    h = n // 2
    a = re[..., :h].copy()
    b = im[..., :h].copy()
    b[..., 0] = re[..., h]
    return a.astype(F32), b.astype(F32)


def unfold_idft_f64(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Real row from its folded slots, by the inverse DFT written out in fp64.

    x_n = (1/N) sum_{f=0}^{N-1} X_f exp(+2 pi i f n / N) with X_0 = a_0, X_{N/2} = b_0,
    X_f = a_f + i b_f and X_{N-f} = conj(X_f) for 0 < f < N/2.
    """
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    h = a.shape[-1]
    N = 2 * h
    X = np.zeros(a.shape[:-1] + (N,), dtype=np.complex128)
    X[..., 0] = a[..., 0]
    X[..., h] = b[..., 0]
    X[..., 1:h] = a[..., 1:] + 1j * b[..., 1:]
    X[..., h + 1:] = np.conj(X[..., 1:h][..., ::-1])
    nn = np.arange(N)
    E = np.exp(2j * np.pi * np.outer(np.arange(N), nn) / N)  # [f, n]
    x = (X @ E) / N
    return x.real
