"""Pins of the CPU oracle against what the pages and the mathematics fix (no GPU needed).

Each test checks the oracle against something other than itself: hand-worked fixtures, closed
forms printed on the pages, textbook definitions, library routines, brute force in exact
rational arithmetic, or invariants.  A plausible mistake (dropped term, wrong sign or index,
transposed operand, wrong tie rule) fails at least one of them.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import attention as A
from oracle import cache as C
from oracle import nf4 as N
from oracle import quant as Q
from oracle import transforms as T
from oracle.quant import Side

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "packing.json")))


def rng(seed=0):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------- packing
@pytest.mark.parametrize("case", GOLD["pack_bits"])
def test_pack_bits_golden(case):
    got = Q.pack_bits(np.array([case["codes"]]), case["bits"])[0].tolist()
    assert got == case["bytes"]
    back = Q.unpack_bits(np.array([case["bytes"]], dtype=np.uint8), case["bits"], len(case["codes"]))
    assert back[0].tolist() == case["codes"]


def test_pack_trits_golden():
    case = GOLD["pack_trits"][0]
    t = np.array([case["t"]])
    assert Q.pack_trits(t + 1)[0].tolist() == case["bytes"]
    assert (Q.unpack_trits(np.array([case["bytes"]], np.uint8), 7) - 1)[0].tolist() == case["t"]


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 6, 8])
def test_pack_roundtrip(b):
    c = rng(b).integers(0, 2 ** b, size=(7, 128))
    assert (Q.unpack_bits(Q.pack_bits(c, b), b, 128) == c).all()


def test_row_bytes():
    assert Side("int", 4).row_bytes(128) == 64
    assert Side("int", 3).row_bytes(256) == 96
    assert Side("int", 2).row_bytes(256) == 64
    assert Side("ternary", group=8).row_bytes(128) == 26
    assert Side("sign", group=4).row_bytes(128) == 16
    assert Side("polar", 4, 8).row_bytes(128) == 96
    assert Side("cart", 6).row_bytes(128) == 96


# ----------------------------------------------------------------------------- grids: golden
def _rows(x):
    return np.array([x], dtype=np.float16)


@pytest.mark.parametrize("case", GOLD["int_absmax"])
def test_int_absmax_golden(case):
    r = Q.quantize_rows(_rows(case["x"]), Side("int", case["bits"], group=4))
    assert float(r["scales"][0, 0]) == case["d"]
    assert r["q"][0].tolist() == case["q"]
    assert r["bytes"][0].tolist() == [case["byte"]]


def test_int_minmax_golden():
    case = GOLD["int_minmax"][0]
    r = Q.quantize_rows(_rows(case["x"]), Side("int", case["bits"], scale="minmax", group=4))
    assert float(r["scales"][0, 0]) == case["d"] and float(r["zeros"][0, 0]) == case["z"]
    assert r["q"][0].tolist() == case["q"]
    assert r["bytes"][0].tolist() == [case["byte"]]


def test_ternary_golden():
    case = GOLD["ternary"][0]
    r = Q.quantize_rows(_rows(case["x"]), Side("ternary", group=4))
    assert float(r["scales"][0, 0]) == case["s"]
    assert r["q"][0].tolist() == case["t"]
    assert r["bytes"][0].tolist() == [case["byte"]]


def test_nf4_golden():
    case = GOLD["nf4"][0]
    r = Q.quantize_rows(_rows(case["x"]), Side("nf4", group=4))
    assert float(r["scales"][0, 0]) == case["s"]
    assert r["q"][0].tolist() == case["codes"]
    assert r["bytes"][0].tolist() == case["bytes"]


def test_sign_golden():
    case = GOLD["sign"][0]
    r = Q.quantize_rows(_rows(case["x"]), Side("sign", group=4))
    assert float(r["scales"][0, 0]) == case["s"]
    assert r["q"][0].tolist() == case["t"]
    assert r["bytes"][0].tolist() == [case["byte"]]


# ----------------------------------------------------------------------------- grids: brute force
def _nearest_exact(x: float, levels):
    """Index of the nearest level in exact rational arithmetic, ties to the larger level."""
    fx = Fraction(x)
    best = None
    for i, lv in enumerate(levels):
        dist = abs(fx - lv)
        if best is None or dist < best[0] or (dist == best[0] and lv > levels[best[1]]):
            best = (dist, i)
    return best[1]


@pytest.mark.parametrize("b", [2, 3, 4, 8])
def test_int_absmax_nearest_grid_point(b):
    x = (rng(b).standard_normal((6, 64)) * 3).astype(np.float16)
    side = Side("int", b, group=32, rot=0)
    r = Q.quantize_rows(x, side)
    qmin, qmax = -(2 ** (b - 1)), 2 ** (b - 1) - 1
    for i in range(6):
        for gi in range(2):
            d = Fraction(float(r["scales"][i, gi]))
            grp = x[i, gi * 32:(gi + 1) * 32].astype(np.float64)
            # the extreme element maps to the full-range end of the grid
            j = int(np.argmax(np.abs(grp)))
            assert r["q"][i, gi * 32 + j] == qmin
            levels = [k * d for k in range(qmin, qmax + 1)]
            for jj in range(32):
                if d == 0:
                    continue
                # levels are in k order; nearest in value with ties to larger code = larger k
                fx = Fraction(float(grp[jj]))
                dists = [abs(fx - lv) for lv in levels]
                m = min(dists)
                want = max(k for k, dd in zip(range(qmin, qmax + 1), dists) if dd == m)
                assert r["q"][i, gi * 32 + jj] == want


@pytest.mark.parametrize("b", [2, 3, 4])
def test_int_minmax_nearest_grid_point(b):
    x = (rng(10 + b).standard_normal((5, 64)) * 2 + 0.7).astype(np.float16)
    r = Q.quantize_rows(x, Side("int", b, scale="minmax", group=32))
    for i in range(5):
        for gi in range(2):
            d = Fraction(float(r["scales"][i, gi]))
            z = Fraction(float(r["zeros"][i, gi]))
            levels = [z + k * d for k in range(2 ** b)]
            for jj in range(32):
                want = _nearest_exact(float(x[i, gi * 32 + jj]), levels)
                assert r["q"][i, gi * 32 + jj] == want


def test_minmax_zero_point_signed_zero():
    """IEEE 754 minimum orders -0 below +0: a group whose smallest value is zero stores z = -0
    exactly when it holds a -0, +0 otherwise (the sign bit is all that differs)."""
    x = np.zeros((3, 8), dtype=np.float16)
    x[0, 5] = np.float16(-0.0)          # +0 ... -0 ... : min is -0
    x[1, :] = np.float16(-0.0)          # all -0
    x[2, 3] = np.float16(1.5)           # +0 and a positive value: min is +0
    r = Q.quantize_rows(x, Side("int", 4, scale="minmax", group=8))
    assert r["zeros"][:, 0].view(np.uint16).tolist() == [0x8000, 0x8000, 0x0000]
    assert r["scales"][:, 0].view(np.uint16).tolist()[:2] == [0x0000, 0x0000]
    assert r["scales"][2, 0] == np.float16(0.1)  # fp16(1.5 / 15)


def test_nf4_nearest_level():
    x = (rng(3).standard_normal((4, 128))).astype(np.float16)
    r = Q.quantize_rows(x, Side("nf4", group=64))
    L = [Fraction(float(v)) for v in N.nf4_levels()]
    for i in range(4):
        for gi in range(2):
            s = Fraction(float(r["scales"][i, gi]))
            for jj in range(64):
                want = _nearest_exact(float(x[i, gi * 64 + jj]), [lv * s for lv in L])
                assert r["q"][i, gi * 64 + jj] == want


def test_ternary_nearest_level():
    x = (rng(4).standard_normal((4, 64))).astype(np.float16)
    r = Q.quantize_rows(x, Side("ternary", group=8))
    for i in range(4):
        for gi in range(8):
            s = Fraction(float(r["scales"][i, gi]))
            for jj in range(8):
                want = _nearest_exact(float(x[i, gi * 8 + jj]), [-s, Fraction(0), s]) - 1
                assert r["q"][i, gi * 8 + jj] == want


def test_round_half_up_exact_adversarial():
    """Exact ties and values one fp32 ulp either side of a tie."""
    d = np.float16(0.1).astype(np.float64)
    xs, want = [], []
    for k in range(-8, 8):
        tie = (Fraction(2 * k + 1, 2)) * Fraction(float(d))
        t32 = np.float32(float(tie))
        for v in (np.nextafter(t32, np.float32(-1e9)), t32, np.nextafter(t32, np.float32(1e9))):
            xs.append(float(v))
            r = Fraction(float(v)) / Fraction(float(d)) + Fraction(1, 2)
            want.append(math.floor(r))
    got = Q.round_half_up_exact(np.array(xs), d)
    assert got.tolist() == want


def test_roundtrip_error_bound():
    """|x - x_hat| <= |d|/2 inside the grid hull (the ggml grid clamps one side)."""
    x = (rng(5).standard_normal((16, 128)) * 4).astype(np.float16)
    for b in (2, 3, 4):
        side = Side("int", b, group=32)
        r = Q.quantize_rows(x, side)
        d = np.repeat(r["scales"].astype(np.float64), 32, axis=1)
        inside = (r["q"] > -(2 ** (b - 1))) & (r["q"] < 2 ** (b - 1) - 1)
        err = np.abs(x.astype(np.float64) - r["exact"])
        assert (err[inside] <= np.abs(d[inside]) / 2 + 1e-12).all()
        assert (err <= np.abs(d) + 1e-12).all()


def test_level_sets():
    """Grids named on the pages: int2 -2..1 ("E22L"), ternary {-1,0,1}, sign {-1,1}."""
    x = (rng(6).standard_normal((64, 128)) * 3).astype(np.float16)
    assert set(np.unique(Q.quantize_rows(x, Side("int", 2, group=128))["q"])) == {-2, -1, 0, 1}
    assert set(np.unique(Q.quantize_rows(x, Side("int", 4, group=32))["q"])) <= set(range(-8, 8))
    assert set(np.unique(Q.quantize_rows(x, Side("ternary", group=8))["q"])) == {-1, 0, 1}
    assert set(np.unique(Q.quantize_rows(x, Side("sign", group=4))["q"])) == {-1, 1}


def test_sign_scale_least_squares_and_page_error():
    """s = mean|x| minimises sum (x - s t)^2 for t = sign(x); on Gaussian rows the relative
    error norm tends to sqrt(1 - 2/pi) = 0.603, inside the 0.54-0.63 K/V rel-err that post 6
    ("Debunk audit") reports for sign KV."""
    x = rng(7).standard_normal((256, 128)).astype(np.float16)
    side = Side("sign", group=128)
    r = Q.quantize_rows(x, side)
    t = np.where(x >= 0, 1.0, -1.0)
    s_ls = (x.astype(np.float64) * t).sum(axis=1) / 128.0
    assert np.allclose(r["scales"][:, 0].astype(np.float64), s_ls, rtol=1e-3)
    rel = math.sqrt(A.rel_sq_error(x, r["exact"]))
    assert abs(rel - math.sqrt(1 - 2 / math.pi)) < 0.01
    assert 0.54 <= rel <= 0.63


# ----------------------------------------------------------------------------- NF4 construction
def test_nf4_construction_properties():
    L = N.nf4_levels()
    assert len(L) == 16 and (np.diff(L) > 0).all()
    assert L[0] == -1.0 and L[-1] == 1.0 and 0.0 in L
    assert (L < 0).sum() == 7 and (L > 0).sum() == 8
    # quantile spacing, checked through the normal CDF (erf), not the inverse used to build it
    top = N.nf4_levels_f64()
    z = statistics_inv(N.DELTA)
    phi = lambda v: 0.5 * (1 + math.erf(v / math.sqrt(2)))
    pos = sorted(v for v in top if v > 0)
    neg = sorted(-v for v in top if v < 0)
    assert np.allclose([phi(v * z) for v in pos], np.linspace(N.DELTA, 0.5, 9)[:-1][::-1], atol=1e-12)
    assert np.allclose([phi(v * z) for v in neg], np.linspace(N.DELTA, 0.5, 8)[:-1][::-1], atol=1e-12)
    # fp16 levels: midpoints times any fp16 scale are exact in fp32 (thresholds are exact)
    mids = (L[:-1] + L[1:]) / 2
    for s in np.float16([0.1, 3.7, 1000.0, 6e-5]).astype(np.float64):
        assert ((mids * s).astype(np.float32).astype(np.float64) == mids * s).all()


def statistics_inv(p):
    import statistics
    return statistics.NormalDist().inv_cdf(p)


# ----------------------------------------------------------------------------- Hadamard
@pytest.mark.parametrize("n", [128, 256])
def test_hadamard_matrix(n):
    H = T.sylvester(n)
    ii, jj = np.meshgrid(np.arange(n), np.arange(n), indexing="ij")
    pc = np.vectorize(lambda a: bin(a).count("1"))(ii & jj)
    assert (H == (-1.0) ** pc).all()  # Sylvester = (-1)^popcount(i & j)
    assert np.array_equal(H @ H.T, n * np.eye(n))


@pytest.mark.parametrize("n", [128, 256])
def test_fwht_matches_matrix_and_norm(n):
    x = rng(n).standard_normal((5, n)).astype(np.float32)
    y = T.fwht_f32(x, n).astype(np.float64)
    ref = x.astype(np.float64) @ (T.sylvester(n) / math.sqrt(n)).T
    assert np.allclose(y, ref, rtol=0, atol=1e-5 * np.abs(x).max())
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x.astype(np.float64), axis=1), rtol=1e-6)
    e = np.eye(n, dtype=np.float32)[3:4]
    col = T.fwht_f32(e, n)[0].astype(np.float64)
    assert set(np.abs(col).tolist()) == {float(T.hadamard_scale(n))}
    assert np.allclose(T.hadamard_inverse_f64(y, n), x, atol=1e-5)


def test_hadamard_scale_is_nearest_fp32():
    for n in (128, 256):
        r = T.hadamard_scale(n)
        exact = 1 / math.sqrt(n)
        lo = np.nextafter(r, np.float32(0))
        hi = np.nextafter(r, np.float32(1))
        assert abs(float(r) - exact) <= abs(float(lo) - exact)
        assert abs(float(r) - exact) <= abs(float(hi) - exact)


def test_fwht_block_diagonal():
    x = rng(9).standard_normal((3, 256)).astype(np.float32)
    y = T.fwht_f32(x, 128)
    assert np.array_equal(y[:, :128], T.fwht_f32(x[:, :128], 128))
    assert np.array_equal(y[:, 128:], T.fwht_f32(x[:, 128:], 128))


# ----------------------------------------------------------------------------- FFT
def test_dft_matches_definition_and_library():
    x = rng(11).standard_normal((4, 128)).astype(np.float32)
    re, im = T.dft_dit_f32(x)
    n = np.arange(128)
    W = np.exp(-2j * np.pi * np.outer(n, n) / 128)
    ref = x.astype(np.float64) @ W.T
    scale = np.linalg.norm(x.astype(np.float64))
    assert np.abs(re - ref.real).max() < 1e-5 * scale
    assert np.abs(im - ref.imag).max() < 1e-5 * scale
    lib = np.fft.fft(x.astype(np.float64), axis=-1)
    assert np.abs((re + 1j * im) - lib).max() < 1e-5 * scale
    # Hermitian symmetry of a real row's spectrum (the reply: "the FFT is Hermitian-symmetric")
    X = re.astype(np.float64) + 1j * im.astype(np.float64)
    assert np.abs(X[:, 1:] - np.conj(X[:, 1:][:, ::-1])).max() < 1e-5 * scale
    # Parseval
    assert np.allclose((np.abs(X) ** 2).sum(axis=1) / 128, (x.astype(np.float64) ** 2).sum(axis=1), rtol=1e-5)


def test_fold_unfold_roundtrip():
    x = rng(12).standard_normal((3, 128)).astype(np.float32)
    a, b = T.fold_spectrum(*T.dft_dit_f32(x))
    assert a.shape == (3, 64)
    assert np.allclose(T.unfold_idft_f64(a, b), x, atol=1e-5)


def test_polar_exact_phase_reduces_to_magnitude_error():
    """The reply's first control (quantize only the spectrum magnitudes, keep the phase
    exact): the reconstruction error is then the magnitude rounding alone."""
    x = rng(13).standard_normal((8, 128)).astype(np.float16)
    bm = 4
    mc, pc, s = Q.quant_polar(x.astype(np.float32), bm, 8)
    a, b = T.fold_spectrum(*T.dft_dit_f32(x.astype(np.float32)))
    ang = np.arctan2(b.astype(np.float64), a.astype(np.float64))
    m = mc * s[:, None]
    xr = T.unfold_idft_f64(m * np.cos(ang), m * np.sin(ang))
    mag = np.hypot(a.astype(np.float64), b.astype(np.float64))
    assert (np.abs(m - mag) <= s[:, None] / 2 + 1e-6).all()
    # error energy equals the magnitude error energy through Parseval on the folded slots
    e_slot = (m - mag) ** 2
    e_slot[:, 1:] *= 2
    assert np.allclose(((xr - x.astype(np.float64)) ** 2).sum(axis=1), e_slot.sum(axis=1) / 128, rtol=1e-3, atol=1e-9)


def test_polar_phase_codes_uniform_grid():
    x = rng(14).standard_normal((32, 128)).astype(np.float16)
    for bm, bp in ((4, 8), (5, 7), (6, 6), (7, 5), (8, 4)):
        r = Q.quantize_rows(x, Side("polar", bm, bp))
        mc, pc = r["q"][:, :64], r["q"][:, 64:]
        assert mc.max() == 2 ** bm - 1 and mc.min() >= 0
        assert pc.min() >= 0 and pc.max() < 2 ** bp
        a, b = T.fold_spectrum(*T.dft_dit_f32(x.astype(np.float32)))
        ang = np.arctan2(b.astype(np.float64), a.astype(np.float64))
        phi = Q.phase_angles_f64(bp)[pc]
        dphi = np.angle(np.exp(1j * (ang - phi)))
        assert np.abs(dphi).max() <= math.pi / 2 ** bp + 1e-9


# ----------------------------------------------------------------------------- effective bits
def test_effective_bits_closed_forms():
    D = 256
    b = Q.bits_per_value
    # "E21W" "Result": 3.5 bits for 3-bit at group 32, 4.5 for 4-bit
    assert b(Side("int", 3, group=32), D) == 3.5
    assert b(Side("int", 4, group=32), D) == 4.5
    # "E22L" "What I tested": A 3.125, B 3.25, C 3.5, D 3.625 (averaged over K and V)
    avg = lambda k, v: (b(k, D) + b(v, D)) / 2
    assert avg(Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)) == 3.125
    assert avg(Side("int", 4, group=64, rot=256), Side("int", 2, group=64, rot=256)) == 3.25
    assert avg(Side("int", 4, group=32), Side("int", 2, group=32, rot=256)) == 3.5
    assert avg(Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256)) == 3.625
    # post 6: NF4/g64 at 4.25 b, "NF4-K + int4-g64 V (4.25b)"
    assert b(Side("nf4", group=64), 128) == 4.25
    assert avg(Side("nf4", group=64), Side("int", 4, group=64)) == 4.25
    # "E21W": the 3.19-bit allocation (K 2 bits in 2 layers, V 4 bits in 3 layers, 3 bits
    # elsewhere, groups of 128, 8 layers)
    Kb = [2, 2] + [3] * 6
    Vb = [4] * 3 + [3] * 5
    tot = sum(b(Side("int", k, group=128), D) for k in Kb) + sum(b(Side("int", v, group=128), D) for v in Vb)
    assert tot / 16 == 3.1875 and round(tot / 16, 2) == 3.19
    # the reply: (4 + 8) * 33 / 64 = 6.1875 payload bits at head_dim 64 with 33 one-sided
    # bins; the folded 32-slot layout reaches the 6-bit asymptote, +16/128 for the scale at 128
    assert (4 + 8) * (64 // 2 + 1) / 64 == 6.1875
    assert Side("polar", 4, 8).row_bytes(64) * 8 / 64 == 6.0
    for bm, bp in ((4, 8), (5, 7), (6, 6), (7, 5), (8, 4)):
        assert b(Side("polar", bm, bp), 128) == 6.125
    assert b(Side("cart", 6), 128) == 6.125
    assert b(Side("int", 6, group=128, rot=128), 128) == 6.125


def test_per_layer_spec_follows_the_allocation():
    """"E21W" "Result": the rotated g128 allocation with 2-bit K in layers 2 and 7, 4-bit V in
    layers 1, 3 and 4 and 3 bits elsewhere averages 3.19 bits (exactly 3.1875 with the scales);
    each layer's unit is quantized with that layer's own grid."""
    D = 256
    side = lambda b: Side("int", b, group=128, rot=256)
    lk = tuple(side(2 if l in (2, 7) else 3) for l in range(8))
    lv = tuple(side(4 if l in (1, 3, 4) else 3) for l in range(8))
    s = C.Spec(8, 1, 1, 1, D, side(4), side(4), layer_k=lk, layer_v=lv)
    assert C.effective_bits(s, 6000) == 3.1875
    x = (rng(21).standard_normal((3, D))).astype(np.float16)
    for l, (kb, vb) in enumerate(zip((3, 3, 2, 3, 3, 3, 3, 2), (3, 4, 3, 4, 4, 3, 3, 3))):
        kq, vq = C.quantize_unit(s, x, x, None, layer=l)
        assert kq["bytes"].shape == (3, D * kb // 8) and vq["bytes"].shape == (3, D * vb // 8)
        assert np.array_equal(kq["bytes"], Q.quantize_rows(x, side(kb))["bytes"])


def test_effective_bits_anchor_layer():
    """Post 6 "Corrected semantics" gives 4.69 effective bits for NF4 g64 with layer-0-only
    anchors, which matches one fully fp16 layer out of 26 (Gemma-3-1B depth): 4.25 + 11.75/26."""
    s = C.Spec(26, 1, 1, 4, 256, Side("nf4", group=64), Side("nf4", group=64),
               frozenset({0}), "all", 0)
    assert abs(C.effective_bits(s, 4096) - 4.69) < 0.02


def test_anchor_rules():
    s = C.Spec(4, 1, 1, 1, 128, Side(), Side(), frozenset({0, 2}), "first_n", 48)
    t = np.arange(100)
    assert C.anchored(s, 0, t, 100).sum() == 48 and C.anchored(s, 1, t, 100).sum() == 0
    s.anchor_rule, s.anchor_n = "window", 64
    m = C.anchored(s, 2, t, 100)
    assert m.sum() == 64 and m[36:].all() and not m[:36].any()
    s.anchor_rule = "all"
    assert C.anchored(s, 0, t, 100).all()


# ----------------------------------------------------------------------------- attention
def _brute_attention(q, K, V, kv_len):
    """Pure-Python textbook softmax attention on tiny shapes."""
    Hq, D = len(q), len(q[0])
    Hkv = len(K)
    G = Hq // Hkv
    out = []
    for h in range(Hq):
        j = h // G
        s = [sum(q[h][c] * K[j][t][c] for c in range(D)) / math.sqrt(D) for t in range(kv_len)]
        m = max(s)
        e = [math.exp(v - m) for v in s]
        z = sum(e)
        out.append([sum(e[t] / z * V[j][t][c] for t in range(kv_len)) for c in range(D)])
    return out


def test_attention_fp16_format_is_textbook():
    r = rng(20)
    Hkv, Hq, D, Tn = 2, 4, 16, 40
    K = r.standard_normal((Hkv, Tn, D)).astype(np.float16)
    V = r.standard_normal((Hkv, Tn, D)).astype(np.float16)
    q = r.standard_normal((Hq, D)).astype(np.float16)
    side = Side("fp16")
    Kh = np.stack([Q.to_original_f64(Q.quantize_rows(K[j], side)["exact"], side) for j in range(Hkv)])
    Vh = np.stack([Q.to_original_f64(Q.quantize_rows(V[j], side)["exact"], side) for j in range(Hkv)])
    o, lse, p = A.attention(q, Kh, Vh, 33)
    ref = _brute_attention(q.astype(float).tolist(), K.astype(float).tolist(), V.astype(float).tolist(), 33)
    assert np.allclose(o, ref, atol=1e-12)
    assert np.allclose(p.sum(axis=1), 1.0)


def test_attention_split_merge_equals_one_pass():
    r = rng(21)
    K = r.standard_normal((1, 50, 8))
    V = r.standard_normal((1, 50, 8))
    q = r.standard_normal((2, 8))
    o, lse, _ = A.attention(q, K, V, 50)
    o1, l1, _ = A.attention(q, K[:, :20], V[:, :20], 20)
    o2, l2, _ = A.attention(q, K[:, 20:], V[:, 20:], 30)
    M = np.maximum(l1, l2)
    w1, w2 = np.exp(l1 - M), np.exp(l2 - M)
    om = (w1[:, None] * o1 + w2[:, None] * o2) / (w1 + w2)[:, None]
    assert np.allclose(om, o) and np.allclose(M + np.log(w1 + w2), lse)


def test_metrics_closed_forms():
    p = np.array([0.5, 0.5])
    qd = np.array([0.25, 0.75])
    assert A.kl(p, p) == 0.0
    assert abs(A.kl(p, qd) - (0.5 * math.log(2) + 0.5 * math.log(2 / 3))) < 1e-15
    assert A.rel_l2([3.0, 4.0], [3.0, 4.0]) == 0.0
    assert abs(A.rel_l2([3.0, 5.0], [3.0, 4.0]) - 0.2) < 1e-15
    assert abs(A.rel_sq_error([1.0, 1.0], [1.0, 0.0]) - 0.5) < 1e-15


def test_channel_scale_then_rotation_order():
    """Variant D of "E21W": per-channel scale first, then rotation; dequant rotates back and
    multiplies the scale back in."""
    r = rng(22)
    x = (r.standard_normal((4, 256)) * 3).astype(np.float16)
    c = (np.abs(r.standard_normal(256)) + 0.5).astype(np.float16)
    side = Side("int", 8, group=32, rot=256, chan_scale=True)
    out = Q.quantize_rows(x, side, np.broadcast_to(c, x.shape))
    xo = Q.to_original_f64(out["exact"], side, np.broadcast_to(c, x.shape))
    assert A.rel_sq_error(x, xo) < 1e-4
    y = T.fwht_f32(x.astype(np.float32) / c.astype(np.float32), 256)
    assert np.array_equal(Q.transform_rows(x, side, np.broadcast_to(c, x.shape)), y)


# ----------------------------------------------------------------------------- anchors in reconstruction
def _rot_int8_bound(x16, side, out):
    """Per-row bound on the original-domain error of a rotated absmax int grid: the rotation is
    orthonormal, so the row error norm equals the stored-domain one, at most |d|/2 per element
    inside the grid hull and |d| where the positive side clamps."""
    d = np.repeat(np.abs(out["scales"].astype(np.float64)), side.group, axis=1)
    return np.sqrt((d ** 2).sum(axis=1))


@pytest.mark.parametrize("rule,n", [("first_n", 48), ("window", 40), ("all", 0)])
def test_reconstruct_unit_anchor_substitution(rule, n):
    """Post 6 "Corrected semantics": an anchored row is attended as its original fp16 row --
    K's own row for keys, V's for values, unrotated -- and every other row is the dequantized
    row in the original domain.  Keys and values are drawn independently, so substituting the
    wrong side, the rotated row, or the wrong token set cannot pass."""
    r = rng(31)
    T, D = 120, 128
    side = Side("int", 8, group=32, rot=128)
    spec = C.Spec(1, 1, 1, 1, D, side, side, frozenset({0}), rule, n)
    K16 = (r.standard_normal((T, D)) * 2).astype(np.float16)
    V16 = (r.standard_normal((T, D)) * 3 + 1).astype(np.float16)
    seq_len = 100  # a window protects the last n stored tokens, not the last rows of the buffer
    kq, vq = C.quantize_unit(spec, K16, V16)
    Kh, Vh = C.reconstruct_unit(spec, 0, K16, V16, kq, vq, seq_len)
    t = np.arange(T)
    want = {"first_n": t < n, "window": (t >= seq_len - n) & (t < seq_len), "all": t < seq_len}[rule]
    assert want.sum() > 0
    for Xh, X16, q in ((Kh, K16, kq), (Vh, V16, vq)):
        x = X16.astype(np.float64)
        assert np.array_equal(Xh[want], x[want])              # exact original rows
        err = np.sqrt(((Xh - x) ** 2).sum(axis=1))
        bound = _rot_int8_bound(X16, side, q)
        assert (err[~want] <= bound[~want] * (1 + 1e-6) + 1e-9).all()  # dequantized, unrotated
        assert (err[~want] > 0).all()                        # and really the quantized row
    # a layer outside the anchor set is quantized everywhere
    spec2 = C.Spec(2, 1, 1, 1, D, side, side, frozenset({0}), rule, n)
    Kh1, Vh1 = C.reconstruct_unit(spec2, 1, K16, V16, kq, vq, seq_len)
    assert (np.sqrt(((Kh1 - K16.astype(np.float64)) ** 2).sum(axis=1)) > 0).all()


# ----------------------------------------------------------------------------- composite rFFT reconstruction
def _folded_reference(x16):
    """Folded slots (X_0, X_64 | X_f) of each row from numpy's FFT in fp64 (independent of the
    oracle's fp32 DIT and fold)."""
    X = np.fft.rfft(x16.astype(np.float64), axis=-1)  # 65 bins
    a = X[:, :64].real.copy()
    b = X[:, :64].imag.copy()
    b[:, 0] = X[:, 64].real
    return a, b


def _parseval_folded(ea, eb):
    """Energy of the real row whose folded-slot error is (ea, eb), N = 128."""
    w = np.full(ea.shape, 2.0)
    w[:, 0] = 1.0
    return (w * (ea ** 2 + eb ** 2)).sum(axis=1) / 128.0


@pytest.mark.parametrize("bits", [6, 8])
def test_cartesian_reconstruction_matches_parseval(bits):
    """The reply's Cartesian control: the stored reals are the folded spectrum's (re, im) pairs on
    a signed grid, and the inverse transform's row error is the Parseval-weighted stored error.
    Against numpy's FFT: a swapped (re, im) interleave, a misplaced Nyquist bin or a missing
    factor 2 on the one-sided bins fails the equality."""
    x16 = (rng(32).standard_normal((16, 128)) * 3).astype(np.float16)
    side = Side("cart", bits)
    out = Q.quantize_rows(x16, side)
    a_ref, b_ref = _folded_reference(x16)
    y = out["exact"]
    ea, eb = y[:, 0::2] - a_ref, y[:, 1::2] - b_ref
    d = np.abs(out["scales"].astype(np.float64))  # [R, 1]
    assert (np.abs(ea) <= d * (1 + 1e-3)).all() and (np.abs(eb) <= d * (1 + 1e-3)).all()
    xr = Q.to_original_f64(y, side)
    got = ((xr - x16.astype(np.float64)) ** 2).sum(axis=1)
    assert np.allclose(got, _parseval_folded(ea, eb), rtol=1e-6, atol=1e-10)
    assert (got <= (254 / 128) * d[:, 0] ** 2 * (1 + 1e-3)).all()


@pytest.mark.parametrize("bm,bp", [(4, 8), (5, 7), (6, 6), (7, 5), (8, 4)])
def test_polar_reconstruction_within_magnitude_and_phase_bound(bm, bp):
    """The reply's polar codec: per slot the reconstruction error is at most the magnitude step
    error plus the chord of the phase step, |dm| + m^ * pi / 2^bp; through Parseval the row error
    is bounded by those per-slot bounds.  The reference spectrum is numpy's, so the composite
    (DIT FFT, fold, codes, cos/sin, unfold, inverse DFT) is checked end to end."""
    x16 = (rng(33).standard_normal((16, 128)) * 2).astype(np.float16)
    side = Side("polar", bm, bp)
    out = Q.quantize_rows(x16, side)
    a_ref, b_ref = _folded_reference(x16)
    mag = np.hypot(a_ref, b_ref)
    s = out["scales"].astype(np.float64)  # [R, 1]
    mh = out["q"][:, :64] * s
    dm = np.abs(mh - mag)
    assert (dm <= s / 2 + 1e-3 * mag.max(axis=1, keepdims=True)).all()
    slot_bound = dm + mh * (math.pi / 2 ** bp) + 1e-6 * mag.max(axis=1, keepdims=True)
    y = out["exact"]
    ea, eb = y[:, 0::2] - a_ref, y[:, 1::2] - b_ref
    assert (np.hypot(ea, eb) <= slot_bound).all()
    xr = Q.to_original_f64(y, side)
    got = ((xr - x16.astype(np.float64)) ** 2).sum(axis=1)
    assert np.allclose(got, _parseval_folded(ea, eb), rtol=1e-6, atol=1e-10)
    w = np.full(slot_bound.shape, 2.0)
    w[:, 0] = 1.0
    assert (got <= (w * slot_bound ** 2).sum(axis=1) / 128.0).all()


# ----------------------------------------------------------------------------- value grids after E22L
from oracle import lloyd as LM

# J. Max, "Quantizing for minimum distortion" (1960), Table I, the Gaussian optimum (positive
# half, 4 decimals) and its mean squared error (to the precision compared) -- a published table,
# independent of the iteration.
MAX_1960 = {2: ([0.4528, 1.5104], 0.1175), 3: ([0.2451, 0.7560, 1.3439, 2.1520], 0.03455),
            4: ([0.1284, 0.3881, 0.6568, 0.9424, 1.2562, 1.6180, 2.0690, 2.7326], 0.00950)}


def _gauss_mse(levels):
    """Expected (X - nearest level)^2 for X ~ N(0, 1), by midpoint-rule integration."""
    x = np.linspace(-12, 12, 2_400_001)
    w = np.exp(-0.5 * x * x) / math.sqrt(2 * math.pi) * (x[1] - x[0])
    idx = np.searchsorted((levels[:-1] + levels[1:]) / 2.0, x)
    return float((w * (x - levels[idx]) ** 2).sum())


@pytest.mark.parametrize("b", [2, 3, 4])
def test_lloyd_max_levels(b):
    """Gaussian Lloyd-Max levels ("E22L" "Result": the next value grid to test): Max's table, the
    two optimality conditions (midpoint thresholds, centroid levels) at the fixed point, odd
    symmetry, and the table's distortion."""
    lv = LM.lloyd_max_levels_f64(b)
    half, mse = MAX_1960[b]
    assert np.allclose(lv[2 ** (b - 1):], half, atol=6e-5)
    assert np.allclose(lv, -lv[::-1], atol=1e-12)
    assert np.abs(LM.centroids((lv[:-1] + lv[1:]) / 2) - lv).max() < 1e-10
    assert abs(_gauss_mse(lv) - mse) < 1e-3 * mse
    # fp16 storage: every level is an fp16 value within half an fp16 ulp of the optimum
    l16 = LM.lloyd_max_levels(b)
    assert np.array_equal(l16, l16.astype(np.float16).astype(np.float64))
    assert np.all(np.abs(l16 - lv) <= np.abs(lv) * 2 ** -11)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_lloyd_nearest_level(b):
    x = (rng(40 + b).standard_normal((4, 64)) * 1.7).astype(np.float16)
    x[0, :8] = 0.0
    r = Q.quantize_rows(x, Side("lloyd", b, group=16))
    L = [Fraction(float(v)) for v in LM.lloyd_max_levels(b)]
    for i in range(4):
        for gi in range(4):
            grp = x[i, gi * 16:(gi + 1) * 16].astype(np.float64)
            # the scale is the group RMS (fp32 sum of rounded squares in channel order)
            acc = np.float32(0)
            for v in grp.astype(np.float32):
                acc = np.float32(acc + np.float32(v * v))
            s = np.float16(np.sqrt(np.float32(acc / np.float32(16))))
            assert r["scales"][i, gi] == s
            S = Fraction(float(s))
            for jj in range(16):
                want = _nearest_exact(float(grp[jj]), [lv * S for lv in L]) if S != 0 else 2 ** (b - 1)
                assert r["q"][i, gi * 16 + jj] == want
    assert set(np.unique(r["q"])) <= set(range(2 ** b))


@pytest.mark.parametrize("b", [2, 3, 4])
def test_symmetric_grid_nearest_level(b):
    """The symmetric b-bit grid (levels +-(k + 1/2) d, "E22L" "Result"): nearest level in exact
    arithmetic with ties up, the outermost level at the group's largest magnitude, and the level
    set symmetric about zero (no zero level)."""
    x = (rng(50 + b).standard_normal((4, 64)) * 2.3).astype(np.float16)
    x[1, :16] = 0.0
    # exact ties: multiples of d where d comes out exact (m = 2^(b-1) - 1/2 times a power of two)
    x[2, 32:48] = np.array([(2 ** (b - 1) - 0.5) * 0.25] + [0.25 * k for k in range(-7, 8)], dtype=np.float16)
    r = Q.quantize_rows(x, Side("int", b, scale="sym", group=16))
    nlev = 2 ** b
    for i in range(4):
        for gi in range(4):
            grp = x[i, gi * 16:(gi + 1) * 16].astype(np.float64)
            d = Fraction(float(r["scales"][i, gi]))
            m = np.abs(grp).max()
            assert float(r["scales"][i, gi]) == float(np.float16(np.float32(m) / np.float32(2 ** (b - 1) - 0.5)))
            levels = [(Fraction(2 * q - (nlev - 1), 2)) * d for q in range(nlev)]
            for jj in range(16):
                want = _nearest_exact(float(grp[jj]), levels) if d != 0 else 2 ** (b - 1)
                assert r["q"][i, gi * 16 + jj] == want
    lv = sorted({float(v) for v in (r["q"] - (nlev - 1) / 2.0).ravel()})
    assert all(abs(v) >= 0.5 for v in lv) and max(lv) <= (nlev - 1) / 2.0
    assert set(np.unique(Q.quantize_rows(x, Side("int", 2, scale="sym", group=64))["q"] - 1.5)) == {-1.5, -0.5, 0.5, 1.5}


def test_key_mean_is_the_exact_mean_rounded():
    """The key mean (llama.cpp #21385, the comment on subtracting a shared per-head key mean): the
    exact rational mean of the fp16 keys, through fp64, rounded to fp16."""
    K = (rng(60).standard_normal((777, 64)) * 3 + 5).astype(np.float16)
    K[0] *= 50
    mu = C.key_mean(K)
    for j in range(64):
        S = sum(Fraction(float(v)) for v in K[:, j])
        assert mu[j] == np.float16(float(S / 777))


def test_key_mean_subtraction_restores_and_helps():
    """Keys with a large shared per-head mean (the comment: about half of the key energy): the
    quantized rows are the residual k - mu, the restored row is residual + mu (within the grid's
    error bound), and at 3 bits the K error is far below the same grid without the subtraction."""
    r = rng(61)
    n_tok, D = 300, 128
    mean = r.standard_normal(D) * 4.0
    K = (mean[None, :] + r.standard_normal((n_tok, D))).astype(np.float16)
    V = r.standard_normal((n_tok, D)).astype(np.float16)
    k_sub = Side("int", 3, group=32, rot=128, mean_sub=True)
    k_raw = Side("int", 3, group=32, rot=128)
    v = Side("int", 4, group=32)
    errs = {}
    for name, ks in (("sub", k_sub), ("raw", k_raw)):
        spec = C.Spec(1, 1, 1, 1, D, ks, v)
        kq, vq = C.quantize_unit(spec, K, V, first_rows=200)
        Kh, _ = C.reconstruct_unit(spec, 0, K, V, kq, vq, n_tok)
        if name == "sub":
            mu = C.key_mean(K[:200])  # the first append's 200 rows
            assert np.array_equal(kq["mu"], mu)
            # the grid sees the fp32 residual k - mu, rotated after the subtraction
            resid = (K.astype(np.float32) - mu.astype(np.float32)).astype(np.float32)
            q, d = Q.quant_int_absmax(T.fwht_f32(resid, 128), 3, 32)
            assert np.array_equal(kq["q"], q) and np.array_equal(kq["scales"].astype(np.float64), d)
            # restored: the residual's reconstruction plus mu
            assert np.allclose(Kh - mu.astype(np.float64), Q.to_original_f64(kq["exact"], k_raw), rtol=0, atol=1e-12)
        errs[name] = A.rel_sq_error(K, Kh)
    assert errs["sub"] < 0.25 * errs["raw"]
    # bits: one fp16 mean vector per (sequence, kv-head), like a channel-scale vector
    s = C.Spec(1, 1, 1, 1, D, k_sub, v)
    assert C.effective_bits(s, 1000) == pytest.approx((Q.bits_per_value(k_sub, D) + 16 / 1000 + Q.bits_per_value(v, D)) / 2)


@pytest.mark.parametrize("abits", [8, 4])
def test_int_anchor_rows(abits):
    """Post 6, "The winning recipe" item 4 (the anchor-precision dial, fp16 -> int8 -> int4): an
    anchored row is attended as the original row on a b-bit grid in groups of 32 (one fp16 scale
    each), within that grid's error bound, far closer than the ternary rows around it, and the
    effective bits count b + 16/32 per anchored value."""
    r = rng(70 + abits)
    n_tok, D = 100, 128
    side = Side("ternary", group=8)
    K16 = (r.standard_normal((n_tok, D)) * 2).astype(np.float16)
    V16 = (r.standard_normal((n_tok, D)) * 3).astype(np.float16)
    spec = C.Spec(1, 1, 1, 1, D, side, side, frozenset({0}), "first_n", 30, anchor_bits=abits)
    kq, vq = C.quantize_unit(spec, K16, V16)
    Kh, Vh = C.reconstruct_unit(spec, 0, K16, V16, kq, vq, n_tok)
    for Xh, X16 in ((Kh, K16), (Vh, V16)):
        x = X16.astype(np.float64)
        a, rest = x[:30], x[30:]
        g = a.reshape(30, D // 32, 32)
        d = np.abs(g).max(axis=-1, keepdims=True) / 2 ** (abits - 1)    # |d| before fp16 rounding
        err = np.abs(Xh[:30].reshape(30, D // 32, 32) - g)
        assert (err <= d * (1 + 2 ** -10) + 1e-12).all()
        assert (Xh[:30] != x[:30]).any()                                   # not the fp16 row itself
        assert A.rel_sq_error(a, Xh[:30]) < 0.1 * A.rel_sq_error(rest, Xh[30:])
        # the grid's level set: code values x / d are integers in [-2^(b-1), 2^(b-1) - 1]
        dd = np.repeat(Q.quantize_rows(X16[:30], Side("int", abits, group=32))["scales"].astype(np.float64), 32, axis=1)
        lv = Xh[:30] / np.where(dd == 0, 1, dd)
        assert np.allclose(lv, np.round(lv)) and lv.min() >= -(2 ** (abits - 1)) and lv.max() <= 2 ** (abits - 1) - 1
    eb = C.effective_bits(spec, n_tok)
    base = Q.bits_per_value(side, D)
    assert eb == pytest.approx((70 * base + 30 * (abits + 16 / 32)) / n_tok)


# ----------------------------------------------------------------------------- sorted groups
@pytest.mark.parametrize("D,b,g", [(128, 2, 8), (128, 2, 4), (64, 3, 8), (256, 2, 16)])
def test_sorted_groups(D, b, g):
    """Post 6, "The winning recipe" item 1: rows sorted descending, consecutive groups quantized
    (the outliers land together in one wide group).  The stored ranks form a permutation that orders the row
    descending (equal values in channel order); every value is the nearest level of its group's
    min-max grid; the top group holds the row's largest values; the bytes are the codes then the
    ceil(log2 D)-bit ranks."""
    r = rng(80 + b + g)
    x = (r.standard_normal((5, D)) * 2).astype(np.float16)
    x[0, ::7] *= 20                     # outlier channels
    x[1, :g] = x[1, g:2 * g]            # equal values across channels
    x[2, 5] = x[2, 9]
    side = Side("sorted", b, group=g)
    out = Q.quantize_rows(x, side)
    rank = out["rank"]
    for i in range(5):
        assert sorted(rank[i].tolist()) == list(range(D))
        order = np.argsort(rank[i])                 # channel at each sorted position
        vals = x[i].astype(np.float64)[order]
        assert (np.diff(vals) <= 0).all()
        for p in range(D - 1):
            if vals[p] == vals[p + 1]:
                assert order[p] < order[p + 1]
        assert vals[:g].min() >= vals[g:].max()
        d = out["scales"][i].astype(np.float64)
        z = out["zeros"][i].astype(np.float64)
        for gi in range(D // g):
            grp = vals[gi * g:(gi + 1) * g]
            D_, Z_ = Fraction(float(d[gi])), Fraction(float(z[gi]))
            assert z[gi] == float(np.float16(grp.min()))
            levels = [Z_ + k * D_ for k in range(2 ** b)]
            for jj in range(g):
                assert out["q"][i, gi * g + jj] == _nearest_exact(float(grp[jj]), levels)
        # stored value of channel j is its sorted position's level
        for j in range(D):
            p = rank[i, j]
            assert out["exact"][i, j] == z[p // g] + out["q"][i, p] * d[p // g]
    rb = Q.rank_bits(D)
    assert out["bytes"].shape[1] == (D * b + D * rb + 7) // 8
    assert np.array_equal(Q.unpack_bits(out["bytes"][:, D * b // 8:], rb, D), rank)


def test_sorted_groups_honest_bits_and_error():
    """The page counts 2 bits (plus metadata) for sorted-group 2-bit; the stored permutation adds
    ceil(log2 D) bits per value: 2 + 32/8 + 7 = 13 bits at head_dim 128 with groups of 8 (a scale
    and a zero point per group).  On rows with outlier channels the sorted groups cut the error of
    plain 2-bit groups of the same size."""
    assert Q.bits_per_value(Side("sorted", 2, group=8), 128) == 13.0
    assert Q.bits_per_value(Side("sorted", 2, group=4), 128) == 2 + 8 + 7
    r = rng(90)
    x = r.standard_normal((64, 128))
    x[:, [3, 50, 77, 100]] *= 20
    x = x.astype(np.float16)
    e_sorted = A.rel_sq_error(x, Q.quantize_rows(x, Side("sorted", 2, group=8))["exact"])
    e_plain = A.rel_sq_error(x, Q.quantize_rows(x, Side("int", 2, group=8))["exact"])
    e_plain_mm = A.rel_sq_error(x, Q.quantize_rows(x, Side("int", 2, scale="minmax", group=8))["exact"])
    assert e_sorted < 0.6 * e_plain and e_sorted < 0.6 * e_plain_mm


# ----------------------------------------------------------------------------- per-head allocation
from oracle import headalloc as HA


def test_renyi2_closed_forms():
    """H_2 = -log2 sum p^2 ("Finding 2"): log2 n for n equal weights, 0 for one certain key,
    -log2(p^2 + (1 - p)^2) for two."""
    for n in (1, 2, 7, 64, 1000):
        assert HA.renyi2(np.full(n, 1.0 / n)) == pytest.approx(math.log2(n), abs=1e-12)
    assert HA.renyi2(np.array([1.0, 0.0, 0.0])) == 0.0
    assert HA.renyi2(np.array([0.25, 0.75])) == pytest.approx(-math.log2(0.25 ** 2 + 0.75 ** 2))
    r = rng(91).random(50)
    p = r / r.sum()
    assert 0.0 <= HA.renyi2(p) <= math.log2(50)


def test_head_bits_rule_and_sink_count():
    """b_h = b_avg + 0.25 (H_avg - H_2(h)): the average is kept before rounding, a head at the mean
    entropy gets b_avg, one bit more entropy costs a quarter bit; the bottom 2% of heads are sinks:
    3 of GPT-2's 144 heads ("Finding 2")."""
    H2 = rng(92).uniform(0.5, 9.0, size=144)
    raw = 4 + 0.25 * (H2.mean() - H2)
    assert raw.mean() == pytest.approx(4.0, abs=1e-12)
    b = HA.head_bits(H2, 4.0)
    assert (np.abs(b - raw) <= 0.5).all() and b.min() >= 2 and b.max() <= 8
    flat = np.full(12, 5.0)
    assert (HA.head_bits(flat, 4.0) == 4).all()
    two = np.array([3.0, 7.0])  # mean 5: the diffuse head loses half a bit, the sharp one gains it
    assert HA.head_bits(two, 4.0).tolist() == [5, 4]  # 4.5 rounds up, 3.5 rounds up
    s = HA.sink_heads(H2)
    assert len(s) == 3 and set(s) == set(np.argsort(H2)[:3])
    assert len(HA.sink_heads(np.ones(12))) == 0 and HA.sink_heads(np.arange(50.0)).tolist() == [0]


def test_per_head_spec_bits():
    """A layer with per-head formats averages its heads' bits; an fp16 sink head counts 16."""
    D = 128
    s3, s4, f16 = Side("int", 3, group=32), Side("int", 4, group=32), Side("fp16")
    hk = ((s3, s4, f16, s4),)
    spec = C.Spec(1, 1, 4, 4, D, s4, s4, head_k=hk, head_v=hk)
    want = (3.5 + 4.5 + 16 + 4.5) / 4
    assert C.effective_bits(spec, 100) == pytest.approx(want)
    x = rng(93).standard_normal((5, D)).astype(np.float16)
    for h, side in enumerate(hk[0]):
        kq, _ = C.quantize_unit(spec, x, x, head=h)
        assert np.array_equal(kq["bytes"], Q.quantize_rows(x, side)["bytes"])
