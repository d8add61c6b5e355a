"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on seeded inputs.

Codes, scales and stored-domain dequantization are compared bit for bit; decode attention
within max relative error 2e-3 per (query, head) vector.  Sizes span several 128-token tiles
and a ragged tail, so split-K boundaries, partial tiles and the merge are all exercised.
"""
import numpy as np
import pytest
import torch

from kvq_harness import TOL, Case
from quantized_decode_attention_append_b200 import synth
from quantized_decode_attention_append_b200.kvq import Config
from quantized_decode_attention_append_b200.kvq import KVQError, Side

pytestmark = pytest.mark.gpu


def cfg_of(D, k, v, B=2, H=2, Hq=4, L=1, cap=None, T=300, **kw):
    return Config(n_layers=L, batch=B, n_kv_heads=H, n_q_heads=Hq, head_dim=D, capacity=cap or T, k=k, v=v,
                  max_queries=max(B, 16), **kw)


def queries(cfg, n, pos, seed=1, layer=0):
    return synth.queries(seed, layer, n, cfg.n_q_heads, cfg.head_dim, pos)


# --------------------------------------------------------------------------------- Tiny (full size)
def test_tiny_config_full():
    """1 layer, 2 KV heads, 4 query heads, head_dim 128, 512 tokens; Hadamard-128 int4 absmax g32."""
    s = Side("int", 4, group=32, rot=128)
    cfg = cfg_of(128, s, s, B=1, H=2, Hq=4, T=512)
    c = Case(cfg, 512)
    c.check_codes(0)
    c.check_dequant(0)
    c.decode_and_compare(0, queries(cfg, 1, 512))


FORMATS = [
    (128, Side("int", 4, group=32), Side("int", 4, group=32)),
    (128, Side("int", 2, group=128, rot=128), Side("int", 3, group=64, rot=128)),
    (128, Side("int", 8, group=16), Side("int", 5, group=8)),
    (128, Side("nf4", group=64), Side("int", 4, group=64)),
    (128, Side("ternary", group=8), Side("ternary", group=8)),
    (128, Side("sign", group=4), Side("sign", group=4)),
    (128, Side("polar", 4, 8), Side("polar", 8, 4)),
    (128, Side("polar", 5, 7), Side("polar", 6, 6)),
    (128, Side("polar", 7, 5), Side("cart", 6)),
    (128, Side("int", 6, group=128, rot=128), Side("int", 6, group=128, rot=128)),
    (256, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),
    (256, Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256)),
    (256, Side("int", 4, group=128, rot=256), Side("fp16")),
    (256, Side("int", 4, group=32), Side("int", 4, group=32)),
    (256, Side("int", 3, scale="minmax", group=32), Side("int", 3, scale="minmax", group=32)),
    (256, Side("int", 4, scale="minmax", group=32, rot=256), Side("int", 4, scale="minmax", group=32, rot=256)),
    (256, Side("int", 3, scale="minmax", group=32, chan_scale=True), Side("int", 3, scale="minmax", group=32)),
    (256, Side("int", 4, scale="minmax", group=32, rot=256, chan_scale=True),
     Side("int", 4, scale="minmax", group=32, rot=256)),
    (256, Side("int", 4, group=64, rot=128), Side("nf4", group=32)),
    (64, Side("int", 4, group=16), Side("sign", group=8)),
    (64, Side("nf4", group=64), Side("ternary", group=4)),
    (256, Side("ternary", group=8, rot=256), Side("sign", group=16, rot=128)),
    (256, Side("int", 7, group=64), Side("int", 5, scale="minmax", group=32)),
]


@pytest.mark.parametrize("D,k,v", FORMATS, ids=[f"{d}-{k.fmt}{k.bits}g{k.group}r{k.rot}-{v.fmt}{v.bits}g{v.group}"
                                                   for d, k, v in FORMATS])
def test_format_parity(D, k, v):
    cfg = cfg_of(D, k, v, T=300)
    c = Case(cfg, 300)
    c.check_codes(0)
    c.check_dequant(0)
    c.decode_and_compare(0, queries(cfg, 2, 300))


BULK = [
    (128, Side("nf4", group=64), Side("int", 4, group=64)),
    (128, Side("ternary", group=8), Side("sign", group=4)),
    (128, Side("int", 4, group=32, rot=128), Side("int", 3, scale="minmax", group=16)),
    (256, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),
    (256, Side("int", 3, scale="minmax", group=32, rot=256, chan_scale=True), Side("sign", group=8)),
    (64, Side("int", 8, group=64), Side("nf4", group=16)),
]


@pytest.mark.parametrize("D,k,v", BULK, ids=[f"{d}-{k.fmt}{k.bits}g{k.group}-{v.fmt}{v.bits}g{v.group}" for d, k, v in BULK])
def test_bulk_prefill_and_token_appends_agree(D, k, v):
    """A prefill above the small-append threshold (2 x 2 x 2100 rows) takes the unrolled
    thread-per-row kernel; token-by-token appends take the warp-per-row kernel.  Both must give
    the oracle's bytes."""
    T = 2100
    cfg = cfg_of(D, k, v, T=T)
    bulk = Case(cfg, T)
    inc = Case(cfg, T, chunks=[1] * 9 + [500, 1, 1590])
    for side in (0, 1):
        for what in ("codes", "scales", "zeros"):
            a, b = bulk.cache.view(0, side, what), inc.cache.view(0, side, what)
            if a is not None:
                assert torch.equal(a[:, :T].cpu(), b[:, :T].cpu()), (side, what)
    assert inc.cache.view(0, 0, "seq_len").cpu().tolist() == [T, T]
    bulk.check_codes(0)
    bulk.decode_and_compare(0, queries(cfg, 2, T))


@pytest.mark.parametrize("rule,n", [("first_n", 48), ("window", 64), ("all", 0)])
def test_anchor_rules(rule, n):
    s = Side("ternary", group=8)
    cfg = cfg_of(128, s, s, L=2, T=300, anchor_layers=(0,), anchor_rule=rule, anchor_n=n)
    c = Case(cfg, 300)
    for l in (0, 1):
        c.check_codes(l)
        c.check_dequant(l)
        c.decode_and_compare(l, queries(cfg, 2, 300, layer=l), kv_len=[300, 299])


def test_window_anchor_ring_wraps():
    """A window smaller than the appended run: ring slots are reused as tokens arrive."""
    s = Side("sign", group=4)
    cfg = cfg_of(128, s, s, T=260, anchor_layers=(0,), anchor_rule="window", anchor_n=64)
    c = Case(cfg, 260, chunks=[100, 1, 1, 30, 128])
    c.check_dequant(0)
    c.decode_and_compare(0, queries(cfg, 2, 260))


def test_decode_ragged_lengths_and_seq_ids():
    s = Side("int", 4, group=32, rot=128)
    cfg = cfg_of(128, s, s, B=3, T=400)
    c = Case(cfg, 400)
    q = queries(cfg, 6, 400)
    c.decode_and_compare(0, q, seq_ids=[0, 1, 2, 2, 1, 0], kv_len=[400, 1, 0, 129, 255, 37])


def test_proxy_queries_share_a_sequence():
    """Proxy queries ("E21W"): the post-RoPE key at position p as the query, causal over t < p."""
    s = Side("int", 4, scale="minmax", group=32, rot=256)
    cfg = Config(n_layers=1, batch=1, n_kv_heads=4, n_q_heads=4, head_dim=256, capacity=600, k=s, v=s,
                 max_queries=16)
    c = Case(cfg, 600)
    pos = synth.proxy_positions(1, 16, 300, 600)
    q = torch.from_numpy(c.K[0][0][:, pos].transpose(1, 0, 2).copy())  # [16, Hq=Hkv, D]
    c.decode_and_compare(0, q, seq_ids=[0] * 16, kv_len=pos.tolist())


def test_capacity_error_and_flags():
    s = Side("int", 4, group=32)
    cfg = cfg_of(128, s, s, T=100, cap=128)
    c = Case(cfg, 100)
    k = torch.zeros(2, 2, 29, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(KVQError) as e:
        c.cache.append(0, k, k)
    assert e.value.status == -3
    assert c.cache.view(0, 0, "seq_len").cpu().tolist() == [100, 100]
    from quantized_decode_attention_append_b200 import kvq
    assert kvq.kvq_error_flags(c.cache.h) == 0


def test_sm_scale_override():
    s = Side("int", 8, group=32)
    cfg = cfg_of(128, s, s, T=160, sm_scale=0.05)
    c = Case(cfg, 160)
    c.decode_and_compare(0, queries(cfg, 2, 160))


def test_fp16_output_path():
    s = Side("int", 4, group=32, rot=128)
    cfg = cfg_of(128, s, s, T=256)
    c = Case(cfg, 256)
    q = queries(cfg, 2, 256).cuda()
    o32 = c.cache.decode(0, q)
    o16 = c.cache.decode(0, q, fp32=False)
    assert torch.allclose(o16.float(), o32, rtol=1e-3, atol=1e-3)


# ------------------------------------------------------------------- decision-boundary inputs
ADVERSARIAL = [
    (128, Side("int", 4, group=32), Side("int", 3, group=64)),
    (128, Side("int", 2, group=128), Side("int", 8, group=16)),
    (128, Side("int", 4, group=64), Side("int", 4, group=64)),
    (128, Side("nf4", group=64), Side("int", 4, group=64)),
    (128, Side("ternary", group=8), Side("sign", group=4)),
    (128, Side("nf4", group=16), Side("ternary", group=4)),
    (256, Side("int", 4, scale="minmax", group=32), Side("int", 3, scale="minmax", group=16)),
    (64, Side("int", 3, group=16), Side("nf4", group=32)),
]


@pytest.mark.parametrize("D,k,v", ADVERSARIAL, ids=[f"{d}-{k.fmt}{k.bits}g{k.group}-{v.fmt}{v.bits}g{v.group}"
                                                       for d, k, v in ADVERSARIAL])
@pytest.mark.parametrize("chunks", [None, [1] * 6 + [58]], ids=["bulk", "tokens"])
def test_decision_boundaries(D, k, v, chunks):
    """Rows whose values sit exactly on rounding ties, NF4 thresholds, both-sign maxima and
    signed zeros: codes and scales still bit-identical to the oracle."""
    import adversarial
    T = 64
    cfg = cfg_of(D, k, v, T=T)
    c = Case(cfg, T, chunks=chunks, inputs=lambda l: (adversarial.rows(11 + l, 2, 2, T, D),
                                                      adversarial.rows(97 + l, 2, 2, T, D)))
    c.check_codes(0)
    c.check_dequant(0)


# ------------------------------------------------------------------------------ per-layer formats
def test_per_layer_bit_allocation():
    """"E21W" "Result": rotated groups of 128 with 2-bit K in layers 2 and 7, 4-bit V in layers
    1, 3 and 4, 3 bits elsewhere (3.19 bits on average).  Each layer is quantized with its own
    grid and decoded from it."""
    side = lambda b: Side("int", b, group=128, rot=256)
    lk = tuple(side(2 if l in (2, 7) else 3) for l in range(8))
    lv = tuple(side(4 if l in (1, 3, 4) else 3) for l in range(8))
    cfg = cfg_of(256, side(4), side(4), B=1, H=2, Hq=4, L=8, T=300, layer_k=lk, layer_v=lv)
    c = Case(cfg, 300)
    for l in range(8):
        assert c.cache.layout(l, 0).row_bytes == 256 * lk[l].bits // 8
        assert c.cache.layout(l, 1).row_bytes == 256 * lv[l].bits // 8
        c.check_codes(l)
        c.decode_and_compare(l, queries(cfg, 1, 300, layer=l))


def test_per_layer_format_families():
    """Layers of one cache in different families: each layer takes its own append and decode
    kernels (register-decode and shared-tile tensor-core paths side by side)."""
    lk = (Side("nf4", group=64), Side("sign", group=4), Side("int", 3, scale="minmax", group=32),
          Side("ternary", group=8))
    lv = (Side("int", 4, group=64), Side("sign", group=4), Side("int", 4, scale="minmax", group=32),
          Side("ternary", group=8))
    cfg = cfg_of(128, lk[0], lv[0], B=2, H=2, Hq=8, L=4, T=300, layer_k=lk, layer_v=lv)
    c = Case(cfg, 300)
    for l in range(4):
        c.check_codes(l)
        c.check_dequant(l)
        c.decode_and_compare(l, queries(cfg, 2, 300, layer=l))


# ---------------------------------------------- decision boundaries behind a pre-transform
def _pow2_chan(seed, H, D):
    r = np.random.default_rng(seed)
    return (2.0 ** r.integers(-2, 3, size=(H, D))).astype(np.float16)


ROTATED_TIES = [
    (256, Side("int", 4, group=32, rot=256), Side("int", 2, group=128, rot=256)),
    (256, Side("int", 3, group=64, rot=256), Side("int", 4, group=128, rot=128)),
    (256, Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256)),
    (128, Side("int", 4, group=32, rot=128), Side("int", 2, group=16, rot=128)),
    (128, Side("int", 4, group=64, rot=128), Side("nf4", group=64, rot=128)),
    (256, Side("int", 4, group=32, rot=256, chan_scale=True), Side("ternary", group=8, rot=256)),
    (256, Side("int", 2, group=128, rot=128, chan_scale=True), Side("int", 4, scale="minmax", group=32, rot=256)),
]


@pytest.mark.parametrize("D,k,v", ROTATED_TIES, ids=[f"{d}-{k.fmt}{k.bits}g{k.group}r{k.rot}c{int(k.chan_scale)}-"
                                                       f"{v.fmt}{v.bits}g{v.group}r{v.rot}" for d, k, v in ROTATED_TIES])
@pytest.mark.parametrize("chunks", [None, [1] * 5 + [59]], ids=["bulk", "tokens"])
def test_rotated_decision_boundaries(D, k, v, chunks):
    """Rows whose Hadamard image (after an exact power-of-two channel scale for K) puts absmax ties
    of both signs and x/d on half-integers: the rotated path's exact near-tie fallback must give
    the oracle's codes and scales ("E21W" variants B and D, "E22L" "What I tested")."""
    import adversarial
    T = 64
    cfg = cfg_of(D, k, v, T=T)
    chan = _pow2_chan(5, 2, D)

    def inputs(l):
        K = adversarial.spike_rows(21 + l, 2, 2, T, D, k.rot)
        if k.chan_scale:  # x = spike * c, so x / c is the spike exactly
            K = (K.astype(np.float32) * chan[None, :, None, :].astype(np.float32)).astype(np.float16)
        return K, adversarial.spike_rows(77 + l, 2, 2, T, D, v.rot)

    c = Case(cfg, T, chunks=chunks, inputs=inputs, chan=lambda l: chan)
    c.check_codes(0)
    c.check_dequant(0)
    c.decode_and_compare(0, queries(cfg, 2, T))


@pytest.mark.parametrize("bm,bp", [(4, 8), (5, 7), (6, 6), (7, 5), (8, 4)])
def test_polar_phase_boundaries(bm, bp):
    """Spectrum slots whose angle sits next to a phase-code boundary (k + 1/2) 2 pi / 2^bp: inside
    the GPU's fp64 fallback band and just outside it.  Phase codes must equal the oracle's
    (the reply, "The finite-phase implementation and the physical codec may be worth
    separating": one phase-angle index per coefficient)."""
    import adversarial
    T = 64
    rows = adversarial.polar_boundary_rows(40 + bp, 2 * 2 * T, bp)
    K = rows.reshape(2, 2, T, 128)
    V = rows[::-1].copy().reshape(2, 2, T, 128)
    s = Side("polar", bm, bp)
    cfg = cfg_of(128, s, s, T=T)
    c = Case(cfg, T, inputs=lambda l: (K, V))
    c.check_codes(0)
    c.check_dequant(0)
    c.decode_and_compare(0, queries(cfg, 2, T))
