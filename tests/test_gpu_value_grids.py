"""GPU parity of the value grids named for the next run in "E22L" "Result" (a symmetric 2-bit grid
and Lloyd-Max levels for a Gaussian after rotation) and of key-mean subtraction (llama.cpp #21385,
the comment on a shared per-head key mean: subtract the running mean before quantization,
restore it after).

Codes, scales and key means are compared bit for bit with the oracle; stored-domain
dequantization bit for bit; decode attention within 2e-3 per (query, head).
"""
import numpy as np
import pytest
import torch

from kvq_harness import Case
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, Side

pytestmark = pytest.mark.gpu


def cfg_of(D, k, v, B=2, H=2, G=2, T=300, **kw):
    return Config(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=H * G, head_dim=D, capacity=T, k=k, v=v,
                  max_queries=8, **kw)


GRIDS = [
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 2, scale="sym", group=128, rot=256)),  # tensor cores
    (256, 4, Side("int", 4, group=128, rot=256), Side("lloyd", 2, group=128, rot=256)),
    (256, 4, Side("int", 4, group=128, rot=256), Side("lloyd", 3, group=128, rot=256)),
    (128, 2, Side("lloyd", 4, group=64, rot=128), Side("lloyd", 3, group=32)),
    (128, 2, Side("int", 3, scale="sym", group=32, rot=128), Side("int", 4, scale="sym", group=16)),
    (64, 2, Side("int", 2, scale="sym", group=64), Side("lloyd", 2, group=8)),
    (256, 1, Side("int", 8, scale="sym", group=256 // 2), Side("int", 5, scale="sym", group=32, rot=256)),
]


@pytest.mark.parametrize("D,G,k,v", GRIDS, ids=[f"{d}G{g}-{k.fmt}{k.bits}{k.scale[:3]}g{k.group}-{v.fmt}{v.bits}"
                                                 f"{v.scale[:3]}g{v.group}r{v.rot}" for d, g, k, v in GRIDS])
@pytest.mark.parametrize("chunks", [None, [1] * 3 + [150, 1, 146]], ids=["bulk", "mixed"])
def test_value_grid_parity(D, G, k, v, chunks):
    T = 300
    cfg = cfg_of(D, k, v, G=G, T=T)
    c = Case(cfg, T, chunks=chunks)
    c.check_codes(0)
    c.check_dequant(0)
    q = synth.queries(1, 0, 3, cfg.n_q_heads, D, T)
    c.decode_and_compare(0, q[:2])
    c.decode_and_compare(0, q, seq_ids=[1, 0, 1], kv_len=[300, 129, 7])


def _shared_mean_inputs(seed, B, H, T, D, gain=4.0):
    """The seeded law plus a per-(sequence, kv-head) shared key vector (a large common component,
    as the comment describes for the failing models' keys)."""
    K = synth.kv_rows(seed, "k", 0, list(range(B)), list(range(H)), list(range(T)), D, "cpu").numpy()
    V = synth.kv_rows(seed, "v", 0, list(range(B)), list(range(H)), list(range(T)), D, "cpu").numpy()
    r = np.random.default_rng(seed)
    mu = (r.standard_normal((B, H, 1, D)) * gain).astype(np.float32)
    return (K.astype(np.float32) + mu).astype(np.float16), V


MEAN_CASES = [
    (128, 4, Side("int", 4, group=32, rot=128, mean_sub=True), Side("int", 4, group=32, rot=128), {}),  # tensor cores
    (128, 4, Side("nf4", group=64, mean_sub=True), Side("int", 4, group=64), {}),                      # tensor cores
    (128, 2, Side("int", 3, group=32, rot=128, mean_sub=True), Side("int", 3, group=32, rot=128),
     dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=40)),
    (256, 4, Side("int", 3, scale="minmax", group=32, rot=256, chan_scale=True, mean_sub=True),
     Side("int", 2, scale="sym", group=128, rot=256), {}),
    (128, 1, Side("polar", 5, 7, mean_sub=True), Side("int", 4, group=32), {}),
]


@pytest.mark.parametrize("D,G,k,v,anc", MEAN_CASES, ids=[f"{d}G{g}-{k.fmt}{k.bits}r{k.rot}-{v.fmt}{v.bits}"
                                                         for d, g, k, v, _ in MEAN_CASES])
@pytest.mark.parametrize("chunks", [None, [200, 1, 1, 98]], ids=["bulk", "prefill+tokens"])
def test_key_mean_subtraction_parity(D, G, k, v, anc, chunks):
    T = 300
    cfg = cfg_of(D, k, v, G=G, T=T, **anc)
    c = Case(cfg, T, chunks=chunks, inputs=lambda l: _shared_mean_inputs(9, 2, 2, T, D))
    c.check_codes(0)      # the key mean of the first append included
    c.check_dequant(0)    # original domain adds the mean back
    q = synth.queries(1, 0, 2, cfg.n_q_heads, D, T)
    c.decode_and_compare(0, q)
    c.decode_and_compare(0, q, kv_len=[300, 250])


def test_key_mean_is_recomputed_after_an_emptied_cache():
    """The mean belongs to a sequence's first append: emptying the cache and appending other keys
    gives their mean; a per-sequence append to an empty sequence sets only that sequence's mean."""
    D, T = 128, 160
    k = Side("int", 4, group=32, rot=128, mean_sub=True)
    v = Side("int", 4, group=32)
    cfg = cfg_of(D, k, v, G=4, T=T)
    c = Case(cfg, T, inputs=lambda l: _shared_mean_inputs(3, 2, 2, T, D))
    first = c.cache.view(0, 0, "key_mean").cpu().clone()
    c.cache.set_seq_len(-1, 0)
    K2, V2 = _shared_mean_inputs(4, 2, 2, T, D, gain=2.0)
    sid = torch.tensor([1], dtype=torch.int32, device="cuda")
    c.cache.append(0, torch.from_numpy(K2[1:2]).cuda().contiguous(), torch.from_numpy(V2[1:2]).cuda().contiguous(),
                   seq_ids=sid)
    torch.cuda.synchronize()
    now = c.cache.view(0, 0, "key_mean").cpu()
    from oracle import cache as OC
    assert torch.equal(now[:2], first[:2])  # sequence 0 was not appended to: its mean is untouched
    for h in range(2):
        want = OC.key_mean(K2[1, h])
        assert np.array_equal(now[2 + h].numpy().view(np.uint16), want.view(np.uint16))
    assert kvq.kvq_error_flags(c.cache.h) == 0


ANCHOR_CASES = [
    (128, 4, Side("ternary", group=8), Side("ternary", group=8), "first_n", 48, 8),   # "ternboth_a8"
    (128, 4, Side("sign", group=4), Side("sign", group=4), "first_n", 48, 8),         # "signboth_a8"
    (128, 4, Side("nf4", group=64), Side("int", 4, group=64), "window", 64, 4),
    (256, 2, Side("int", 4, group=128, rot=256, mean_sub=True), Side("lloyd", 2, group=128, rot=256), "all", 0, 8),
    (64, 2, Side("int", 3, scale="sym", group=16), Side("int", 4, scale="minmax", group=32), "first_n", 20, 4),
]


@pytest.mark.parametrize("D,G,k,v,rule,n,abits", ANCHOR_CASES,
                         ids=[f"{d}-{k.fmt}-{v.fmt}-{r}{n}-a{a}" for d, g, k, v, r, n, a in ANCHOR_CASES])
@pytest.mark.parametrize("chunks", [None, [130, 1, 1, 1, 67]], ids=["bulk", "tokens"])
def test_int_anchor_parity(D, G, k, v, rule, n, abits, chunks):
    """Post 6, "The winning recipe" item 4 (anchor-precision dial) and "Best results" (int8 anchors
    with ternary and sign KV): anchored rows stored on an 8/4-bit grid; codes, scales, anchors,
    dequantization and attention against the oracle."""
    T = 200
    cfg = Config(n_layers=2, batch=2, n_kv_heads=2, n_q_heads=2 * G, head_dim=D, capacity=T, k=k, v=v, max_queries=8,
                 anchor_layers=(0,), anchor_rule=rule, anchor_n=n, anchor_bits=abits)
    c = Case(cfg, T, chunks=chunks)
    for l in (0, 1):
        c.check_codes(l)
        c.check_anchors(l)
        c.check_dequant(l)
        q = synth.queries(1, l, 2, cfg.n_q_heads, D, T)
        c.decode_and_compare(l, q, kv_len=[200, 151])


SORTED = [
    (128, 4, Side("sorted", 2, group=8), Side("sorted", 2, group=4), {}),                  # the page's g8 K / g4 V
    (128, 2, Side("sorted", 3, group=8, rot=128), Side("sorted", 4, group=16), {}),
    (256, 2, Side("sorted", 2, group=8, mean_sub=True), Side("sorted", 2, group=32, rot=256),
     dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=33)),
    (64, 1, Side("sorted", 2, group=4, chan_scale=True), Side("int", 4, group=16), {}),
]


@pytest.mark.parametrize("D,G,k,v,anc", SORTED, ids=[f"{d}-{k.fmt}{k.bits}g{k.group}r{k.rot}-{v.fmt}{v.bits}g{v.group}"
                                                     for d, g, k, v, _ in SORTED])
@pytest.mark.parametrize("chunks", [None, [1, 1, 120, 1, 77]], ids=["bulk", "tokens"])
def test_sorted_group_parity(D, G, k, v, anc, chunks):
    """Sorted groups with their stored ranks (post 6, "The winning recipe" item 1): codes, ranks,
    scales and zero points bit for bit, dequantization, and attention from the shared-tile decode."""
    T = 200
    cfg = cfg_of(D, k, v, G=G, T=T, **anc)
    c = Case(cfg, T, chunks=chunks)
    c.check_codes(0)
    c.check_anchors(0)
    c.check_dequant(0)
    q = synth.queries(1, 0, 2, cfg.n_q_heads, D, T)
    c.decode_and_compare(0, q)
    c.decode_and_compare(0, q, kv_len=[200, 64])
