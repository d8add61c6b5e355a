"""GPU parity of the tensor-core decode instances (GQA 4 and 2) against the CPU oracle.

Each case fills a cache through kvq_quantize_append, decodes through kvq_decode_attention and
compares every (query, head) output with the oracle's fp64 attention over its own
reconstruction (max relative error 2e-3).  Lengths span several 128/256-token tiles with ragged
tails; anchors start the quantized range off a tile boundary.  A profiler pass checks that the
tensor-core kernel is the one that ran.
"""
import pytest
import torch

from kvq_harness import Case, kernel_names
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, Side

pytestmark = pytest.mark.gpu

MMA_CASES = [
    (128, 4, Side("nf4", group=64), Side("int", 4, group=64)),
    (128, 4, Side("int", 4, group=64), Side("int", 4, group=64)),
    (128, 4, Side("int", 4, group=32, rot=128), Side("int", 4, group=32, rot=128)),
    (128, 2, Side("int", 4, group=32, rot=128), Side("int", 4, group=32, rot=128)),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 4, group=128)),
    (256, 4, Side("int", 4, group=128, rot=256), Side("fp16")),
    (256, 4, Side("int", 4, group=32), Side("int", 4, group=32)),
    (256, 4, Side("int", 4, group=128, rot=256, chan_scale=True), Side("int", 2, group=128, rot=256)),
    (128, 4, Side("sign", group=4), Side("sign", group=4)),
    (128, 4, Side("ternary", group=8), Side("ternary", group=8)),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256)),
]


def ids(c):
    D, G, k, v = c
    return f"D{D}G{G}-{k.fmt}{k.bits}g{k.group}r{k.rot}{'c' if k.chan_scale else ''}-{v.fmt}{v.bits}g{v.group}r{v.rot}"


def make(D, G, k, v, T, B=2, H=2, L=1, **kw):
    cfg = Config(n_layers=L, batch=B, n_kv_heads=H, n_q_heads=H * G, head_dim=D, capacity=T, k=k, v=v,
                 max_queries=8, **kw)
    return cfg, Case(cfg, T)


@pytest.mark.parametrize("case", MMA_CASES, ids=[ids(c) for c in MMA_CASES])
def test_mma_decode_parity(case):
    D, G, k, v = case
    T = 700
    cfg, c = make(D, G, k, v, T)
    q = synth.queries(1, 0, 4, cfg.n_q_heads, D, T)
    c.decode_and_compare(0, q[:2])
    c.decode_and_compare(0, q, seq_ids=[0, 1, 1, 0], kv_len=[700, 513, 256, 17])


@pytest.mark.parametrize("rule,n", [("first_n", 48), ("window", 100)])
def test_mma_decode_with_anchors(rule, n):
    cfg, c = make(128, 4, Side("nf4", group=64), Side("int", 4, group=64), 600, L=2,
                  anchor_layers=(0,), anchor_rule=rule, anchor_n=n)
    for l in (0, 1):
        q = synth.queries(1, l, 2, cfg.n_q_heads, 128, 600)
        c.decode_and_compare(l, q, kv_len=[600, 555])


@pytest.mark.parametrize("k,v", [(Side("nf4", group=64), Side("int", 4, group=64)),
                                 (Side("sign", group=4), Side("sign", group=4)),
                                 (Side("ternary", group=8), Side("ternary", group=8))],
                         ids=["nf4-int4", "sign", "ternary"])
def test_mma_kernel_is_the_one_that_runs(k, v):
    cfg, c = make(128, 4, k, v, 512)
    q = synth.queries(1, 0, 2, cfg.n_q_heads, 128, 512).cuda()
    c.cache.decode(0, q)
    torch.cuda.synchronize()
    names = kernel_names(lambda: c.cache.decode(0, q), ["decode_tc_kernel", "merge_kernel"])
    assert "decode_tc_kernel" in names and "merge_kernel" in names
    assert "decode_generic_kernel" not in names
    assert kvq.kvq_last_launch_count(c.cache.h) == 2


def test_symmetric_v_runs_on_tensor_cores():
    """The symmetric 2-bit V grid ("E22L" "Result") under a 256-wide rotation has a register-decode
    instance."""
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=8, head_dim=256, capacity=512,
                 k=Side("int", 4, group=128, rot=256), v=Side("int", 2, scale="sym", group=128, rot=256), max_queries=8)
    c = Case(cfg, 512)
    q = synth.queries(1, 0, 2, cfg.n_q_heads, 256, 512).cuda()
    c.cache.decode(0, q)
    torch.cuda.synchronize()
    names = kernel_names(lambda: c.cache.decode(0, q), ["decode_tc_kernel", "merge_kernel"])
    assert "decode_tc_kernel" in names and "decode_generic_kernel" not in names


def test_append_is_one_launch_for_common_pairs():
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=8, head_dim=128, capacity=128,
                 k=Side("nf4", group=64), v=Side("int", 4, group=64), max_queries=8)
    c = Case(cfg, 64)
    k = synth.kv_rows(3, "k", 0, list(range(cfg.batch)), list(range(cfg.n_kv_heads)), [64], 128, "cuda")
    v = synth.kv_rows(3, "v", 0, list(range(cfg.batch)), list(range(cfg.n_kv_heads)), [64], 128, "cuda")
    c.cache.append(0, k, v)
    torch.cuda.synchronize()
    assert kvq.kvq_last_launch_count(c.cache.h) == 1


def test_mma_long_sequence_many_splits():
    """One sequence, 4 kv-heads, 40K tokens: the split planner spreads it over many CTAs."""
    cfg, c = make(256, 4, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256), 40000, B=1, H=4)
    q = synth.queries(1, 0, 1, cfg.n_q_heads, 256, 40000)
    c.decode_and_compare(0, q)
