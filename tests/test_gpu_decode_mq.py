"""GPU parity of the multi-query tensor-core decode (GQA 1 or 2, more queries than sequences: the
proxy-query setup of "E21W" "What I tested", each query a post-RoPE key attending the keys before
it) against the CPU oracle, and a check that it is the kernel that runs.
"""
import numpy as np
import pytest
import torch

from kvq_harness import Case, kernel_names
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, Side

pytestmark = pytest.mark.gpu


def proxies(c, l, pos, G):
    K = c.K[l][0]  # [H, T, D] of sequence 0
    q = K[:, pos].transpose(1, 0, 2)  # [n, H, D]
    return torch.from_numpy(np.repeat(q, G, axis=1).copy())


MQ = [
    (256, 1, Side("int", 4, scale="minmax", group=32), Side("int", 4, scale="minmax", group=32), {}),
    (256, 1, Side("int", 3, scale="minmax", group=32, rot=256, chan_scale=True),
     Side("int", 3, scale="minmax", group=32, rot=256), {}),
    (128, 1, Side("polar", 5, 7), Side("cart", 6), {}),
    (128, 1, Side("int", 6, group=128, rot=128), Side("int", 6, group=128, rot=128), {}),
    (128, 2, Side("nf4", group=64, mean_sub=True), Side("lloyd", 3, group=32),
     dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=40)),
    (64, 1, Side("sorted", 2, group=8), Side("int", 2, scale="sym", group=16),
     dict(anchor_layers=(0,), anchor_rule="window", anchor_n=50)),
    (256, 2, Side("sign", group=4), Side("ternary", group=8), {}),
    (128, 1, Side("int", 4, group=64), Side("fp16"), {}),
]


@pytest.mark.parametrize("D,G,k,v,anc", MQ, ids=[f"{d}G{g}-{k.fmt}{k.bits}{k.scale[:3]}-{v.fmt}{v.bits}"
                                                 for d, g, k, v, _ in MQ])
def test_many_proxy_queries_on_one_sequence(D, G, k, v, anc):
    T = 700
    H = 2
    cfg = Config(n_layers=1, batch=1, n_kv_heads=H, n_q_heads=H * G, head_dim=D, capacity=T, k=k, v=v,
                 max_queries=100, **anc)
    c = Case(cfg, T, chunks=[500, 1, 199])
    pos = synth.proxy_positions(1, 100, 5, T)  # > 64 rows per CTA: several query blocks
    q = proxies(c, 0, pos, G)
    c.decode_and_compare(0, q, seq_ids=[0] * 100, kv_len=pos.tolist())


def test_odd_capacity_unaligned_staging():
    """Capacity 701 and three kv-heads: a tile's packed ranges start at every alignment, so the
    staging copies take their 16-byte, 4-byte and plain-byte forms."""
    D, T = 128, 701
    cfg = Config(n_layers=1, batch=1, n_kv_heads=3, n_q_heads=3, head_dim=D, capacity=T,
                 k=Side("polar", 4, 8), v=Side("int", 3, scale="minmax", group=32), max_queries=80)
    c = Case(cfg, T, chunks=[333, 368])
    pos = synth.proxy_positions(2, 80, 3, T)
    q = proxies(c, 0, pos, 1)
    c.decode_and_compare(0, q, seq_ids=[0] * 80, kv_len=pos.tolist())


def test_queries_of_several_sequences_in_one_block():
    """Rows of one CTA reading different sequences: one pass per sequence, other rows masked."""
    D, G, T = 128, 2, 400
    s = Side("int", 4, group=32, rot=128)
    cfg = Config(n_layers=1, batch=3, n_kv_heads=2, n_q_heads=4, head_dim=D, capacity=T, k=s, v=s, max_queries=16)
    c = Case(cfg, T)
    q = synth.queries(1, 0, 11, cfg.n_q_heads, D, T)
    seq = [0, 2, 1, 1, 0, 2, 2, 0, 1, 0, 2]
    kl = [400, 1, 0, 399, 7, 255, 400, 33, 128, 64, 300]
    c.decode_and_compare(0, q, seq_ids=seq, kv_len=kl)


def test_multi_query_kernel_is_the_one_that_runs():
    D, T = 256, 512
    s = Side("int", 4, scale="minmax", group=32)
    cfg = Config(n_layers=1, batch=1, n_kv_heads=4, n_q_heads=4, head_dim=D, capacity=T, k=s, v=s, max_queries=32)
    c = Case(cfg, T)
    q = torch.from_numpy(c.K[0][0][:, 100:132].transpose(1, 0, 2).copy()).cuda()
    sid = torch.zeros(32, dtype=torch.int32, device="cuda")
    kl = torch.arange(100, 132, dtype=torch.int32, device="cuda")
    c.cache.decode(0, q, sid, kl)
    torch.cuda.synchronize()
    names = kernel_names(lambda: c.cache.decode(0, q, sid, kl), ["mq_prep_kernel", "decode_mq_kernel", "merge_kernel"])
    assert "mq_prep_kernel" in names and "decode_mq_kernel" in names and "decode_generic_kernel" not in names
    assert kvq.kvq_last_launch_count(c.cache.h) == 3  # query preparation, split pass, merge
