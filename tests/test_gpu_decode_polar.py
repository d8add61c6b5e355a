"""GPU parity of the CUDA-core polar decode (rFFT polar K and V, one query per sequence, GQA 1, 2
or 4: "Fourier Magnitude KV Cache Quantization", the reply on finite-phase codes) against the CPU
oracle, and checks of which kernel serves which query layout.
"""
import numpy as np
import pytest
import torch

from kvq_harness import Case, kernel_names
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, Side

pytestmark = pytest.mark.gpu

D = 128

# (magnitude bits, phase bits) of K and V: the compiled-in 4 + 8 split, the other splits of the
# 6.125-bit budget, the narrowest fields and unequal phase widths (two phase tables)
SPLITS = [((4, 8), (4, 8)), ((5, 7), (5, 7)), ((6, 6), (6, 6)), ((7, 5), (8, 4)), ((1, 1), (3, 2)),
          ((4, 8), (6, 6)), ((8, 8), (2, 8))]


@pytest.mark.parametrize("ks,vs", SPLITS, ids=[f"k{a}+{b}-v{c}+{d}" for (a, b), (c, d) in SPLITS])
def test_polar_splits(ks, vs):
    """Capacity 701 and three kv-heads: tiles start at every staging alignment; 700 tokens end in
    a ragged tile."""
    T = 700
    cfg = Config(n_layers=1, batch=2, n_kv_heads=3, n_q_heads=3, head_dim=D, capacity=701,
                 k=Side("polar", *ks), v=Side("polar", *vs))
    c = Case(cfg, T, chunks=[300, 1, 399])
    q = synth.queries(1, 0, 2, 3, D, T)
    c.decode_and_compare(0, q)


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("split", [(4, 8), (5, 7)])
def test_polar_gqa_groups(G, split):
    T = 513
    s = Side("polar", *split)
    cfg = Config(n_layers=1, batch=3, n_kv_heads=2, n_q_heads=2 * G, head_dim=D, capacity=T, k=s, v=s)
    c = Case(cfg, T)
    q = synth.queries(2, 0, 3, 2 * G, D, T)
    c.decode_and_compare(0, q)


def test_polar_lengths_and_sequence_ids():
    """Queries over a subset of the batch in another order, attending 0, 1, a tile minus one, a
    tile, a tile plus one and all of their tokens."""
    T = 640
    s = Side("polar", 4, 8)
    cfg = Config(n_layers=1, batch=6, n_kv_heads=2, n_q_heads=2, head_dim=D, capacity=T, k=s, v=s)
    c = Case(cfg, T)
    q = synth.queries(3, 0, 6, 2, D, T)
    c.decode_and_compare(0, q, seq_ids=[5, 0, 3, 1, 2, 4], kv_len=[0, 1, 63, 64, 65, 640])


@pytest.mark.parametrize("anc", [dict(anchor_rule="first_n", anchor_n=40),
                                 dict(anchor_rule="window", anchor_n=70)], ids=["first_n", "window"])
def test_polar_with_anchor_rows(anc):
    """Anchored rows go to the generic kernel's anchor split; the polar kernel masks them (the
    first tile starts inside the anchored prefix, or the range ends before the window)."""
    T = 400
    s = Side("polar", 4, 8)
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=4, head_dim=D, capacity=T, k=s, v=s,
                 anchor_layers=(0,), **anc)
    c = Case(cfg, T)
    q = synth.queries(4, 0, 2, 4, D, T)
    c.decode_and_compare(0, q, kv_len=[T, 333])


def test_polar_key_mean_subtraction():
    T = 300
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=2, head_dim=D, capacity=T,
                 k=Side("polar", 4, 8, mean_sub=True), v=Side("polar", 4, 8))
    c = Case(cfg, T, chunks=[128, 172])
    q = synth.queries(5, 0, 2, 2, D, T)
    c.decode_and_compare(0, q)


def test_polar_long_sequence_one_wave():
    """8192 tokens, 8 kv-heads, batch 1 (the config-4 decode shape): one wave of splits, about
    forty per head."""
    T = 8192
    s = Side("polar", 4, 8)
    cfg = Config(n_layers=1, batch=1, n_kv_heads=8, n_q_heads=8, head_dim=D, capacity=T, k=s, v=s)
    c = Case(cfg, T)
    q = synth.queries(6, 0, 1, 8, D, T)
    c.decode_and_compare(0, q)


def test_polar_kernel_is_the_one_that_runs():
    T = 256
    s = Side("polar", 4, 8)
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=2, head_dim=D, capacity=T, k=s, v=s, max_queries=8)
    c = Case(cfg, T)
    q = synth.queries(7, 0, 2, 2, D, T).cuda()
    c.cache.decode(0, q)
    torch.cuda.synchronize()
    names = kernel_names(lambda: c.cache.decode(0, q), ["decode_polar_kernel", "merge_kernel"])
    assert "decode_polar_kernel" in names
    assert "decode_mq_kernel" not in names and "mq_prep_kernel" not in names and "decode_generic_kernel" not in names
    assert kvq.kvq_last_launch_count(c.cache.h) == 2  # split pass (queries transformed inside), merge
    # more queries than sequences (proxy queries share a sequence): the multi-query kernel
    q8 = torch.from_numpy(np.ascontiguousarray(c.K[0][0][:, 100:108].transpose(1, 0, 2))).cuda()
    sid = torch.zeros(8, dtype=torch.int32, device="cuda")
    kl = torch.arange(100, 108, dtype=torch.int32, device="cuda")
    names = kernel_names(lambda: c.cache.decode(0, q8, sid, kl), ["decode_mq_kernel"])
    assert "decode_mq_kernel" in names and "decode_polar_kernel" not in names


def test_polar_calls_in_a_row():
    """Calls with other query counts, sequence subsets, lengths and layers one after another."""
    T = 500
    s = Side("polar", 4, 8)
    cfg = Config(n_layers=2, batch=4, n_kv_heads=2, n_q_heads=4, head_dim=D, capacity=T, k=s, v=s)
    c = Case(cfg, T)
    for l, sids, kl in [(0, [0, 1, 2, 3], None), (1, [2], [137]), (0, [3, 1], [500, 64]), (1, [0, 1, 2, 3], None)]:
        q = synth.queries(8 + l, l, len(sids), 4, D, T)
        c.decode_and_compare(l, q, seq_ids=sids, kv_len=kl)
