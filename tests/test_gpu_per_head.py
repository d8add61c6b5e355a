"""Per-(layer, kv-head) formats (llama.cpp #21385 "Finding 2" and "Feature Request: Per-Head KV Cache
Types": per-head bits from attention entropy, sink heads left unquantized, per-head dequantization
dispatch) against the oracle.

Heads of one layer with different formats live in separate head groups (their own arena regions
and launches); the caller still passes and receives all heads at once.
"""
import numpy as np
import pytest
import torch

from kvq_harness import Case
from quantized_decode_attention_append_b200 import headalloc, kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, Side

pytestmark = pytest.mark.gpu


def test_mixed_head_formats_parity():
    i4 = Side("int", 4, group=32, rot=128)
    nf = Side("nf4", group=64)
    i3 = Side("int", 3, group=32, rot=128, mean_sub=True)
    f16 = Side("fp16")
    hk = ((i4, i4, nf, f16, i3, i3), (f16, i4, i4, i4, i4, nf))
    hv = ((i4, i4, Side("int", 4, group=64), f16, Side("lloyd", 2, group=32), Side("lloyd", 2, group=32)),
          (f16, i4, i4, i4, i4, Side("int", 4, group=64)))
    T = 300
    cfg = Config(n_layers=2, batch=2, n_kv_heads=6, n_q_heads=24, head_dim=128, capacity=T, k=i4, v=i4,
                 max_queries=8, head_k=hk, head_v=hv, anchor_layers=(1,), anchor_rule="first_n", anchor_n=20)
    c = Case(cfg, T, chunks=[200, 1, 99])
    assert [c.cache.layout(0, 0, h).head0 for h in range(6)] == [0, 0, 2, 3, 4, 4]
    assert [c.cache.layout(1, 0, h).n_heads for h in range(6)] == [1, 4, 4, 4, 4, 1]
    for l in (0, 1):
        c.check_codes(l)
        c.check_anchors(l)
        c.check_dequant(l)
        q = synth.queries(1, l, 3, cfg.n_q_heads, 128, T)
        c.decode_and_compare(l, q[:2])
        c.decode_and_compare(l, q, seq_ids=[1, 0, 1], kv_len=[300, 257, 5])
    # one decode pass + merge per head group (group with the 4-head TC instance included)
    c.cache.decode(0, synth.queries(1, 0, 2, cfg.n_q_heads, 128, T).cuda())
    assert kvq.kvq_last_launch_count(c.cache.h) >= 2 * 4


def test_per_head_append_to_a_subset_and_noalloc():
    """Per-sequence appends and the no-allocation decode go through every head group."""
    a, b_ = Side("int", 4, group=32), Side("sign", group=4)
    cfg = Config(n_layers=1, batch=3, n_kv_heads=2, n_q_heads=8, head_dim=128, capacity=256, k=a, v=a,
                 max_queries=4, head_k=((a, b_),), head_v=((a, b_),))
    c = Case(cfg, 100)
    K = synth.kv_rows(0, "k", 0, [2], [0, 1], list(range(100, 130)), 128, "cuda")
    V = synth.kv_rows(0, "v", 0, [2], [0, 1], list(range(100, 130)), 128, "cuda")
    c.cache.append(0, K, V, seq_ids=torch.tensor([2], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert c.cache.view(0, 0, "seq_len").cpu().tolist() == [100, 100, 130]
    q = synth.queries(1, 0, 3, 8, 128, 130).cuda()
    ref = c.cache.decode(0, q)
    out = torch.empty_like(ref)
    kvq.kvq_decode_attention_noalloc(c.cache.h, 0, q, 3, None, None, out)
    torch.cuda.synchronize()
    assert torch.allclose(out, ref, rtol=1e-6, atol=1e-6)
    assert kvq.kvq_error_flags(c.cache.h) == 0


def test_entropy_calibrated_allocation():
    """The calibration pass: per-head Renyi entropies of fp16 attention with proxy queries (post-
    RoPE keys, causal), bits from b_h = 4 + 0.25 (H_avg - H_2(h)), the lowest-entropy head kept at
    fp16; the cache built from that table matches the oracle."""
    L, B, H, D, T = 2, 1, 4, 128, 600
    H2 = np.zeros((L, H))
    pos = synth.proxy_positions(1, 16, 300, 600)
    for l in range(L):
        K = synth.kv_rows(0, "k", l, [0], list(range(H)), list(range(T)), D, "cuda")[0]
        q = K[:, pos].transpose(0, 1).contiguous()  # [16, H, D] (G = 1)
        H2[l] = headalloc.head_entropy(q, K, pos.tolist()).cpu().numpy()
    hk, hv, bits = headalloc.allocate(H2, 4.0, side_of_bits=lambda b: Side("int", b, group=32, rot=128),
                                      sink_frac=0.125)
    flat = [b for row in bits for b in row]
    assert flat.count(16) == 1 and all(2 <= b <= 8 for b in flat if b != 16)
    cfg = Config(n_layers=L, batch=B, n_kv_heads=H, n_q_heads=H, head_dim=D, capacity=T, k=hk[0][0], v=hv[0][0],
                 max_queries=16, head_k=hk, head_v=hv)
    c = Case(cfg, T)
    for l in range(L):
        c.check_codes(l)
        qp = torch.from_numpy(c.K[l][0][:, pos].transpose(1, 0, 2).copy())
        c.decode_and_compare(l, qp, seq_ids=[0] * 16, kv_len=pos.tolist())
