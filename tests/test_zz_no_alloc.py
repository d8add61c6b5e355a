"""kvq_decode_attention_noalloc: decode attention with no device allocation behind it.

Some callers cannot call cudaMalloc where they decode: a serving runtime that hands nearly all of
HBM to its own pool and budgets every other byte, or a latency-critical loop that must not take
the device synchronisation an allocation can cause.  For them the split-K scratch of the decode
lives in a fixed device array inside the library.  This file runs last so that a
failure here leaves every other test already run; it passes alone in a fresh process and after
the rest of the suite.
"""
import pytest
import torch

from kvq_harness import TOL, Case
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, KVQError, Side

pytestmark = pytest.mark.gpu


def _rel(a, b):
    return ((a - b).abs().amax(dim=-1) / b.abs().amax(dim=-1)).max().item()


@pytest.mark.parametrize("D,k,v", [
    (128, Side("nf4", group=64), Side("int", 4, group=64)),                      # tensor-core kernel
    (256, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),
    (128, Side("int", 3, scale="minmax", group=32), Side("polar", 5, 7)),        # shared-tile kernel
])
def test_noalloc_decode_matches_regular_decode_twice(D, k, v):
    T = 900
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=8, head_dim=D, capacity=T, k=k, v=v, max_queries=4)
    c = Case(cfg, T)
    q = synth.queries(1, 0, 3, cfg.n_q_heads, D, T).cuda()
    seq = torch.tensor([0, 1, 1], dtype=torch.int32, device="cuda")
    kl = torch.tensor([900, 517, 3], dtype=torch.int32, device="cuda")
    ref_out, ref_lse = c.cache.decode(0, q, seq, kl, lse=True)

    def noalloc(layer, qq, sid, kvl):
        out = torch.full_like(ref_out, float("nan"))
        lse = torch.full_like(ref_lse, float("nan"))
        kvq.kvq_decode_attention_noalloc(c.cache.h, layer, qq, qq.shape[0], sid, kvl, out, lse)
        torch.cuda.synchronize()
        return out, lse

    for _ in range(2):  # two calls in a row share (and overwrite) the fixed scratch
        out, lse = noalloc(0, q, seq, kl)
        assert _rel(out, ref_out) <= TOL
        assert torch.allclose(lse, ref_lse, rtol=1e-5, atol=1e-5)
    # and against the CPU oracle's attention over the same packed cache
    c.decode_and_compare(0, q.cpu(), seq_ids=[0, 1, 1], kv_len=[900, 517, 3], decode=noalloc)


def test_noalloc_rejects_requests_beyond_its_scratch():
    s = Side("int", 4, group=32)
    cfg = Config(n_layers=1, batch=1, n_kv_heads=8, n_q_heads=32, head_dim=128, capacity=256, k=s, v=s,
                 max_queries=1024)
    c = Case(cfg, 256)
    n_q = 1024  # 1024 x 32 heads x (splits + 1) x 132 floats > 2^21
    q = torch.zeros(n_q, 32, 128, dtype=torch.float16, device="cuda")
    seq = torch.zeros(n_q, dtype=torch.int32, device="cuda")
    out = torch.empty(n_q, 32, 128, device="cuda")
    with pytest.raises(KVQError) as e:
        kvq.kvq_decode_attention_noalloc(c.cache.h, 0, q, n_q, seq, None, out)
    assert e.value.status == -3
    # more queries than the handle's max_queries: the same status as kvq_decode_attention
    with pytest.raises(KVQError) as e:
        kvq.kvq_decode_attention_noalloc(c.cache.h, 0, q, n_q + 1, seq, None, out)
    assert e.value.status == -3
