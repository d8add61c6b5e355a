"""Per-sequence appends (kvq_quantize_append with seq_ids) and the decode's bounded wait.

Appends that reach only some sequences leave the others untouched; the cache then holds
sequences of different lengths, and codes and attention of every sequence are compared with the
oracle on that sequence's own rows ("E22L" "What I tested": keys and values quantized on entry
to the cache, one sequence at a time as it decodes).
"""
import numpy as np
import pytest
import torch

from kvq_harness import TOL, oracle_spec
from oracle import attention as OA
from oracle import cache as OC
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, KVCache, KVQError, Side

pytestmark = pytest.mark.gpu

B, H, CAP = 4, 2, 400

FORMATS = [
    (128, Side("int", 4, group=32, rot=128), Side("int", 4, group=32, rot=128), {}),
    (128, Side("nf4", group=64), Side("fp16"), {}),
    (128, Side("polar", 4, 8), Side("cart", 6), {}),
    (128, Side("ternary", group=8), Side("sign", group=4), dict(anchor_layers=(0,), anchor_rule="window", anchor_n=32)),
    (256, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256),
     dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=48)),
]


def _rows(side, b, t0, n, D):
    return synth.kv_rows(0, side, 0, [b], list(range(H)), list(range(t0, t0 + n)), D, "cuda")[0]


@pytest.mark.parametrize("D,k,v,anc", FORMATS, ids=[f"{d}-{k.fmt}-{v.fmt}" for d, k, v, _ in FORMATS])
def test_append_to_subsets_of_sequences(D, k, v, anc):
    cfg = Config(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=2 * H, head_dim=D, capacity=CAP, k=k, v=v,
                 max_queries=8, **anc)
    cache = KVCache(cfg)
    lens = [0] * B
    # (sequence list or None for all, tokens per listed sequence)
    plan = [(None, 120), ([2, 0], 37), ([3], 1), ([3], 1), ([1, 3, 0], 60), ([2], 200), ([0, 2], 1)]
    for ids, n in plan:
        seqs = list(range(B)) if ids is None else ids
        K = torch.stack([_rows("k", b, lens[b], n, D) for b in seqs]).contiguous()
        V = torch.stack([_rows("v", b, lens[b], n, D) for b in seqs]).contiguous()
        sid = None if ids is None else torch.tensor(ids, dtype=torch.int32, device="cuda")
        cache.append(0, K, V, seq_ids=sid)
        for b in seqs:
            lens[b] += n
    torch.cuda.synchronize()
    assert lens == [218, 180, 358, 182]
    assert cache.view(0, 0, "seq_len").cpu().tolist() == lens
    assert kvq.kvq_error_flags(cache.h) == 0

    # device-side refusals: a listed sequence without room for all its rows gets none of them,
    # an id outside the batch is skipped; the other listed sequences still advance
    K = torch.stack([_rows("k", b, lens[b], 50, D) for b in (2, 1)]).contiguous()
    V = torch.stack([_rows("v", b, lens[b], 50, D) for b in (2, 1)]).contiguous()
    cache.append(0, K, V, seq_ids=torch.tensor([2, 1], dtype=torch.int32, device="cuda"))
    lens[1] += 50
    assert kvq.kvq_error_flags(cache.h) == kvq.ERRF_CAPACITY
    K1 = _rows("k", 3, lens[3], 1, D)[None].contiguous()
    V1 = _rows("v", 3, lens[3], 1, D)[None].contiguous()
    cache.append(0, K1, V1, seq_ids=torch.tensor([7], dtype=torch.int32, device="cuda"))
    assert kvq.kvq_error_flags(cache.h) == kvq.ERRF_SEQ_ID
    assert cache.view(0, 0, "seq_len").cpu().tolist() == lens

    spec = oracle_spec(cfg)
    codes = [cache.view(0, s, "codes").cpu().numpy() for s in (0, 1)]
    q = synth.queries(1, 0, B, cfg.n_q_heads, D, max(lens)).cuda()
    out = cache.decode(0, q).cpu().numpy()
    for b in range(B):
        T = lens[b]
        K16 = synth.kv_rows(0, "k", 0, [b], list(range(H)), list(range(T)), D, "cpu")[0].numpy()
        V16 = synth.kv_rows(0, "v", 0, [b], list(range(H)), list(range(T)), D, "cpu")[0].numpy()
        Ks, Vs = [], []
        for h in range(H):
            kq, vq = OC.quantize_unit(spec, K16[h], V16[h])
            u = b * H + h
            assert np.array_equal(codes[0][u, :T], kq["bytes"]), (b, h, "k")
            assert np.array_equal(codes[1][u, :T], vq["bytes"]), (b, h, "v")
            Kh, Vh = OC.reconstruct_unit(spec, 0, K16[h], V16[h], kq, vq, T)
            Ks.append(Kh)
            Vs.append(Vh)
        ref, _, _ = OA.attention(q[b].cpu().numpy(), np.stack(Ks), np.stack(Vs), T, spec.sm_scale)
        for hq in range(cfg.n_q_heads):
            err = np.abs(out[b, hq] - ref[hq]).max() / np.abs(ref[hq]).max()
            assert err <= TOL, (b, hq, err)
    cache.close()


def test_append_sequence_list_arguments():
    s = Side("int", 4, group=32)
    cfg = Config(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=H, head_dim=128, capacity=64, k=s, v=s)
    cache = KVCache(cfg)
    L = kvq.lib()
    k = torch.zeros(B, H, 1, 128, dtype=torch.float16, device="cuda")
    ids = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    st = kvq._stream(None)
    p = lambda t: kvq._ptr(t)
    assert L.kvq_quantize_append(cache.h, 0, p(k), p(k), None, B - 1, 1, st) == -1   # NULL list needs n_seqs = batch
    assert L.kvq_quantize_append(cache.h, 0, p(k), p(k), p(ids), 0, 1, st) == -1
    assert L.kvq_quantize_append(cache.h, 0, p(k), p(k), p(ids), B + 1, 1, st) == -1
    assert L.kvq_quantize_append(cache.h, 0, p(k), p(k), p(ids), 2, 65, st) == -3    # more rows than capacity
    assert L.kvq_quantize_append(cache.h, 0, p(k), p(k), p(ids), 2, 1, st) == 0
    with pytest.raises(ValueError):
        cache.append(0, k, k, seq_ids=ids)  # 4 sequences of rows for a list of 2
    torch.cuda.synchronize()
    assert cache.view(0, 0, "seq_len").cpu().tolist() == [1, 1, 0, 0]
    # after a per-sequence append the host bound is no longer exact; a full append of 63 rows
    # still fits every sequence and is accepted, and the device keeps each length exact
    k63 = torch.zeros(B, H, 63, 128, dtype=torch.float16, device="cuda")
    cache.append(0, k63, k63)
    torch.cuda.synchronize()
    assert cache.view(0, 0, "seq_len").cpu().tolist() == [64, 64, 63, 63]
    assert kvq.kvq_error_flags(cache.h) == 0
    cache.close()


@pytest.mark.parametrize("D,k,v", [
    (128, Side("nf4", group=64), Side("int", 4, group=64)),                      # one CTA barrier per tile
    (256, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),  # producer warp
])
def test_decode_wait_gives_up_and_reports(D, k, v, monkeypatch):
    """The decode's only wait (a consumer polling the barrier of a staged tile) is bounded.  With
    the test hook the first wait of every CTA polls a barrier nothing arrives on; the kernel must
    report KVQ_ERRF_WAIT_TIMEOUT, write empty partials (out = 0, lse = -inf), let the copies it
    issued land, and leave the context usable."""
    T = 1000
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=8, head_dim=D, capacity=T, k=k, v=v, max_queries=2)
    monkeypatch.setenv("KVQ_TEST_STALL_FIRST_WAIT", "200000")
    stalled = KVCache(cfg)
    monkeypatch.delenv("KVQ_TEST_STALL_FIRST_WAIT")
    normal = KVCache(cfg)
    K = synth.kv_rows(0, "k", 0, [0, 1], [0, 1], list(range(T)), D, "cuda")
    V = synth.kv_rows(0, "v", 0, [0, 1], [0, 1], list(range(T)), D, "cuda")
    for c in (stalled, normal):
        c.append(0, K, V)
    q = synth.queries(1, 0, 2, 8, D, T).cuda()
    out, lse = stalled.decode(0, q, lse=True)
    torch.cuda.synchronize()
    assert kvq.kvq_error_flags(stalled.h) & kvq.ERRF_WAIT_TIMEOUT
    assert torch.all(out == 0) and torch.all(torch.isneginf(lse))
    ref = normal.decode(0, q)
    torch.cuda.synchronize()
    assert kvq.kvq_error_flags(normal.h) == 0
    assert torch.isfinite(ref).all() and ref.abs().max() > 0
    stalled.close()
    normal.close()
