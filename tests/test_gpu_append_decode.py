"""kvq_append_decode: one decode step (append each listed sequence's new rows, then decode one
query per listed sequence over its whole new length) in one split-K launch where the layer
allows it.  It must leave the cache and give the outputs of kvq_quantize_append followed by
kvq_decode_attention, and match the CPU oracle ("E22L" "What I tested": keys and values
quantized on entry to the cache; "Fourier Magnitude KV Cache Quantization" post 6, "The
winning recipe", component 2: generated tokens appended, some anchored, then attended).
"""
import numpy as np
import pytest
import torch

from kvq_harness import TOL, oracle_spec
from oracle import attention as OA
from oracle import cache as OC
from quantized_decode_attention_append_b200 import kvq, synth
from quantized_decode_attention_append_b200.kvq import Config, KVCache, Side

pytestmark = pytest.mark.gpu

B, H = 3, 2

# (head_dim, GQA group, K, V, anchors, fused) -- fused: a register-decode instance serves the pair
FORMATS = [
    (128, 4, Side("nf4", group=64), Side("int", 4, group=64), {}, True),
    (128, 4, Side("int", 4, group=64), Side("int", 4, group=64), {}, True),
    (128, 2, Side("int", 4, group=32), Side("int", 4, group=32), {}, True),
    (128, 4, Side("sign", group=4), Side("sign", group=4), {}, True),
    (128, 4, Side("ternary", group=8), Side("ternary", group=8),
     dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=40), True),
    (128, 4, Side("ternary", group=8), Side("ternary", group=8),
     dict(anchor_layers=(0,), anchor_rule="window", anchor_n=24), True),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256), {}, True),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 2, scale="sym", group=128, rot=256), {}, True),
    (256, 4, Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256), {}, True),
    (256, 4, Side("int", 4, group=128, rot=256), Side("fp16"), {}, True),
    (128, 1, Side("polar", 4, 8), Side("polar", 4, 8), {}, False),          # no register-decode instance
    (128, 4, Side("nf4", group=64, mean_sub=True), Side("int", 4, group=64), {}, False),  # key mean
]


def _rows(side, b, t0, n, D):
    return synth.kv_rows(0, side, 0, [b], list(range(H)), list(range(t0, t0 + n)), D, "cuda")[0]


def _pair(D, G, k, v, anc, cap):
    cfg = Config(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=H * G, head_dim=D, capacity=cap, k=k, v=v,
                 max_queries=8, **anc)
    return cfg, KVCache(cfg), KVCache(cfg)


def _step_rows(seqs, lens, n, D):
    K = torch.stack([_rows("k", b, lens[b], n, D) for b in seqs]).contiguous()
    V = torch.stack([_rows("v", b, lens[b], n, D) for b in seqs]).contiguous()
    return K, V


def _same_cache(a, b, lens):
    """Codes, scales and anchor rows of every stored token, and the lengths, equal."""
    n_anch = a.cfg.anchor_n if a.cfg.anchor_layers else 0
    for side in (0, 1):
        ca, cb = a.view(0, side, "codes"), b.view(0, side, "codes")
        sa, sb = a.view(0, side, "scales"), b.view(0, side, "scales")
        aa, ab = a.view(0, side, "anchors"), b.view(0, side, "anchors")
        for s in range(B):
            for h in range(H):
                u = s * H + h
                T = lens[s]
                assert torch.equal(ca[u, :T], cb[u, :T]), ("codes", side, s, h)
                if sa is not None:
                    assert torch.equal(sa[u, :T], sb[u, :T]), ("scales", side, s, h)
                if aa is not None:
                    m = min(n_anch, T)
                    assert torch.equal(aa[u, :m], ab[u, :m]), ("anchors", side, s, h)
    assert a.view(0, 0, "seq_len").cpu().tolist() == b.view(0, 0, "seq_len").cpu().tolist() == lens


@pytest.mark.parametrize("D,G,k,v,anc,fused", FORMATS,
                         ids=[f"{d}G{g}-{k.fmt}{k.bits}-{v.fmt}{v.bits}{'-' + a['anchor_rule'] if a else ''}"
                              f"{'-mean' if k.mean_sub else ''}" for d, g, k, v, a, _ in FORMATS])
def test_fused_step_equals_append_then_decode(D, G, k, v, anc, fused):
    cfg, A, Bc = _pair(D, G, k, v, anc, 400)
    lens = [0] * B
    # prefill: different lengths per sequence (bulk appends to subsets)
    for ids, n in ((None, 150), ([0, 2], 61), ([1], 17)):
        seqs = list(range(B)) if ids is None else ids
        K, V = _step_rows(seqs, lens, n, D)
        sid = None if ids is None else torch.tensor(ids, dtype=torch.int32, device="cuda")
        A.append(0, K, V, seq_ids=sid)
        Bc.append(0, K, V, seq_ids=sid)
        for b in seqs:
            lens[b] += n
    # decode steps: all sequences, a subset, then two tokens at once
    for step, (ids, n) in enumerate(((None, 1), ([2, 0], 1), (None, 1), ([1], 2))):
        seqs = list(range(B)) if ids is None else ids
        K, V = _step_rows(seqs, lens, n, D)
        q = synth.queries(1, step, len(seqs), cfg.n_q_heads, D, 1000 + step).cuda()
        sid = None if ids is None else torch.tensor(ids, dtype=torch.int32, device="cuda")
        out_a, lse_a = A.append_decode(0, K, V, q, seq_ids=sid, lse=True)
        na = kvq.kvq_last_launch_count(A.h)
        Bc.append(0, K, V, seq_ids=sid)
        out_b, lse_b = Bc.decode(0, q, seq_ids=sid, lse=True)
        for b in seqs:
            lens[b] += n
        torch.cuda.synchronize()
        torch.testing.assert_close(out_a, out_b, rtol=1e-6, atol=1e-6)
        torch.testing.assert_close(lse_a, lse_b, rtol=1e-6, atol=1e-6)
        if fused:
            assert na == (3 if cfg.anchor_layers else 2), na  # split pass (+ anchor pass) + merge
        else:
            assert na > 2, na
    _same_cache(A, Bc, lens)
    assert kvq.kvq_error_flags(A.h) == 0
    A.close()
    Bc.close()


def test_fused_step_against_oracle():
    """NF4-K g64 + int4-g64 V (the batch-16 stress formats) after fused steps: codes bit-exact and
    attention within tolerance of the oracle on every sequence's whole cache."""
    D, G = 128, 4
    cfg = Config(n_layers=1, batch=B, n_kv_heads=H, n_q_heads=H * G, head_dim=D, capacity=300,
                 k=Side("nf4", group=64), v=Side("int", 4, group=64), max_queries=8)
    cache = KVCache(cfg)
    lens = [0] * B
    K, V = _step_rows(range(B), lens, 200, D)
    cache.append(0, K, V)
    lens = [200] * B
    out = None
    for step in range(3):
        K, V = _step_rows(range(B), lens, 1, D)
        q = synth.queries(1, step, B, cfg.n_q_heads, D, 201 + step).cuda()
        out = cache.append_decode(0, K, V, q)
        lens = [x + 1 for x in lens]
    assert kvq.kvq_last_launch_count(cache.h) == 2
    spec = oracle_spec(cfg)
    codes = [cache.view(0, s, "codes").cpu().numpy() for s in (0, 1)]
    out = out.cpu().numpy()
    for b in range(B):
        T = lens[b]
        K16 = synth.kv_rows(0, "k", 0, [b], list(range(H)), list(range(T)), D, "cpu")[0].numpy()
        V16 = synth.kv_rows(0, "v", 0, [b], list(range(H)), list(range(T)), D, "cpu")[0].numpy()
        Ks, Vs = [], []
        for h in range(H):
            kq, vq = OC.quantize_unit(spec, K16[h], V16[h])
            assert np.array_equal(codes[0][b * H + h, :T], kq["bytes"]), (b, h, "k")
            assert np.array_equal(codes[1][b * H + h, :T], vq["bytes"]), (b, h, "v")
            Kh, Vh = OC.reconstruct_unit(spec, 0, K16[h], V16[h], kq, vq, T)
            Ks.append(Kh)
            Vs.append(Vh)
        q = synth.queries(1, 2, B, cfg.n_q_heads, D, 203)[b].numpy()
        ref, _, _ = OA.attention(q, np.stack(Ks), np.stack(Vs), T, spec.sm_scale)
        for hq in range(cfg.n_q_heads):
            err = np.abs(out[b, hq] - ref[hq]).max() / np.abs(ref[hq]).max()
            assert err <= TOL, (b, hq, err)
    cache.close()


def test_fused_step_refuses_a_full_sequence():
    """A listed sequence without room gets none of its rows and is decoded over its old rows
    (KVQ_ERRF_CAPACITY); the other sequences advance."""
    D, G, cap = 128, 4, 160
    cfg, A, Bc = _pair(D, G, Side("nf4", group=64), Side("int", 4, group=64), {}, cap)
    lens = [0] * B
    K, V = _step_rows(range(B), lens, 100, D)
    A.append(0, K, V)
    Bc.append(0, K, V)
    lens = [100] * B
    K, V = _step_rows([1], lens, cap - 100, D)  # sequence 1 full
    sid = torch.tensor([1], dtype=torch.int32, device="cuda")
    A.append(0, K, V, seq_ids=sid)
    Bc.append(0, K, V, seq_ids=sid)
    lens[1] = cap
    K, V = _step_rows(range(B), lens, 1, D)
    q = synth.queries(1, 5, B, cfg.n_q_heads, D, 500).cuda()
    out_a = A.append_decode(0, K, V, q)
    assert kvq.kvq_error_flags(A.h) == kvq.ERRF_CAPACITY
    Bc.append(0, K, V)
    assert kvq.kvq_error_flags(Bc.h) == kvq.ERRF_CAPACITY
    out_b = Bc.decode(0, q)
    lens = [101, cap, 101]
    torch.testing.assert_close(out_a, out_b, rtol=1e-6, atol=1e-6)
    _same_cache(A, Bc, lens)
    A.close()
    Bc.close()


def test_multi_wave_step_runs_the_two_calls():
    """A split-K grid of more than one wave (batch 16 x 8 kv-heads, capacity 32768) takes the
    two calls inside kvq_append_decode, with the same results, also for a subset of sequences
    appending two tokens each."""
    D, G, Bb, Hh, T0 = 128, 4, 16, 8, 1000
    cfg = Config(n_layers=1, batch=Bb, n_kv_heads=Hh, n_q_heads=Hh * G, head_dim=D, capacity=32768,
                 k=Side("nf4", group=64), v=Side("int", 4, group=64), max_queries=Bb)
    A, Bc = KVCache(cfg), KVCache(cfg)
    rows = lambda side, t0, n: synth.kv_rows(0, side, 0, list(range(Bb)), list(range(Hh)),
                                             list(range(t0, t0 + n)), D, "cuda")
    A.append(0, rows("k", 0, T0), rows("v", 0, T0))
    Bc.append(0, rows("k", 0, T0), rows("v", 0, T0))
    q = synth.queries(1, 0, Bb, cfg.n_q_heads, D, T0 + 1).cuda()
    out_a = A.append_decode(0, rows("k", T0, 1), rows("v", T0, 1), q)
    assert kvq.kvq_last_launch_count(A.h) == 3  # append, split pass, merge
    Bc.append(0, rows("k", T0, 1), rows("v", T0, 1))
    out_b = Bc.decode(0, q)
    torch.testing.assert_close(out_a, out_b, rtol=0, atol=0)
    assert A.view(0, 0, "seq_len").cpu().tolist() == [T0 + 1] * Bb
    # a second step on half of the sequences, two tokens each
    ids = list(range(0, Bb, 2))
    sid = torch.tensor(ids, dtype=torch.int32, device="cuda")
    k2 = synth.kv_rows(0, "k", 0, ids, list(range(Hh)), [T0 + 1, T0 + 2], D, "cuda")
    v2 = synth.kv_rows(0, "v", 0, ids, list(range(Hh)), [T0 + 1, T0 + 2], D, "cuda")
    q2 = synth.queries(1, 1, len(ids), cfg.n_q_heads, D, T0 + 3).cuda()
    out_a = A.append_decode(0, k2, v2, q2, seq_ids=sid)
    Bc.append(0, k2, v2, seq_ids=sid)
    out_b = Bc.decode(0, q2, seq_ids=sid)
    torch.testing.assert_close(out_a, out_b, rtol=0, atol=0)
    lens = [T0 + 3 if b % 2 == 0 else T0 + 1 for b in range(Bb)]
    assert A.view(0, 0, "seq_len").cpu().tolist() == Bc.view(0, 0, "seq_len").cpu().tolist() == lens
    for side in (0, 1):
        for what in ("codes", "scales"):
            va, vb = A.view(0, side, what), Bc.view(0, side, what)
            for b in range(Bb):
                u = slice(b * Hh, (b + 1) * Hh)
                assert torch.equal(va[u, :lens[b]], vb[u, :lens[b]]), (side, what, b)
    assert kvq.kvq_error_flags(A.h) == 0
    A.close()
    Bc.close()


def test_per_head_formats_step_runs_the_two_calls():
    """A layer with per-head formats (two head groups) takes the two calls inside
    kvq_append_decode, with the results of kvq_quantize_append then kvq_decode_attention."""
    a, s = Side("int", 4, group=32), Side("sign", group=4)
    cfg = Config(n_layers=1, batch=3, n_kv_heads=2, n_q_heads=8, head_dim=128, capacity=256, k=a, v=a,
                 max_queries=4, head_k=((a, s),), head_v=((a, s),))
    A, Bc = KVCache(cfg), KVCache(cfg)
    lens = [0] * 3
    K, V = _step_rows(range(3), lens, 90, 128)
    A.append(0, K, V)
    Bc.append(0, K, V)
    lens = [90] * 3
    K, V = _step_rows(range(3), lens, 1, 128)
    q = synth.queries(1, 0, 3, cfg.n_q_heads, 128, 91).cuda()
    out_a = A.append_decode(0, K, V, q)
    assert kvq.kvq_last_launch_count(A.h) > 3  # one append and one decode per head group
    Bc.append(0, K, V)
    out_b = Bc.decode(0, q)
    torch.testing.assert_close(out_a, out_b, rtol=0, atol=0)
    assert A.view(0, 0, "seq_len").cpu().tolist() == [91] * 3
    A.close()
    Bc.close()


def test_append_decode_argument_errors():
    """Host-side refusals of kvq_append_decode, before any launch."""
    cfg = Config(n_layers=1, batch=2, n_kv_heads=2, n_q_heads=8, head_dim=128, capacity=64,
                 k=Side("nf4", group=64), v=Side("int", 4, group=64), max_queries=2)
    c = KVCache(cfg)
    L = kvq.lib()
    p = kvq._ptr
    k = torch.zeros(2, 2, 1, 128, dtype=torch.float16, device="cuda")
    q = torch.zeros(2, 8, 128, dtype=torch.float16, device="cuda")
    out = torch.empty(2, 8, 128, dtype=torch.float32, device="cuda")
    st = kvq._stream(None)
    ids3 = torch.tensor([0, 1, 1], dtype=torch.int32, device="cuda")
    assert L.kvq_append_decode(c.h, 0, p(k), p(k), None, 1, 1, p(q), p(out), 1, None, st) == -1      # NULL list: n_seqs = batch
    assert L.kvq_append_decode(c.h, 1, p(k), p(k), None, 2, 1, p(q), p(out), 1, None, st) == -1      # no such layer
    assert L.kvq_append_decode(c.h, 0, p(k), p(k), None, 2, 0, p(q), p(out), 1, None, st) == -1      # no rows
    assert L.kvq_append_decode(c.h, 0, p(k), p(k), None, 2, 1, None, p(out), 1, None, st) == -1      # no queries
    assert L.kvq_append_decode(c.h, 0, p(k), p(k), p(ids3), 3, 1, p(q), p(out), 1, None, st) == -1   # more ids than batch
    assert L.kvq_append_decode(c.h, 0, p(k), p(k), None, 2, 65, p(q), p(out), 1, None, st) == -3     # more rows than capacity
    with pytest.raises(ValueError):
        c.append_decode(0, k, k, q[:1])  # one query for two sequences
    assert kvq.kvq_last_launch_count(c.h) >= 0
    torch.cuda.synchronize()
    assert c.view(0, 0, "seq_len").cpu().tolist() == [0, 0]
    c.close()
