"""Full-size parity: the workloads bench.py times, filled and decoded exactly as bench.py does
(bulk prefill, then one-token appends, then decode through kvq_decode_attention), checked on
sampled (layer, sequence, kv-head) units against the oracle: packed codes and scales bit for bit
on sampled rows, attention within 2e-3 for every query head of the sampled units.
"""
import numpy as np
import pytest
import torch

import bench
from kvq_harness import TOL, oracle_spec
from oracle import attention as OA
from oracle import cache as OC
from quantized_decode_attention_append_b200 import synth
from quantized_decode_attention_append_b200.kvq import KVCache

pytestmark = pytest.mark.gpu


def test_generator_gpu_equals_cpu():
    """The seeded inputs are bit-identical on the GPU and the CPU (the oracle's copy)."""
    for side in ("k", "v"):
        g = synth.kv_rows(3, side, 5, [0, 7], [1, 2], list(range(0, 4000, 7)), 128, "cuda").cpu()
        c = synth.kv_rows(3, side, 5, [0, 7], [1, 2], list(range(0, 4000, 7)), 128, "cpu")
        assert torch.equal(g.view(torch.int16), c.view(torch.int16))
    qg = synth.queries(1, 4, 3, 32, 256, 65536, "cuda").cpu()
    qc = synth.queries(1, 4, 3, 32, 256, 65536, "cpu")
    assert torch.equal(qg.view(torch.int16), qc.view(torch.int16))


def run_full(name, samples, n_append=1):
    w = dict(bench.WORKLOADS[name])
    L, B, Hkv, Hq, D, T = w["L"], w["B"], w["Hkv"], w["Hq"], w["D"], w["T"]
    cfg = bench.make_config(w, T)
    cache = KVCache(cfg, "cuda")
    T0 = T - n_append
    bench.fill_cache(cache, w, T0, seed=0, device="cuda")
    for l in range(L):  # decode-time appends, as in a bench step
        for t in range(T0, T):
            kn = synth.kv_rows(0, "k", l, list(range(B)), list(range(Hkv)), [t], D, "cuda")
            vn = synth.kv_rows(0, "v", l, list(range(B)), list(range(Hkv)), [t], D, "cuda")
            cache.append(l, kn, vn)
    spec = oracle_spec(cfg)
    G = Hq // Hkv
    worst = 0.0
    rng = np.random.default_rng(7)
    for (l, b, h) in samples:
        q = synth.queries(1, l, B, Hq, D, T).cuda()
        out = cache.decode(l, q).cpu().numpy()
        K16 = synth.kv_rows(0, "k", l, [b], [h], list(range(T)), D, "cpu")[0, 0].numpy()
        V16 = synth.kv_rows(0, "v", l, [b], [h], list(range(T)), D, "cpu")[0, 0].numpy()
        kq, vq = OC.quantize_unit(spec, K16, V16)
        u = b * Hkv + h
        rows = np.unique(np.concatenate([rng.integers(0, T, 512), [0, 1, T0 - 1, T - 1]]))
        for side, o in ((0, kq), (1, vq)):
            got = cache.view(l, side, "codes")[u, :T].cpu().numpy()
            assert np.array_equal(got[rows], o["bytes"][rows]), (name, l, b, h, side)
            sc = cache.view(l, side, "scales")
            if sc is not None:
                assert np.array_equal(sc[u, :T].cpu().numpy()[rows].view(np.uint16),
                                      o["scales"][rows].view(np.uint16)), (name, l, b, h, side, "scales")
        Kh, Vh = OC.reconstruct_unit(spec, l, K16, V16, kq, vq, T)
        qn = q.cpu().numpy()[b, h * G:(h + 1) * G]
        ref, _, _ = OA.attention(qn, Kh[None], Vh[None], T, spec.sm_scale)
        for j in range(G):
            err = np.abs(out[b, h * G + j] - ref[j]).max() / np.abs(ref[j]).max()
            worst = max(worst, err)
            assert err <= TOL, (name, l, b, h, j, err)
    cache.close()
    return worst


def test_fullsize_stress_nf4():
    """32 layers x 16 sequences x 8 kv-heads x 32768 tokens, NF4 K + int4 V (18.3 GB packed)."""
    run_full("stress-nf4", [(0, 0, 0), (31, 15, 7), (17, 9, 3)])


def test_fullsize_stress_ternary_anchors():
    """Ternary g8 with fp16 anchors on layer 0, tokens < 48."""
    run_full("stress-ternary", [(0, 3, 5), (1, 3, 5)])


def test_fullsize_stress_sign():
    run_full("stress-sign", [(5, 1, 2)])


@pytest.mark.parametrize("name", ["64k-A", "64k-konly", "64k-v3"])
def test_fullsize_64k(name):
    """8 layers x 4 kv-heads x 16 query heads x 65536 tokens, rotated 4-bit K with 2-bit,
    fp16 or 3-bit V."""
    run_full(name, [(0, 0, 0), (7, 0, 3)])


CFG2_VARIANTS = {  # "E21W" variants at 3 and 4 bits, groups of 32, head_dim 256
    "A": dict(rot=0, chan_scale=False), "B": dict(rot=256, chan_scale=False),
    "C": dict(rot=0, chan_scale=True), "D": dict(rot=256, chan_scale=True),
}


@pytest.mark.parametrize("variant", list(CFG2_VARIANTS))
@pytest.mark.parametrize("bits", [3, 4])
def test_fullsize_proxy_query_slice(variant, bits):
    """8 layers x 4 kv-heads, head_dim 256, 6000 tokens, per-token min-max g32; 128 proxy queries
    (post-RoPE keys at positions drawn from [3000, 6000), causal over earlier keys)."""
    from kvq_harness import Case
    from quantized_decode_attention_append_b200.kvq import Config, Side
    v = CFG2_VARIANTS[variant]
    k = Side("int", bits, scale="minmax", group=32, rot=v["rot"], chan_scale=v["chan_scale"])
    vs = Side("int", bits, scale="minmax", group=32, rot=v["rot"])
    cfg = Config(n_layers=8, batch=1, n_kv_heads=4, n_q_heads=4, head_dim=256, capacity=6000, k=k, v=vs,
                 max_queries=128)
    c = Case(cfg, 6000, calib_T=6000)
    pos = synth.proxy_positions(1, 128, 3000, 6000)
    for l in (0, 7):
        q = torch.from_numpy(c.K[l][0][:, pos].transpose(1, 0, 2).copy())
        c.decode_and_compare(l, q, seq_ids=[0] * 128, kv_len=pos.tolist())


@pytest.mark.parametrize("arm", [("polar", 4, 8), ("polar", 6, 6), ("cart", 6, 0), ("int", 6, 0)])
def test_fullsize_fourier_polar(arm):
    """32 layers x 8 kv-heads, head_dim 128, 8192 tokens; rFFT polar (mag/phase bit split),
    Cartesian and Hadamard-128 int6 controls at 6.125 bits; sampled layers."""
    from kvq_harness import Case
    from quantized_decode_attention_append_b200.kvq import Config, Side
    fmt, b1, b2 = arm
    s = Side("int", 6, group=128, rot=128) if fmt == "int" else Side(fmt, b1, b2)
    cfg = Config(n_layers=32, batch=1, n_kv_heads=8, n_q_heads=8, head_dim=128, capacity=8192, k=s, v=s,
                 max_queries=129)
    c = Case(cfg, 8192, layers=[0, 31])
    pos = synth.proxy_positions(1, 128, 4096, 8192)
    for l in (0, 31):
        qp = torch.from_numpy(c.K[l][0][:, pos].transpose(1, 0, 2).copy())
        qd = synth.queries(1, l, 1, 8, 128, 8192)
        q = torch.cat([qd, qp[:16]], dim=0)
        c.check_codes(l, rows=np.arange(0, 8192, 97))
        c.decode_and_compare(l, q, seq_ids=[0] * 17, kv_len=[8192] + pos[:16].tolist())
