"""The C-ABI library loads, exports every symbol include/kvq.h declares, and rejects bad
configurations on the host (no GPU needed)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from oracle import nf4 as ORACLE_NF4
from quantized_decode_attention_append_b200 import kvq
from quantized_decode_attention_append_b200.kvq import Config, Side

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_symbols():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    return sorted(set(re.findall(r"\b(kvq_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    L = kvq.lib()
    syms = header_symbols()
    assert len(syms) >= 13
    for s in syms:
        assert hasattr(L, s), s
    assert sorted(kvq.EXPORTS) == syms


def base_cfg(**kw):
    c = Config(n_layers=2, batch=2, n_kv_heads=2, n_q_heads=4, head_dim=128, capacity=512,
               k=Side("int", 4, group=32, rot=128), v=Side("int", 4, group=32, rot=128))
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def status_of(cfg):
    c = cfg.to_c()
    n = C.c_uint64(0)
    return kvq.lib().kvq_arena_bytes(C.byref(c), C.byref(n)), n.value


def test_arena_bytes_matches_layout_arithmetic():
    st, n = status_of(base_cfg())
    assert st == 0
    # per layer and side: codes 2*2*512*64, scales 2*2*512*4*2 (256-aligned), then metadata
    per_side = 4 * 512 * 64 + 4 * 512 * 4 * 2
    assert n >= 2 * 2 * per_side and n < 2 * 2 * per_side + 4096


@pytest.mark.parametrize("mut,want", [
    (dict(head_dim=96), -2),
    (dict(n_q_heads=3), -1),
    (dict(n_q_heads=2 * 16), -2),
    (dict(capacity=0), -1),
    (dict(k=Side("int", 9, group=32)), -1),
    (dict(k=Side("int", 4, group=48)), -1),
    (dict(k=Side("int", 4, group=256)), -1),
    (dict(k=Side("int", 4, group=32, rot=256)), -1),
    (dict(v=Side("int", 4, group=32, chan_scale=True)), -1),
    (dict(k=Side("polar", 4, 8, rot=128)), -1),
    (dict(head_dim=256, k=Side("polar", 4, 8), v=Side("polar", 4, 8)), -2),
    (dict(k=Side("nf4", scale="minmax", group=64)), -1),
    (dict(anchor_layers=(5,), anchor_rule="first_n", anchor_n=8), -1),
    (dict(anchor_layers=(0,), anchor_rule="window", anchor_n=0), -1),
    (dict(sm_scale=-1.0), -1),
])
def test_bad_configs_rejected_on_host(mut, want):
    st, _ = status_of(base_cfg(**mut))
    assert st == want


@pytest.mark.parametrize("side", [
    Side("int", 2, group=128, rot=128), Side("int", 3, group=32), Side("int", 8, scale="minmax", group=16),
    Side("nf4", group=64), Side("ternary", group=8), Side("sign", group=4), Side("polar", 5, 7),
    Side("cart", 6), Side("fp16"),
])
def test_good_configs_accepted(side):
    st, n = status_of(base_cfg(k=side, v=side))
    assert st == 0 and n > 0


def test_create_rejects_before_touching_the_device():
    L = kvq.lib()
    c = base_cfg(head_dim=96).to_c()
    h = C.c_void_p()
    assert L.kvq_create(C.byref(c), C.c_void_p(256), 1 << 20, C.byref(h)) == -2
    c = base_cfg().to_c()
    assert L.kvq_create(C.byref(c), C.c_void_p(0), 1 << 20, C.byref(h)) == -1      # null arena
    assert L.kvq_create(C.byref(c), C.c_void_p(4096 + 8), 1 << 30, C.byref(h)) == -1  # misaligned
    assert L.kvq_create(C.byref(c), C.c_void_p(4096), 16, C.byref(h)) == -5         # too small
    assert L.kvq_create(None, C.c_void_p(4096), 16, C.byref(h)) == -1


def test_null_handle_calls_fail_cleanly():
    L = kvq.lib()
    assert L.kvq_quantize_append(None, 0, None, None, None, 1, 1, None) == -1
    assert L.kvq_decode_attention(None, 0, None, 1, None, None, None, 1, None, None) == -1
    assert L.kvq_dequantize(None, 0, 0, 0, 0, 1, None, 1, None) == -1
    assert L.kvq_set_seq_len(None, 0, 0, None) == -1
    L.kvq_free(None)
    assert kvq.kvq_status_str(-3) == "capacity exceeded"


def test_library_nf4_table_equals_oracle_table():
    """The two sides build the NF4 table independently (bisection on erfc vs the stdlib
    inverse CDF); they must agree bit for bit after fp16 rounding."""
    lib_levels = np.array(kvq.kvq_nf4_levels(), dtype=np.float64)
    assert np.array_equal(lib_levels, ORACLE_NF4.nf4_levels())


def layers_status(cfg):
    c = cfg.to_c()
    n = C.c_uint64(0)
    lk, lv = cfg.layer_arrays()
    return kvq.lib().kvq_arena_bytes_layers(C.byref(c), lk, lv, C.byref(n)), n.value


def test_per_layer_formats_arena_bytes():
    """A per-layer table equal to the uniform sides gives the uniform arena; 2-bit K in one
    layer takes exactly the 2-bit codes' bytes there (same groups, same metadata)."""
    s4 = Side("int", 4, group=32, rot=128)
    s2 = Side("int", 2, group=32, rot=128)
    st_u, n_u = status_of(base_cfg())
    st_l, n_l = layers_status(base_cfg(layer_k=(s4, s4), layer_v=(s4, s4)))
    assert st_u == 0 and st_l == 0 and n_u == n_l
    st_m, n_m = layers_status(base_cfg(layer_k=(s2, s4)))
    assert st_m == 0
    units, T = 2 * 2, 512
    assert n_u - n_m == units * T * (128 * 4 // 8 - 128 * 2 // 8)


def test_per_layer_formats_checked_per_entry():
    bad = Side("int", 9, group=32)
    ok = Side("int", 3, group=32)
    assert layers_status(base_cfg(layer_k=(ok, bad)))[0] == -1
    assert layers_status(base_cfg(layer_v=(ok, Side("int", 4, group=32, chan_scale=True))))[0] == -1
    assert layers_status(base_cfg(layer_v=(ok, Side("polar", 4, 8, rot=128))))[0] == -1
    assert layers_status(base_cfg(layer_k=(ok, Side("nf4", group=64)), layer_v=(Side("sign", group=4), ok)))[0] == 0
    # the uniform field is not read where a per-layer array is given
    assert layers_status(base_cfg(k=bad, layer_k=(ok, ok)))[0] == 0
    L = kvq.lib()
    c = base_cfg(head_dim=96).to_c()
    h = C.c_void_p()
    lk, _ = base_cfg(layer_k=(ok, ok)).layer_arrays()
    assert L.kvq_create_layers(C.byref(c), lk, None, C.c_void_p(256), 1 << 20, C.byref(h)) == -2


def test_binding_rejects_bad_tensors_before_the_library():
    """KVCache checks dtype, device, layout and shape on the host (no handle is touched)."""
    import torch
    cache = kvq.KVCache.__new__(kvq.KVCache)
    cache.cfg = base_cfg()
    cache.h = None
    k32 = torch.zeros(2, 2, 3, 128, dtype=torch.float32)
    k16 = torch.zeros(2, 2, 3, 128, dtype=torch.float16)
    with pytest.raises(ValueError, match="fp16 CUDA"):
        cache.append(0, k32, k32)
    with pytest.raises(ValueError, match="fp16 CUDA"):
        cache.append(0, k16, k16)  # host tensor
    with pytest.raises(ValueError, match="q: need"):
        cache.decode(0, torch.zeros(2, 4, 128, dtype=torch.float16))


def test_binding_checks_sequence_list_and_output():
    """The per-sequence append's id list and a caller-supplied decode output are checked on the
    host before the library sees them."""
    import torch
    cache = kvq.KVCache.__new__(kvq.KVCache)
    cache.cfg = base_cfg()
    cache.h = None
    k16 = torch.zeros(1, 2, 3, 128, dtype=torch.float16)
    with pytest.raises(ValueError, match="seq_ids"):
        cache.append(0, k16, k16, seq_ids=torch.zeros(1, dtype=torch.int64))
    with pytest.raises(ValueError, match="seq_ids"):
        cache.append(0, k16, k16, seq_ids=torch.zeros(1, dtype=torch.int32))  # host tensor


def test_header_documents_the_sequence_list():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    decl = text[text.index("kvq_status kvq_quantize_append("):]
    decl = decl[:decl.index(";")]
    assert "const int32_t* seq_ids" in decl and "int32_t n_seqs" in decl and "int32_t n_new" in decl


def test_library_lloyd_tables_equal_oracle_tables():
    """The library iterates Lloyd's conditions in C++ and the oracle in numpy; the fp16 levels
    must agree bit for bit ("E22L" "Result": Gaussian Lloyd-Max levels)."""
    from oracle import lloyd as OL
    for b in (2, 3, 4):
        assert np.array_equal(np.array(kvq.kvq_lloyd_levels(b), dtype=np.float64), OL.lloyd_max_levels(b))
    assert kvq.lib().kvq_lloyd_levels(5, (C.c_float * 32)()) == -1


@pytest.mark.parametrize("mut,want", [
    (dict(v=Side("int", 4, group=32, mean_sub=True)), -1),          # values carry no key mean
    (dict(k=Side("fp16", mean_sub=True)), -1),                     # nothing to subtract it from
    (dict(k=Side("lloyd", 5, group=32)), -1),
    (dict(k=Side("lloyd", 1, group=32)), -1),
    (dict(k=Side("lloyd", 3, scale="minmax", group=32)), -1),
    (dict(k=Side("nf4", scale="sym", group=64)), -1),
])
def test_bad_value_grid_configs(mut, want):
    assert status_of(base_cfg(**mut))[0] == want


@pytest.mark.parametrize("side", [
    Side("int", 2, scale="sym", group=128, rot=128), Side("int", 3, scale="sym", group=32),
    Side("lloyd", 2, group=128, rot=128), Side("lloyd", 4, group=16), Side("int", 4, group=32, mean_sub=True),
])
def test_value_grid_configs_accepted(side):
    v = Side(**{**side.__dict__, "mean_sub": False})
    st, n = status_of(base_cfg(k=side, v=v))
    assert st == 0 and n > 0


def test_key_mean_region_in_the_arena():
    """A K side with mean_sub adds one fp16 vector per (sequence, kv-head) and layer."""
    st0, n0 = status_of(base_cfg())
    st1, n1 = status_of(base_cfg(k=Side("int", 4, group=32, rot=128, mean_sub=True)))
    assert st0 == 0 and st1 == 0
    per_layer = 2 * 2 * 128 * 2  # batch x kv-heads x head_dim x fp16
    assert n1 - n0 == 2 * ((per_layer + 255) // 256 * 256)


@pytest.mark.parametrize("mut,want", [
    (dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=8, anchor_bits=5), -1),
    (dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=8, anchor_bits=8, v=Side("fp16")), -2),
    (dict(anchor_layers=(1,), anchor_rule="window", anchor_n=8, anchor_bits=4, k=Side("polar", 4, 8)), -2),
    (dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=8, anchor_bits=8), 0),
    (dict(anchor_bits=8, v=Side("fp16")), 0),  # no anchored layer: nothing to quantize
])
def test_anchor_precision_configs(mut, want):
    assert status_of(base_cfg(**mut))[0] == want


def test_int_anchor_arena_is_smaller():
    """int8 anchors take half a byte per value plus one fp16 scale per 32 channels, against 2 bytes."""
    kw = dict(anchor_layers=(0, 1), anchor_rule="first_n", anchor_n=256)
    n16 = status_of(base_cfg(**kw))[1]
    n8 = status_of(base_cfg(anchor_bits=8, **kw))[1]
    n4 = status_of(base_cfg(anchor_bits=4, **kw))[1]
    assert n16 > n8 > n4
    assert n16 - n8 == pytest.approx(2 * 2 * 4 * 256 * (128 * 2 - 128 - 8), abs=4 * 512)


def test_sorted_group_configs():
    """Sorted groups (post 6, "The winning recipe" item 1): 2..4 bits, a zero point per group, the
    ranks in ceil(log2 D) bits per value after the codes."""
    ok = Side("sorted", 2, group=8)
    assert status_of(base_cfg(k=ok, v=Side("sorted", 2, group=4)))[0] == 0
    assert status_of(base_cfg(k=Side("sorted", 5, group=8)))[0] == -1
    assert status_of(base_cfg(k=Side("sorted", 2, scale="minmax", group=8)))[0] == -1
    assert status_of(base_cfg(k=ok, anchor_layers=(0,), anchor_rule="first_n", anchor_n=8, anchor_bits=8))[0] == -2
    st, n = status_of(base_cfg(k=ok, v=ok))
    st4, n4 = status_of(base_cfg(k=Side("int", 2, scale="minmax", group=8), v=Side("int", 2, scale="minmax", group=8)))
    # per row: the same codes and metadata plus 7 x 128 rank bits (112 bytes)
    assert st == 0 and st4 == 0 and n - n4 == pytest.approx(2 * 2 * 4 * 512 * 112, abs=2 * 2 * 3 * 256)


def test_head_allocation_matches_the_oracle_rule():
    """The package's calibration (torch) and the oracle's rule (numpy) agree: entropies of the same
    attention, bits per head, and the sink heads (llama.cpp #21385 "Finding 2")."""
    import torch
    from oracle import attention as OA
    from oracle import headalloc as OH
    from quantized_decode_attention_append_b200 import headalloc as HA
    r = np.random.default_rng(5)
    L, H, G, T, D = 3, 4, 2, 60, 32
    H2 = np.zeros((L, H))
    for l in range(L):
        K = (r.standard_normal((H, T, D)) * (1 + l)).astype(np.float16)
        q = (r.standard_normal((6, H * G, D)) * np.linspace(0.2, 3, H * G)[None, :, None]).astype(np.float16)
        kv = [60, 31, 7, 60, 45, 12]
        got = HA.head_entropy(torch.from_numpy(q), torch.from_numpy(K), kv)
        want = np.zeros(H)
        for i in range(6):
            _, _, P = OA.attention(q[i], K, K, kv[i])
            for hq in range(H * G):
                want[hq // G] += OH.renyi2(P[hq]) / (6 * G)
        assert np.allclose(got.numpy(), want, rtol=1e-9, atol=1e-9)
        H2[l] = want
    hk, hv, bits = HA.allocate(H2, 4.0, sink_frac=0.1)
    want_bits = OH.head_bits(H2.reshape(-1), 4.0).reshape(L, H)
    sinks = set(OH.sink_heads(H2.reshape(-1), 0.1).tolist())
    assert len(sinks) == 1
    for l in range(L):
        for h in range(H):
            if l * H + h in sinks:
                assert bits[l][h] == 16 and hk[l][h].fmt == "fp16"
            else:
                assert bits[l][h] == want_bits[l, h] and hk[l][h].bits == want_bits[l, h]
    assert hk == hv


def test_decode_source_hash_covers_every_local_header_of_the_decode_unit():
    """bench.py keys the committed DRAM-traffic summary to a hash of the decode kernels' sources:
    every csrc header the decode translation unit includes (directly or through another header)
    must be in that list, or a kernel change could leave a stale traffic number in the bench line."""
    import bench
    csrc = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                        "quantized_decode_attention_append_b200", "csrc")
    seen, todo = set(), ["decode.cu"]
    while todo:
        f = todo.pop()
        if f in seen:
            continue
        seen.add(f)
        for inc in re.findall(r'^#include "([^"/]+)"', open(os.path.join(csrc, f)).read(), re.M):
            if os.path.exists(os.path.join(csrc, inc)):
                todo.append(inc)
    assert seen <= set(bench.DECODE_SOURCES), sorted(seen - set(bench.DECODE_SOURCES))
