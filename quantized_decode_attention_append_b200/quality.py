"""Quality metrics of the quantized cache on the synthetic workloads (GPU).

The pages' metrics ("E21W" "What I tested"; "E22L" "Result"):
  X1  K / V error: squared error over signal energy, sum (x - x_hat)^2 / sum x^2
  X2  attention-output error: ||o_q - o_f16||_2 / ||o_f16||_2 per (query, head), mean
  X3  attention KL: sum_t p_f16(t) ln(p_f16(t) / p_q(t)) per (query, head), mean
  X5  effective bits per value, scales and anchors included (K and V averaged)
o_q comes from kvq_decode_attention; x_hat from kvq_dequantize (original domain, anchors applied).
The fp16 reference attention and the quantized attention distribution p_q (softmax of q . k_hat)
are computed here with plain fp32 torch math: they are the measuring stick, not the product path.

usage: python -m quantized_decode_attention_append_b200.quality [--config 2|3|4|5|1] [--json out.json]
"""
from __future__ import annotations

import argparse
import json
import math

import torch

from . import synth
from .kvq import DOMAIN_ORIGINAL, Config, KVCache, Side


def eff_bits(cache, cfg, T, anchored_rows_by_layer):
    tot = 0.0
    for l in range(cfg.n_layers):
        a = anchored_rows_by_layer.get(l, 0)
        for side, sd in ((0, cfg.k), (1, cfg.v)):
            lo = cache.layout(l, side)
            per_row = 8 * lo.row_bytes + 16 * lo.n_groups * (2 if lo.zeros >= 0 else 1)
            if sd.fmt == "ternary":
                per_row = 8 * lo.row_bytes + 16 * lo.n_groups
            tot += (T - a) * per_row + a * 16 * cfg.head_dim
            if side == 0 and sd.chan_scale:
                tot += 16 * cfg.head_dim / cfg.batch
    return tot / (cfg.n_layers * 2 * T * cfg.head_dim)


def measure(cfg: Config, T: int, layers, queries_fn, calib_T=512, seed=0):
    """Fill `layers` of a cache, decode the queries queries_fn(layer, K) -> (q [n, Hq, D] fp16,
    seq_ids, kv_len), or a dict of such query sets by suffix, and return the mean metrics over
    layers, units, queries and heads (X2 and X3 once per query set, keys suffixed)."""
    dev = "cuda"
    cache = KVCache(cfg, dev)
    B, H, Hq, D = cfg.batch, cfg.n_kv_heads, cfg.n_q_heads, cfg.head_dim
    G = Hq // H
    sm = cfg.sm_scale or 1.0 / math.sqrt(D)
    x1k, x1v, x2, x3 = [], [], {}, {}
    for l in layers:
        K = synth.kv_rows(seed, "k", l, list(range(B)), list(range(H)), list(range(T)), D, dev)
        V = synth.kv_rows(seed, "v", l, list(range(B)), list(range(H)), list(range(T)), D, dev)
        if cfg.k.chan_scale:
            cache.set_chan_scale(l, synth.channel_scale(seed, l, H, calib_T, D).to(dev))
        cache.append(l, K, V)
        Kh = cache.dequantize(l, 0, 0, T, domain=DOMAIN_ORIGINAL)  # [B, H, T, D] fp32
        Vh = cache.dequantize(l, 1, 0, T, domain=DOMAIN_ORIGINAL)
        Kf, Vf = K.float(), V.float()
        x1k.append(((Kf - Kh) ** 2).sum(dim=(2, 3)) / (Kf ** 2).sum(dim=(2, 3)))
        x1v.append(((Vf - Vh) ** 2).sum(dim=(2, 3)) / (Vf ** 2).sum(dim=(2, 3)))
        sets = queries_fn(l, K)
        if not isinstance(sets, dict):
            sets = {"": sets}
        for tag, (q, seq_ids, kv_len) in sets.items():
            n = q.shape[0]
            sid = torch.tensor(seq_ids, dtype=torch.int32, device=dev)
            kl = torch.tensor(kv_len, dtype=torch.int32, device=dev)
            out = cache.decode(l, q.to(dev), sid, kl)  # [n, Hq, D]
            for i in range(n):
                b, L_ = seq_ids[i], kv_len[i]
                qi = q[i].to(dev).float()  # [Hq, D]
                kh = Kh[b].repeat_interleave(G, dim=0)[:, :L_]  # [Hq, L, D]
                kf = Kf[b].repeat_interleave(G, dim=0)[:, :L_]
                vf = Vf[b].repeat_interleave(G, dim=0)[:, :L_]
                lf = torch.einsum("hd,htd->ht", qi, kf) * sm
                lq = torch.einsum("hd,htd->ht", qi, kh) * sm
                pf = torch.softmax(lf.double(), dim=-1)
                lpq = torch.log_softmax(lq.double(), dim=-1)
                of = torch.einsum("ht,htd->hd", pf.float(), vf)
                x2.setdefault(tag, []).append((torch.linalg.norm(out[i] - of, dim=-1) / torch.linalg.norm(of, dim=-1)).cpu())
                x3.setdefault(tag, []).append((pf * (torch.log(pf.clamp_min(1e-300)) - lpq)).sum(dim=-1).cpu())
    anchored = {}
    if cfg.anchor_rule == "first_n":
        anchored = {l: cfg.anchor_n for l in cfg.anchor_layers}
    elif cfg.anchor_rule == "all":
        anchored = {l: T for l in cfg.anchor_layers}
    bits = eff_bits(cache, cfg, T, anchored)
    cache.close()
    cat = lambda xs: torch.cat([x.flatten().cpu() for x in xs])
    res = {"X1_K": cat(x1k).mean().item(), "X1_V": cat(x1v).mean().item()}
    for tag in x2:
        res["X2_attn_err" + tag] = cat(x2[tag]).mean().item()
        res["X3_KL" + tag] = cat(x3[tag]).mean().item()
    res["X5_bits"] = bits
    return res


def proxy_queries(K, b, pos, G):
    """Proxy queries ("E21W" "What I tested"): the keys of sequence b at positions `pos`, each
    kv-head's key serving its G query heads, attending the keys before it."""
    q = K[b][:, pos].transpose(0, 1).repeat_interleave(G, dim=1).contiguous().cpu()  # [n, Hq, D]
    return q, [b] * len(pos), pos.tolist()


def config2():
    res = {}
    pos = synth.proxy_positions(1, 128, 3000, 6000)
    for bits in (3, 4):
        for name, rot, cs in (("A min-max", 0, False), ("B H256", 256, False), ("C chan-scale", 0, True),
                              ("D chan-scale+H256", 256, True)):
            k = Side("int", bits, scale="minmax", group=32, rot=rot, chan_scale=cs)
            v = Side("int", bits, scale="minmax", group=32, rot=rot)
            cfg = Config(n_layers=8, batch=1, n_kv_heads=4, n_q_heads=4, head_dim=256, capacity=6000, k=k, v=v,
                         max_queries=128)
            qf = lambda l, K: proxy_queries(K, 0, pos, 1)
            res[f"{bits}-bit {name}"] = measure(cfg, 6000, range(8), qf, calib_T=6000)
    return res


def config3():
    res = {}
    arms = {
        "A: H256 4-bit K + 2-bit V g128": (Side("int", 4, group=128, rot=256), Side("int", 2, group=128, rot=256)),
        "K-only: H256 4-bit K g128, fp16 V": (Side("int", 4, group=128, rot=256), Side("fp16")),
        "D': H256 4-bit K + 3-bit V g128": (Side("int", 4, group=128, rot=256), Side("int", 3, group=128, rot=256)),
        "plain 4-bit g32 K and V": (Side("int", 4, group=32), Side("int", 4, group=32)),
    }
    pos = synth.proxy_positions(1, 128, 32768, 65536)
    for name, (k, v) in arms.items():
        cfg = Config(n_layers=8, batch=1, n_kv_heads=4, n_q_heads=16, head_dim=256, capacity=65536, k=k, v=v,
                     max_queries=128)
        qf = lambda l, K: {"": (synth.queries(1, l, 1, 16, 256, 65536), [0], [65536]),
                           "_proxy": proxy_queries(K, 0, pos, 4)}
        res[name] = measure(cfg, 65536, (0, 3, 7), qf)
    return res


def config4():
    res = {}
    pos = synth.proxy_positions(1, 128, 4096, 8192)
    arms = {f"polar {bm}+{bp}": Side("polar", bm, bp) for bm, bp in ((4, 8), (5, 7), (6, 6), (7, 5), (8, 4))}
    arms["Cartesian int6"] = Side("cart", 6)
    arms["H128 int6 g128"] = Side("int", 6, group=128, rot=128)
    for name, s in arms.items():
        cfg = Config(n_layers=32, batch=1, n_kv_heads=8, n_q_heads=8, head_dim=128, capacity=8192, k=s, v=s,
                     max_queries=129)

        def qf(l, K):
            qp = K[0][:, pos].transpose(0, 1).contiguous().cpu()
            qd = synth.queries(1, l, 1, 8, 128, 8192)
            return torch.cat([qd, qp], 0), [0] * 129, [8192] + pos.tolist()
        res[name] = measure(cfg, 8192, (0, 15, 31), qf)
    return res


def config5():
    res = {}
    T = 32768
    arms = {
        "(i) NF4-K g64 + int4-g64 V": (Side("nf4", group=64), Side("int", 4, group=64), {}),
        "(ii) ternary g8, fp16 anchors layer 0 t<48": (Side("ternary", group=8), Side("ternary", group=8),
                                                        dict(anchor_layers=(0,), anchor_rule="first_n", anchor_n=48)),
        "(iii) sign g4": (Side("sign", group=4), Side("sign", group=4), {}),
    }
    for name, (k, v, an) in arms.items():
        cfg = Config(n_layers=32, batch=16, n_kv_heads=8, n_q_heads=32, head_dim=128, capacity=T, k=k, v=v,
                     max_queries=128, **an)

        def qf(l, K):
            px = [proxy_queries(K, b, synth.proxy_positions(1 + b, 8, T // 2, T), 4) for b in range(16)]
            return {"": (synth.queries(1, l, 16, 32, 128, T), list(range(16)), [T] * 16),
                    "_proxy": (torch.cat([p[0] for p in px]), sum((p[1] for p in px), []), sum((p[2] for p in px), []))}
        res[name] = measure(cfg, T, (0, 1, 31), qf)
    return res


def config1():
    s = Side("int", 4, group=32, rot=128)
    cfg = Config(n_layers=1, batch=1, n_kv_heads=2, n_q_heads=4, head_dim=128, capacity=512, k=s, v=s)
    qf = lambda l, K: (synth.queries(1, l, 1, 4, 128, 512), [0], [512])
    return {"H128 int4 g32": measure(cfg, 512, (0,), qf)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--config", default="all")
    ap.add_argument("--json", default="")
    a = ap.parse_args()
    fns = {"1": config1, "2": config2, "3": config3, "4": config4, "5": config5}
    todo = list(fns) if a.config == "all" else a.config.split(",")
    out = {}
    for c in todo:
        out[c] = fns[c]()
        for arm, m in out[c].items():
            print(f"config {c} | {arm:45s} | " + " ".join(f"{k}={v:.4g}" for k, v in m.items()), flush=True)
    if a.json:
        json.dump(out, open(a.json, "w"), indent=1)


if __name__ == "__main__":
    main()
