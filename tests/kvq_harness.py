"""Shared test harness: run the CUDA library and the CPU oracle on the same seeded inputs."""
from __future__ import annotations

from dataclasses import asdict

import numpy as np
import torch

from oracle import attention as OA
from oracle import cache as OC
from oracle import quant as OQ
from quantized_decode_attention_append_b200 import synth
from quantized_decode_attention_append_b200.kvq import Config, KVCache, Side

TOL = 2e-3  # max relative error (inf-norm per query-head vector) of decode attention


def kernel_names(run, want, tries: int = 8, repeat: int = 3) -> str:
    """Names of the CUDA kernels `run()` launches, seen by the torch profiler.  Its kernel records
    sometimes arrive incomplete -- the first launches of a session can be missing -- so each
    session calls `run()` `repeat` times (the same launches each time), and it looks again, up to
    `tries` times with a short pause, until every name in `want` is present."""
    import time

    from torch.profiler import ProfilerActivity, profile
    names = ""
    for i in range(tries):
        torch.cuda.empty_cache()  # room for the profiler's activity buffers after large tests
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            for _ in range(repeat):
                run()
            torch.cuda.synchronize()
        names = " ".join(e.name for e in prof.events())
        if all(w in names for w in want):
            break
        time.sleep(0.05 * (i + 1))
    return names


def oracle_side(s: Side) -> OQ.Side:
    return OQ.Side(**asdict(s))


def oracle_spec(cfg: Config) -> OC.Spec:
    return OC.Spec(cfg.n_layers, cfg.batch, cfg.n_kv_heads, cfg.n_q_heads, cfg.head_dim, oracle_side(cfg.k),
                   oracle_side(cfg.v), frozenset(cfg.anchor_layers), cfg.anchor_rule, cfg.anchor_n,
                   cfg.sm_scale or None, tuple(oracle_side(s) for s in cfg.layer_k),
                   tuple(oracle_side(s) for s in cfg.layer_v), anchor_bits=cfg.anchor_bits,
                   head_k=tuple(tuple(oracle_side(s) for s in row) for row in cfg.head_k),
                   head_v=tuple(tuple(oracle_side(s) for s in row) for row in cfg.head_v))


class Case:
    """A filled cache plus the fp16 inputs that went into it (kept on the host)."""

    def __init__(self, cfg: Config, T: int, seed: int = 0, chunks=None, layers=None, calib_T: int = 512,
                 inputs=None, chan=None):
        """inputs: optional callable l -> (K, V) fp16 arrays [B, H, T, D] replacing the seeded law;
        chan: optional callable l -> fp16 array [H, D] replacing the calibrated channel scale."""
        self.cfg, self.T, self.seed = cfg, T, seed
        self.cache = KVCache(cfg)
        self.K, self.V, self.C = {}, {}, {}
        B, H, D = cfg.batch, cfg.n_kv_heads, cfg.head_dim
        self.first_rows = (chunks or [T])[0]  # rows of each sequence's first append (the key mean's rows)
        layers = range(cfg.n_layers) if layers is None else layers
        for l in layers:
            if inputs is None:
                K = synth.kv_rows(seed, "k", l, list(range(B)), list(range(H)), list(range(T)), D, "cuda")
                V = synth.kv_rows(seed, "v", l, list(range(B)), list(range(H)), list(range(T)), D, "cuda")
            else:
                K, V = (torch.from_numpy(np.ascontiguousarray(a)).cuda() for a in inputs(l))
            if any(cfg.side(l, 0, h).chan_scale for h in range(H)):
                c = (synth.channel_scale(seed, l, H, calib_T, D) if chan is None else
                     torch.from_numpy(np.ascontiguousarray(chan(l), dtype=np.float16))).cuda()
                self.cache.set_chan_scale(l, c)
                self.C[l] = c.cpu().numpy()
            steps = chunks or [T]
            t = 0
            for n in steps:
                self.cache.append(l, K[:, :, t:t + n].contiguous(), V[:, :, t:t + n].contiguous())
                t += n
            assert t == T
            self.K[l] = K.cpu().numpy()
            self.V[l] = V.cpu().numpy()
        torch.cuda.synchronize()
        self.spec = oracle_spec(cfg)

    def oracle_unit(self, l, b, h):
        c = self.C[l][h] if l in self.C else None
        return OC.quantize_unit(self.spec, self.K[l][b, h], self.V[l][b, h], c, layer=l, first_rows=self.first_rows,
                                head=h)

    def views(self, l, side, head, names):
        """Host copies of the arena views of kv-head `head`'s group (None where absent), fetched
        once per head group."""
        key = (l, side, self.cache.layout(l, side, head).head0, tuple(names))
        memo = self.__dict__.setdefault("_views", {})
        if key not in memo:
            out = []
            for w in names:
                t = self.cache.view(l, side, w, head=head)
                out.append(None if t is None else t.cpu().numpy())
            memo[key] = out
        return memo[key]

    def forget_views(self):
        self.__dict__.pop("_views", None)

    def check_codes(self, l, rows=None):
        """Packed codes, scales and zero points of every unit are bit-identical to the oracle."""
        cfg = self.cfg
        self.forget_views()
        for side, name in ((0, "k"), (1, "v")):
            for h in range(cfg.n_kv_heads):
                codes, scales, zeros = self.views(l, side, h, ("codes", "scales", "zeros"))
                (kmean,) = self.views(l, 0, h, ("key_mean",))
                for b in range(cfg.batch):
                    u = self.cache.unit(l, b, h)
                    kq, vq = self.oracle_unit(l, b, h)
                    o = kq if side == 0 else vq
                    sel = slice(None) if rows is None else rows
                    got = codes[u, :self.T][sel]
                    want = o["bytes"][sel]
                    if not np.array_equal(got, want):
                        bad = np.argwhere(got != want)
                        raise AssertionError(f"{name} codes differ at layer {l} unit {u}: first {bad[:5].tolist()}"
                                             f" got {got[tuple(bad[0])]} want {want[tuple(bad[0])]}")
                    if scales is not None:
                        gs = scales[u, :self.T][sel]
                        ws = o["scales"][sel]
                        assert np.array_equal(gs.view(np.uint16), ws.view(np.uint16)), f"{name} scales l{l} u{u}"
                    if zeros is not None:
                        assert np.array_equal(zeros[u, :self.T][sel].view(np.uint16),
                                              o["zeros"][sel].view(np.uint16)), f"{name} zeros l{l} u{u}"
                    if side == 0 and kmean is not None:
                        assert np.array_equal(kmean[u].view(np.uint16), o["mu"].view(np.uint16)), f"key mean l{l} u{u}"

    def check_anchors(self, l):
        """Stored anchor rows of every unit equal the oracle's: fp16 rows, or int codes and scales."""
        cfg = self.cfg
        an = OC.anchored(self.spec, l, np.arange(self.T), self.T)
        if not an.any():
            return
        slots = np.arange(self.T)[an] % cfg.anchor_n if cfg.anchor_rule == "window" else np.arange(self.T)[an]
        self.forget_views()
        for side in (0, 1):
            for h in range(cfg.n_kv_heads):
                codes, sc = self.views(l, side, h, ("anchors", "anchor_scales"))
                for b in range(cfg.batch):
                    u = self.cache.unit(l, b, h)
                    src = (self.K[l] if side == 0 else self.V[l])[b, h][an]
                    want = OC.anchor_rows(self.spec, src)
                    if cfg.anchor_bits == 16:
                        assert np.array_equal(codes[u, slots].view(np.uint16), src.view(np.uint16))
                    else:
                        assert np.array_equal(codes[u, slots], want["bytes"]), f"anchor codes side {side} u{u}"
                        assert np.array_equal(sc[u, slots].view(np.uint16),
                                              want["scales"].view(np.uint16)), f"anchor scales side {side} u{u}"

    def check_dequant(self, l):
        """Stored domain bit-exact; original domain within fp32 transform error."""
        cfg = self.cfg
        for side in (0, 1):
            st = self.cache.dequantize(l, side, 0, self.T).cpu().numpy()
            org = self.cache.dequantize(l, side, 0, self.T, domain=1).cpu().numpy()
            for b in range(cfg.batch):
                for h in range(cfg.n_kv_heads):
                    kq, vq = self.oracle_unit(l, b, h)
                    o = kq if side == 0 else vq
                    assert np.array_equal(st[b, h].view(np.uint32), o["stored"].astype(np.float32).view(np.uint32)), \
                        f"stored dequant side {side} l{l} b{b} h{h}"
                    sd = OC.side_of(self.spec, l, side == 0, h)
                    c = self.C[l][h] if (side == 0 and l in self.C) else None
                    mu = o.get("mu")
                    want = OQ.to_original_f64(o["exact"], sd, None if c is None else np.broadcast_to(c, o["exact"].shape),
                                              None if mu is None else np.broadcast_to(mu, o["exact"].shape))
                    an = OC.anchored(self.spec, l, np.arange(self.T), self.T)
                    src = self.K[l] if side == 0 else self.V[l]
                    if an.any():
                        want[an] = OC.anchor_rows(self.spec, src[b, h][an])["exact"]
                    scale = np.abs(want).max()
                    assert np.abs(org[b, h] - want).max() <= 1e-5 * scale, f"orig dequant side {side} l{l}"

    def reconstructed(self, l, b):
        Ks, Vs = [], []
        for h in range(self.cfg.n_kv_heads):
            kq, vq = self.oracle_unit(l, b, h)
            c = self.C[l][h] if l in self.C else None
            Kh, Vh = OC.reconstruct_unit(self.spec, l, self.K[l][b, h], self.V[l][b, h], kq, vq, self.T, c)
            Ks.append(Kh)
            Vs.append(Vh)
        return np.stack(Ks), np.stack(Vs)

    def decode_and_compare(self, l, q16, seq_ids=None, kv_len=None, tol=TOL, decode=None):
        """Decode through the C ABI; compare every (query, head) output with the oracle.
        decode: optional callable (layer, q, seq_ids, kv_len) -> (out, lse) replacing the cache's
        kvq_decode_attention call (another entry point with the same contract)."""
        n_q = q16.shape[0]
        sid = None if seq_ids is None else torch.tensor(seq_ids, dtype=torch.int32, device="cuda")
        kl = None if kv_len is None else torch.tensor(kv_len, dtype=torch.int32, device="cuda")
        if decode is None:
            out, lse = self.cache.decode(l, q16.cuda(), sid, kl, lse=True)
        else:
            out, lse = decode(l, q16.cuda(), sid, kl)
        out = out.cpu().numpy()
        lse = lse.cpu().numpy()
        qn = q16.cpu().numpy()
        rec = {}
        worst = 0.0
        for i in range(n_q):
            b = i if seq_ids is None else seq_ids[i]
            if b not in rec:
                rec[b] = self.reconstructed(l, b)
            Kh, Vh = rec[b]
            n = self.T if kv_len is None else min(kv_len[i], self.T)
            o, ls, _ = OA.attention(qn[i], Kh, Vh, n, self.spec.sm_scale)
            for h in range(self.cfg.n_q_heads):
                if n == 0:
                    assert np.all(out[i, h] == 0) and np.isneginf(lse[i, h])
                    continue
                err = np.abs(out[i, h] - o[h]).max() / np.abs(o[h]).max()
                worst = max(worst, err)
                assert err <= tol, f"query {i} head {h}: rel err {err:.3e}"
                assert abs(lse[i, h] - ls[h]) <= 1e-3 * max(1.0, abs(ls[h])), f"lse q{i} h{h}"
        return worst
