"""Benchmark: quantized KV-cache decode steps/s on one B200 (replicas on N GPUs).

Default workload (the throughput-stress configuration): 32 layers x 8 KV heads x 32 query
heads, head_dim 128, batch 16 x 32768 tokens, NF4 K (group 64) + int4 V (group 64), 4.25 bits
per value.  One step = append one new token per sequence and decode attention on all 32
layers: kvq_append_decode per layer (one split-K launch that writes the new rows and decodes,
then the merge; kvq_quantize_append + kvq_decode_attention where the formats have no fused
kernel or the queries are proxy positions).
Other workloads: --workload names one of WORKLOADS below.

Timing: W warm-up steps, then K steps between CUDA events on the launching stream, with a
barrier and synchronize on both sides; the max over ranks is reported.  The per-layer KV
working set (570 MB for the default) exceeds L2 (126 MB), so no flush is needed.  CUDA
events around every decode call give the dominant kernel's duration for the roofline.
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOADS = {
    # name: (L, Hkv, Hq, D, B, T, k side, v side, anchors)
    "stress-nf4": dict(L=32, Hkv=8, Hq=32, D=128, B=16, T=32768,
                       k=dict(fmt="nf4", group=64), v=dict(fmt="int", bits=4, group=64),
                       desc="32L x 8kv x 32q, hd128, B16 x 32768 tokens; NF4-K g64 + int4-g64 V (4.25 b)"),
    "stress-int4": dict(L=32, Hkv=8, Hq=32, D=128, B=16, T=32768,
                        k=dict(fmt="int", bits=4, group=64), v=dict(fmt="int", bits=4, group=64),
                        desc="32L x 8kv x 32q, hd128, B16 x 32768 tokens; int4-g64 K and V (4.25 b)"),
    "stress-ternary": dict(L=32, Hkv=8, Hq=32, D=128, B=16, T=32768,
                           k=dict(fmt="ternary", group=8), v=dict(fmt="ternary", group=8),
                           anchors=dict(layers=(0,), rule="first_n", n=48),
                           desc="32L x 8kv x 32q, hd128, B16 x 32768; ternary g8, fp16 anchors layer 0, t < 48"),
    "stress-sign": dict(L=32, Hkv=8, Hq=32, D=128, B=16, T=32768,
                        k=dict(fmt="sign", group=4), v=dict(fmt="sign", group=4),
                        desc="32L x 8kv x 32q, hd128, B16 x 32768; sign g4"),
    "64k-A": dict(L=8, Hkv=4, Hq=16, D=256, B=1, T=65536,
                  k=dict(fmt="int", bits=4, group=128, rot=256), v=dict(fmt="int", bits=2, group=128, rot=256),
                  desc="8L x 4kv x 16q, hd256, B1 x 65536; H256 4-bit K + H256 2-bit V, g128 (3.125 b)"),
    "64k-konly": dict(L=8, Hkv=4, Hq=16, D=256, B=1, T=65536,
                      k=dict(fmt="int", bits=4, group=128, rot=256), v=dict(fmt="fp16"),
                      desc="8L x 4kv x 16q, hd256, B1 x 65536; H256 4-bit K g128, fp16 V"),
    "qwen-proxy128": dict(L=8, Hkv=4, Hq=4, D=256, B=1, T=6000,
                          k=dict(fmt="int", bits=4, scale="minmax", group=32),
                          v=dict(fmt="int", bits=4, scale="minmax", group=32), proxy=(128, 3000, 6000),
                          desc="8L x 4kv x 4q (G 1), hd256, B1 x 6000; per-token min-max 4-bit g32 K and V (arm A); "
                               "128 proxy queries (post-RoPE keys at positions in [3000, 6000), causal)"),
    "qwen-proxy128-h256": dict(L=8, Hkv=4, Hq=4, D=256, B=1, T=6000,
                               k=dict(fmt="int", bits=4, scale="minmax", group=32, rot=256),
                               v=dict(fmt="int", bits=4, scale="minmax", group=32, rot=256), proxy=(128, 3000, 6000),
                               desc="8L x 4kv x 4q (G 1), hd256, B1 x 6000; H256 min-max 4-bit g32 K and V (arm B); "
                                    "128 proxy queries, causal"),
    "polar-4+8": dict(L=32, Hkv=8, Hq=8, D=128, B=1, T=8192,
                      k=dict(fmt="polar", bits=4, bits2=8), v=dict(fmt="polar", bits=4, bits2=8),
                      desc="32L x 8kv x 8q (G 1), hd128, B1 x 8192; rFFT polar K and V, 4-bit magnitude + 8-bit "
                           "phase (6.125 b)"),
    "stress-ternary-a8": dict(L=32, Hkv=8, Hq=32, D=128, B=16, T=32768,
                              k=dict(fmt="ternary", group=8), v=dict(fmt="ternary", group=8),
                              anchors=dict(layers=(0,), rule="first_n", n=48, bits=8),
                              desc="32L x 8kv x 32q, hd128, B16 x 32768; ternary g8, int8 anchors layer 0, t < 48 "
                                   "('ternboth_a8')"),
    "64k-sym2": dict(L=8, Hkv=4, Hq=16, D=256, B=1, T=65536,
                     k=dict(fmt="int", bits=4, group=128, rot=256),
                     v=dict(fmt="int", bits=2, scale="sym", group=128, rot=256),
                     desc="8L x 4kv x 16q, hd256, B1 x 65536; H256 4-bit K + H256 symmetric 2-bit V, g128 "
                          "(3.125 b; the E22L next-run grid)"),
    "64k-v3": dict(L=8, Hkv=4, Hq=16, D=256, B=1, T=65536,
                   k=dict(fmt="int", bits=4, group=128, rot=256), v=dict(fmt="int", bits=3, group=128, rot=256),
                   desc="8L x 4kv x 16q, hd256, B1 x 65536; H256 4-bit K + H256 3-bit V, g128 (3.625 b)"),
}
DEFAULT_WORKLOAD = "stress-nf4"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_PEAKS["hbm_gbs"], "fallback"


def make_config(w, T_cap):
    from quantized_decode_attention_append_b200.kvq import Config, Side
    an = w.get("anchors")
    return Config(n_layers=w["L"], batch=w["B"], n_kv_heads=w["Hkv"], n_q_heads=w["Hq"], head_dim=w["D"],
                  capacity=T_cap, k=Side(**w["k"]), v=Side(**w["v"]),
                  max_queries=w["proxy"][0] if w.get("proxy") else w["B"],
                  anchor_layers=an["layers"] if an else (), anchor_rule=an["rule"] if an else "none",
                  anchor_n=an["n"] if an else 0, anchor_bits=an.get("bits", 16) if an else 16)


def proxy_setup(w, T0, seed, layer, device):
    """Proxy queries ("E21W" "What I tested"): the post-RoPE keys of sequence 0 at n positions drawn
    from [lo, min(hi, T0)), each attending the keys before it.  Returns (q [n, Hq, D], positions)."""
    from quantized_decode_attention_append_b200 import synth
    n, lo, hi = w["proxy"]
    pos = synth.proxy_positions(1, n, lo, min(hi, T0))
    K = synth.kv_rows(seed, "k", layer, [0], list(range(w["Hkv"])), pos.tolist(), w["D"], device)[0]
    return K.transpose(0, 1).contiguous(), pos


def row_bytes_of(cache, side):
    """Stored bytes of one row of `side` (codes + fp16 scales + fp16 zero points), from the
    library's own layout."""
    lo = cache.layout(0, side)
    return lo.row_bytes + 2 * lo.n_groups * (2 if lo.zeros >= 0 else 1)


def decode_bytes(cache, w, kv_len, anchored_rows_per_unit, proxy_pos=None):
    """Algorithmic bytes of one decode call: packed K/V rows + scales for t < kv_len (anchor rows
    as stored for anchored tokens), the queries and the fp32 outputs.  With proxy queries each
    query reads its own causal prefix of sequence 0."""
    D, units = w["D"], w["B"] * w["Hkv"]
    per_tok = row_bytes_of(cache, 0) + row_bytes_of(cache, 1)
    if proxy_pos is not None:
        n = len(proxy_pos)
        return w["Hkv"] * per_tok * float(sum(proxy_pos)) + n * w["Hq"] * D * (2 + 4)
    a = anchored_rows_per_unit
    an = w.get("anchors") or {}
    ab = an.get("bits", 16)
    a_row = 2 * (2 * D if ab == 16 else D * ab // 8 + 2 * (D // 32))  # K and V anchor rows as stored
    kv = units * ((kv_len - a) * per_tok + a * a_row)
    return kv + w["B"] * w["Hq"] * D * (2 + 4)


class ClockSampler:
    """SM clock and clock-event reasons of one GPU, polled through NVML every few milliseconds on a
    host thread between start() and stop() (read-only queries)."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap",
               0x80: "hw_power_brake_slowdown"}

    def __init__(self, dev, period_s=0.004):
        self.dev, self.period = dev, period_s
        self.rows, self.thread, self.err = [], None, None

    def start(self):
        import threading
        import torch
        try:
            import pynvml as N
            N.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(self.dev).uuid)
            self.h = N.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = N.nvmlDeviceGetMaxClockInfo(self.h, N.NVML_CLOCK_SM)
            self.N = N
        except Exception as e:  # no NVML: report it instead of clocks
            self.err = f"nvml unavailable: {type(e).__name__}"
            return
        self.stop_flag = threading.Event()

        def poll():
            while not self.stop_flag.is_set():
                try:
                    self.rows.append((self.N.nvmlDeviceGetClockInfo(self.h, self.N.NVML_CLOCK_SM),
                                      self.N.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
                except Exception as e:
                    self.err = f"nvml query failed: {type(e).__name__}"
                    return
                self.stop_flag.wait(self.period)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [self.err or "not started"]}
        self.stop_flag.set()
        self.thread.join(timeout=5)
        if not self.rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [self.err or "no samples"]}
        sm = sorted(r[0] for r in self.rows)
        reasons = sorted({name for _, m in self.rows for bit, name in self.REASONS.items() if m & bit})
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(self.rows), "period_ms": self.period * 1e3, "source": "nvml"}


DECODE_SOURCES = ("decode.cu", "decode_tc.cuh", "decode_mq.cuh", "decode_polar.cuh", "decode_common.cuh", "fft128.cuh",
                  "quantize_row.cuh", "kvq_internal.h")


def decode_sources_sha256():
    """One hash over the decode kernels' sources, in a fixed order."""
    import hashlib
    h = hashlib.sha256()
    for f in DECODE_SOURCES:
        h.update(open(os.path.join(ROOT, "quantized_decode_attention_append_b200", "csrc", f), "rb").read())
    return h.hexdigest()


def traffic_record(workload):
    """DRAM bytes (read + write) of one decode call -- split-K pass and merge -- from the committed
    ncu summary, or None when that summary was taken on other decode sources."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    rec = json.load(open(p))
    if rec.get("sources_sha256") != decode_sources_sha256():
        return None
    w = rec.get("per_call", {}).get(workload)
    return None if w is None else w["bytes"]


# ----------------------------------------------------------------------------------- CPU oracle
def _oracle_spec(w):
    from oracle import cache as OC
    from oracle import quant as OQ
    an = w.get("anchors")
    return OC.Spec(w["L"], w["B"], w["Hkv"], w["Hq"], w["D"], OQ.Side(**w["k"]), OQ.Side(**w["v"]),
                   frozenset(an["layers"]) if an else frozenset(), an["rule"] if an else "none", an["n"] if an else 0,
                   anchor_bits=an.get("bits", 16) if an else 16)


def _oracle_unit(w, spec, idx, seed):
    """Inputs of oracle unit `idx` (a (layer, sequence, kv-head) of one step) and the function that
    runs it: quantize the unit's T rows, reconstruct them, attend its queries (the unit's query
    heads, or every proxy query of the sequence)."""
    from oracle import cache as OC
    from quantized_decode_attention_append_b200 import synth
    D, T, G = w["D"], w["T"], w["Hq"] // w["Hkv"]
    layer, b, h = idx % w["L"], (idx // w["L"]) % w["B"], idx % w["Hkv"]
    K16 = synth.kv_rows(seed, "k", layer, [b], [h], list(range(T)), D)[0, 0].numpy()
    V16 = synth.kv_rows(seed, "v", layer, [b], [h], list(range(T)), D)[0, 0].numpy()
    if w.get("proxy"):
        n, lo, hi = w["proxy"]
        pos = synth.proxy_positions(1, n, lo, min(hi, T))
        qs = [(K16[p][None, :], int(p)) for p in pos]
    else:
        qs = [(synth.queries(1, layer, 1, G, D, T)[0].numpy()[:G], T)]

    def run():
        kq, vq = OC.quantize_unit(spec, K16, V16)
        Kh, Vh = OC.reconstruct_unit(spec, layer, K16, V16, kq, vq, T)
        for q, kl in qs:
            OC.decode_query(spec, layer, q, Kh[None], Vh[None], kl)
    return run


def _oracle_worker(args):
    """One process of the multi-process sample: time units start, start + stride, ... for
    budget_s seconds (single-threaded numpy); returns (units, seconds)."""
    w, start, stride, budget_s, seed = args
    from threadpoolctl import threadpool_limits
    spec = _oracle_spec(w)
    done, spent, idx = 0, 0.0, start
    with threadpool_limits(1):
        while spent < budget_s and done < 64:
            run = _oracle_unit(w, spec, idx, seed)
            t0 = time.perf_counter()
            run()
            spent += time.perf_counter() - t0
            done += 1
            idx += stride
    return done, spent


def oracle_sample(w, budget_s=15.0, seed=0, processes=0):
    """Time the oracle, as it stands, on whole units of one decode step (see _oracle_unit); input
    generation is outside the timed region.  Single-threaded in this process for budget_s, then,
    if processes > 1, the same work spread over that many spawned processes (one numpy thread
    each) for budget_s of wall time.  Returns a dict of seconds per unit (single thread), units per
    second (all processes), and the counts."""
    single = _oracle_worker((w, 0, 1, budget_s, seed))
    out = {"units_single": single[0], "s_per_unit_single": single[1] / single[0], "processes": 1,
           "units_per_s_multi": single[0] / single[1], "units_multi": single[0]}
    if processes > 1:
        import concurrent.futures as cf
        import multiprocessing as mp
        with cf.ProcessPoolExecutor(max_workers=processes, mp_context=mp.get_context("spawn")) as ex:
            res = list(ex.map(_oracle_worker, [(w, i, processes, budget_s, seed) for i in range(processes)]))
        out["processes"] = processes
        out["units_multi"] = sum(r[0] for r in res)
        out["units_per_s_multi"] = sum(r[0] / r[1] for r in res)  # the processes ran concurrently
    return out


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def cpu_baseline_record(w, budget_s, processes):
    o = oracle_sample(w, budget_s=budget_s, processes=processes)
    units_per_step = w["L"] * w["B"] * w["Hkv"]
    what = (f"{w['proxy'][0]} proxy queries" if w.get("proxy") else f"{w['Hq'] // w['Hkv']} query heads")
    sample = (f"whole (layer, sequence, kv-head) units of one step: quantize + reconstruct {w['T']} rows, attend "
              f"{what}; {o['units_single']} units on 1 thread and {o['units_multi']} units over {o['processes']} "
              f"processes, scaled by {units_per_step} units/step")
    return {"value": o["units_per_s_multi"] / units_per_step, "unit": "steps/s", "cores": o["processes"],
            "kind": "oracle", "sample": sample, "nproc": host_cores(),
            "single_thread": {"value": 1.0 / (o["s_per_unit_single"] * units_per_step), "unit": "steps/s"},
            "multi_process": {"value": o["units_per_s_multi"] / units_per_step, "unit": "steps/s",
                              "processes": o["processes"]}}


def run_reference(args, w, name):
    cpu = cpu_baseline_record(w, args.ref_budget, max(1, min(host_cores(), args.ref_processes)))
    sps = cpu["value"]
    rec = {"impl": "reference", "metric": "decode steps/s", "value": sps, "unit": "steps/s", "n_gpus": args.gpus,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 / sps, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": f"{name}: {w['desc']}"},
           "cpu_baseline": cpu,
           "e2e": {"value": sps, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(rec), flush=True)


# ----------------------------------------------------------------------------------- GPU arm
def fill_cache(cache, w, T0, seed, device, timed=False):
    """Prefill every layer to T0 tokens with bulk appends; optionally time the appends."""
    import torch
    from quantized_decode_attention_append_b200 import synth
    B, H, D = w["B"], w["Hkv"], w["D"]
    chunk = max(1, min(T0, (1 << 28) // (B * H * D)))
    ms, rows = 0.0, 0
    stream = torch.cuda.current_stream()
    first = True  # the first append pays the kernels' first-launch loading: not timed
    for l in range(w["L"]):
        t = 0
        while t < T0:
            n = min(chunk, T0 - t)
            toks = list(range(t, t + n))
            K = synth.kv_rows(seed, "k", l, list(range(B)), list(range(H)), toks, D, device)
            V = synth.kv_rows(seed, "v", l, list(range(B)), list(range(H)), toks, D, device)
            if timed and not first:
                torch.cuda.synchronize()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                # a ~0.5 ms device-side delay ahead of the start event lets the host queue the
                # append before the device reaches it, so the events bracket the kernel alone
                torch.cuda._sleep(1_000_000)
                e0.record(stream)
            cache.append(l, K, V)
            if timed and not first:
                e1.record(stream)
                e1.synchronize()
                ms += e0.elapsed_time(e1)
                rows += B * H * n
            first = False
            t += n
            del K, V
    torch.cuda.synchronize()
    return ms, rows


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings (one all_reduce; replicas exchange nothing else)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def aggregate_steps_per_s(ms_step_max: float, world: int) -> float:
    """Whole-job throughput of `world` replicas, each doing one step per ms_step_max (the slowest)."""
    return world * 1e3 / ms_step_max


def run_gpu(args, w, name):
    import torch
    import torch.distributed as dist

    from quantized_decode_attention_append_b200 import kvq, synth
    from quantized_decode_attention_append_b200.kvq import KVCache

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    L, B, Hkv, Hq, D, T = w["L"], w["B"], w["Hkv"], w["Hq"], w["D"], w["T"]
    K_, W_ = args.steps, args.warmup
    T0 = T - K_ - W_
    cfg = make_config(w, T)
    cache = KVCache(cfg, dev)
    q_ms, q_rows = fill_cache(cache, w, T0, seed=rank, device=dev, timed=True)
    # per-step inputs resident in HBM: one new K/V row per sequence and layer, queries per layer
    knew = [synth.kv_rows(rank, "k", l, list(range(B)), list(range(Hkv)), [T0], D, dev) for l in range(L)]
    vnew = [synth.kv_rows(rank, "v", l, list(range(B)), list(range(Hkv)), [T0], D, dev) for l in range(L)]
    proxy = w.get("proxy")
    if proxy:  # config-2 shape: one sequence, its proxy queries, each causal over earlier keys
        pq = [proxy_setup(w, T0, rank, l, dev) for l in range(L)]
        qs = [p[0] for p in pq]
        proxy_pos = pq[0][1]
        qsid = torch.zeros(len(proxy_pos), dtype=torch.int32, device=dev)
        qlen = torch.tensor(proxy_pos.tolist(), dtype=torch.int32, device=dev)
    else:
        qs = [synth.queries(1, l, B, Hq, D, T0).to(dev) for l in range(L)]
        proxy_pos, qsid, qlen = None, None, None
    n_q = qs[0].shape[0]
    outs = [torch.empty(n_q, Hq, D, device=dev, dtype=torch.float32) for _ in range(L)]
    launches = {"n": 0}

    # one query per sequence: the decode step is kvq_append_decode (append and decode in one
    # split-K launch where the layer's formats allow it); proxy queries append, then decode
    fused_step = not proxy

    def layer_step(l, k, v, q, out):
        if fused_step:
            cache.append_decode(l, k, v, q, out=out)
            launches["n"] += kvq.kvq_last_launch_count(cache.h)
        else:
            cache.append(l, k, v)
            launches["n"] += kvq.kvq_last_launch_count(cache.h)
            cache.decode(l, q, seq_ids=qsid, kv_len=qlen, out=out)
            launches["n"] += kvq.kvq_last_launch_count(cache.h)

    def step():
        for l in range(L):
            layer_step(l, knew[l], vnew[l], qs[l], outs[l])

    def decode_only():
        for l in range(L):
            cache.decode(l, qs[l], seq_ids=qsid, kv_len=qlen, out=outs[l])

    # one eager step (first-call set-up), then capture the step and the decode-only pass
    step()
    per_step_launches = launches["n"]
    torch.cuda.synchronize()
    g_step, g_dec = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_step):
        step()
    with torch.cuda.graph(g_dec):
        decode_only()
    stream = torch.cuda.current_stream(dev)
    for _ in range(W_ - 1):
        g_step.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clocks = ClockSampler(dev)
    clocks.start()
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    t_start.record(stream)
    for i in range(K_):
        g_step.replay()
    t_end.record(stream)
    torch.cuda.synchronize()
    ms = t_start.elapsed_time(t_end)
    # decode launches alone, back to back in a graph: the dominant kernel's duration
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for i in range(K_):
        g_dec.replay()
    d1.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    dec_launch_ms = d0.elapsed_time(d1) / (K_ * L)
    ms, dec_launch_ms = max_over_ranks([ms, dec_launch_ms], dev)
    if world > 1:
        dist.barrier()
    flags = kvq.kvq_error_flags(cache.h)
    ms_step = ms / K_
    # algorithmic bytes per decode call at the cache length the decode-only pass saw
    an = w.get("anchors")
    anchored = an["n"] if an and an["rule"] == "first_n" else 0
    dec_len = T0 + W_ + K_
    mean_len = T0 + W_ + (K_ + 1) / 2.0
    per_layer = lambda n, a: decode_bytes(cache, w, n, a, proxy_pos)
    dec_bytes_step = sum(per_layer(mean_len, anchored if (an and l in an["layers"]) else 0) for l in range(L))
    dec_bytes_launch = sum(per_layer(dec_len, anchored if (an and l in an["layers"]) else 0) for l in range(L)) / L
    achieved = dec_bytes_launch / (dec_launch_ms * 1e-3) / 1e9
    l2 = 126e6
    l2_note = ("per-layer KV working set exceeds L2 (126 MB); no flush" if dec_bytes_launch > l2 else
               f"per-layer KV set {dec_bytes_launch / 1e6:.0f} MB is below L2 (126 MB), but each pass reads all {L} "
               f"layers ({dec_bytes_step / 1e6:.0f} MB) before a layer comes round again; no flush")
    peak, peak_kind = peaks()
    row_io = 2 * 2 * D + row_bytes_of(cache, 0) + row_bytes_of(cache, 1)  # fp16 in + packed out, K and V
    quant_gbps = (q_rows * row_io) / (q_ms * 1e-3) / 1e9 if q_ms > 0 else None

    # end to end through the public API with host buffers: every step copies its new rows and
    # queries in from pinned memory and its attention outputs back out.  A copy stream moves layer
    # l's inputs in (one copy per layer) and layer l's outputs out while other layers compute; the
    # compute stream waits for each layer's inputs (captured with the step, fork/join in the graph).
    parts = [[knew[l], vnew[l], qs[l]] for l in range(L)]
    lay = [sum((x.numel() + 63) // 64 * 64 for x in p) for p in parts]  # 128-byte aligned pieces
    h_in = torch.zeros(sum(lay), dtype=torch.float16).pin_memory()
    d_in = torch.empty_like(h_in, device=dev)
    d_k, d_v, d_q, spans, off = [], [], [], [], 0
    for l in range(L):
        start = off
        for x, dst in zip(parts[l], (d_k, d_v, d_q)):
            h_in[off:off + x.numel()] = x.reshape(-1).cpu()
            dst.append(d_in[off:off + x.numel()].view(x.shape))
            off += (x.numel() + 63) // 64 * 64
        spans.append((start, off))
    d_out = torch.empty(L, n_q, Hq, D, device=dev, dtype=torch.float32)
    h_out = torch.empty(L, n_q, Hq, D, dtype=torch.float32).pin_memory()
    copy_stream = torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(L)]
    ev_out = [torch.cuda.Event() for _ in range(L)]

    pipelined = h_in.numel() * h_in.element_size() >= L * (1 << 16)  # per-layer copies only when large

    def e2e_step():
        main = torch.cuda.current_stream(dev)
        if not pipelined:  # small steps: one copy in, one copy out
            d_in.copy_(h_in, non_blocking=True)
            for l in range(L):
                layer_step(l, d_k[l], d_v[l], d_q[l], d_out[l])
            h_out.copy_(d_out, non_blocking=True)
            return
        copy_stream.wait_stream(main)
        with torch.cuda.stream(copy_stream):
            for l in range(L):
                a, b = spans[l]
                d_in[a:b].copy_(h_in[a:b], non_blocking=True)
                ev_in[l].record(copy_stream)
        for l in range(L):
            main.wait_event(ev_in[l])
            layer_step(l, d_k[l], d_v[l], d_q[l], d_out[l])
            ev_out[l].record(main)
        with torch.cuda.stream(copy_stream):
            for l in range(L):
                copy_stream.wait_event(ev_out[l])
                h_out[l].copy_(d_out[l], non_blocking=True)
        main.wait_stream(copy_stream)

    E = max(1, min(K_, 10))
    cache.set_seq_len(-1, T0 + W_ - 1)
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        g_e2e.replay()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / E
    e2e_ms = max_over_ranks([e2e_ms], dev)[0]
    h2d = h_in.numel() * h_in.element_size()
    d2h = h_out.numel() * h_out.element_size()

    rec = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = cpu_baseline_record(w, args.ref_budget, max(1, min(host_cores(), args.ref_processes)))
        rec = {"metric": "decode steps/s", "value": aggregate_steps_per_s(ms_step, world), "unit": "steps/s",
               "n_gpus": world,
               "steps": K_, "warmup": W_, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "f32", "data": "synthetic",
               "config": {"workload": f"{name}: {w['desc']}", "global_batch": world * B, "seq_len": T,
                          "parallelism": f"replicas{world}", "layers": L,
                          "l2": l2_note,
                          "step": f"append 1 token/seq + decode, all {L} layers, one CUDA graph"
                                  + ("; kvq_append_decode per layer" if fused_step else
                                     "; kvq_quantize_append + kvq_decode_attention per layer")},
               "kv_gbps": dec_bytes_step / (ms_step * 1e-3) / 1e9 * world,
               "decode_ms_per_layer": dec_launch_ms,
               "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                            "frac": achieved / peak, "traffic": traffic_record(name),
                            "kernel": "kvq_decode_attention (split-K pass + merge), back-to-back in a graph",
                            "peak_kind": f"{peak_kind} hbm_gbs (burst copy)",
                            "bytes_per_launch": dec_bytes_launch},
               "quantize": {"gbps": quant_gbps, "frac": (quant_gbps / peak) if quant_gbps else None,
                            "rows": q_rows, "bytes_per_row": row_io,
                            "what": "bulk prefill appends (fp16 K+V read, packed codes + scales written)"},
               "cpu_baseline": cpu,
               "e2e": {"value": aggregate_steps_per_s(e2e_ms, world), "unit": "steps/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h},
               "gpu_launches": per_step_launches * K_,
               "clocks": clk, "error_flags": flags}
        print(json.dumps(rec), flush=True)
    del g_step, g_dec, g_e2e
    cache.close()
    if world > 1:
        dist.destroy_process_group()
    return rec


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--ref-budget", type=float, default=10.0,
                    help="seconds of CPU oracle work to sample (single thread, then again over all processes)")
    ap.add_argument("--ref-processes", type=int, default=16,
                    help="oracle processes for the multi-process sample (capped by the host's cores; each one "
                         "imports numpy and torch)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0, help="profiling only: fewer layers than the workload")
    ap.add_argument("--batch", type=int, default=0, help="profiling only: fewer sequences than the workload")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    w = dict(WORKLOADS[args.workload])
    if args.layers:
        w["L"] = args.layers
        w["desc"] += f" [profiling size: {args.layers} layers]"
    if args.batch:
        w["B"] = args.batch
        w["desc"] += f" [profiling size: batch {args.batch}]"
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args, w, args.workload)
        return
    run_gpu(args, w, args.workload)


if __name__ == "__main__":
    main()
