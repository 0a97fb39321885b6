"""Benchmark: packed K3V3 decode attention at 128K context on B200.

Workload (default): the Qwen2.5-3B-shaped stack -- 36 layers, 16 query / 2 KV
heads, head_dim 128, T = 131072, batch 1, K3V3 -- on synthetic fp16 K/V/q
(seeded, RoPE theta 1e6, per-head decay and outlier blocks).  The packed cache
of every layer is built once by the library (energy + greedy allocation +
quantize-pack); a step is one decode over all 36 layers (query rotation,
split-K decode, merge with R_V^T), captured in a CUDA graph.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs under torchrun: every rank decodes its own independent sequence
(weak scaling; no collective in the data path).  --impl reference times the CPU
fp64 oracle (the method as written, never tuned) on the same workload.
Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "packed K3V3 decode-attn cache GB/s (% HBM peak) & ctx-tokens/s at 128K"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 2 ** 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=2)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="override the workload's context length (overhead studies only)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the per-config and peak-memory blocks (headline workload only)")
    return ap.parse_args()


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def packed_bytes_per_token_head(kb, vb, g_k):
    """Algorithmic bytes one decode reads per (token, KV head): key codes,
    group norms, value codes, value norm (K-only plans, vb = 0: the fp16 value
    row of 256 bytes instead)."""
    if vb == 0:
        return 16 * kb + 2 * g_k + 2 * 128
    return 16 * kb + 2 * g_k + 16 * vb + 2


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        loaded = [x for x in sm if mx and x > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


# --------------------------------------------------------------- profiles
def profile_traffic(kernel_src):
    """dram bytes per decode launch from the committed ncu summary, or None if
    the kernel source changed since that capture."""
    path = os.path.join(ROOT, "profiles", "decode_kernel_qwen2.5-3b_128k.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m = re.search(r"source_sha256:\s*([0-9a-f]{64})", text)
    t = re.search(r"traffic_bytes_per_layer_call:\s*([0-9.eE+]+)", text)
    if not m or not t:
        return None
    if m.group(1) != hashlib.sha256(open(kernel_src, "rb").read()).hexdigest():
        return None
    return float(t.group(1))


L2_BYTES = 126e6


def cache_copies(step_bytes):
    """Copies of the packed cache a timed loop cycles through so that every
    step reads it cold: enough that they exceed the L2 about three times."""
    return max(1, int(math.ceil(3 * L2_BYTES / max(step_bytes, 1.0))))


def workload_config(cfgd, world):
    """The `config` object of both arms' JSON lines (identical keys)."""
    step_bytes = cfgd["layers"] * cfgd["B"] * cfgd["h_kv"] * cfgd["T"] * packed_bytes_per_token_head(
        cfgd["k_bits"], cfgd["v_bits"], 6)
    copies = cache_copies(step_bytes)
    l2 = ("cold: about %.0f MB of packed cache per step > 126 MB L2, layers read in turn"
          % (step_bytes / 1e6)) if copies == 1 else (
          "cold: about %.0f MB of packed cache per step, %d copies of it cycled per timed "
          "loop (%.0f MB > 126 MB L2)" % (step_bytes / 1e6, copies, copies * step_bytes / 1e6))
    return {"workload": cfgd["name"], "layers": cfgd["layers"], "batch": cfgd["B"],
            "q_heads": cfgd["h_q"], "kv_heads": cfgd["h_kv"], "seq_len": cfgd["T"],
            "k_bits": cfgd["k_bits"], "v_bits": cfgd["v_bits"],
            "parallelism": "replicas" if world == 1 else "dp%d (independent sequences)" % world,
            "l2": l2}


# ------------------------------------------------------------ multi-rank
def max_over_ranks(value, world, device=None):
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(value)
    import torch

    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def rank_seed(config, rank, layer):
    """Seed of one rank's layer: every rank decodes its own independent sequence."""
    return (config, rank, layer)


# ------------------------------------------------------------ reference arm
def oracle_pool(cfgd, n_heads=2, seed=2):
    """A few whole KV heads of the workload, coded by the oracle (not timed)."""
    from decode_attention_13_b200 import synth
    from oracle import allocation, quantize

    gq = cfgd["h_q"] // cfgd["h_kv"]
    pool = []
    for i in range(n_heads):
        hd = synth.head((seed, 9999, i), T=cfgd["T"], theta=cfgd["theta"], g_q=gq)
        bits = allocation.greedy_bits(allocation.block_energy(hd["k"]), cfgd["k_bits"], 128)
        pool.append((hd["q"], quantize.quantize_keys(hd["k"], bits, 0),
                     quantize.quantize_values(hd["v"], cfgd["v_bits"])))
    return pool


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info

        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return 1


def _head_slice(kg, vg, n):
    """The first n cached tokens of a coded head (the oracle's data classes)."""
    import dataclasses

    cut = lambda g: dataclasses.replace(g, codes=g.codes[:n], norm16=g.norm16[:n],
                                        norm64=g.norm64[:n])
    return [cut(g) for g in kg], cut(vg)


def oracle_decode_sample(cfgd, pool, seconds, tokens=None):
    """Time the fp64 oracle's decode of KV heads from `pool` until `seconds`
    elapse (at least one); each decode covers the first `tokens` cached tokens
    of a head (all T by default).  Returns (GB/s of packed cache, heads decoded,
    seconds, tokens per decode)."""
    from oracle import attention

    T, kb, vb = cfgd["T"], cfgd["k_bits"], cfgd["v_bits"]
    n = T if tokens is None else max(1, min(T, int(tokens)))
    heads, nbytes, spent = 0, 0.0, 0.0
    while spent < seconds or heads == 0:
        q, kg, vg = pool[heads % len(pool)]
        if n < T:
            kg, vg = _head_slice(kg, vg, n)
        t0 = time.perf_counter()
        attention.decode_rotated(q, kg, vg)
        spent += time.perf_counter() - t0
        nbytes += n * packed_bytes_per_token_head(kb, vb, len(kg))
        heads += 1
    return nbytes / spent / 1e9, heads, spent, n


def run_reference(args, rank, world):
    from decode_attention_13_b200 import synth

    cfgd = dict(synth.CONFIGS[args.config], index=args.config)
    if rank != 0:
        return
    pool = oracle_pool(cfgd)
    threads = oracle_threads()
    # each step decodes a token slice of one head, sized so that the K steps
    # take about --cpu-seconds together (a bounded sample of the same work)
    per_step = args.cpu_seconds / max(1, args.steps)
    _, _, spent, _ = oracle_decode_sample(cfgd, pool, 0.0, tokens=8192)
    tokens = max(1024, int(8192 * per_step / max(spent, 1e-6)))
    for _ in range(args.warmup):
        oracle_decode_sample(cfgd, pool, 0.0, tokens=tokens)
    vals, heads_total, spent_total = [], 0, 0.0
    for _ in range(args.steps):
        v, h, s, n = oracle_decode_sample(cfgd, pool, 0.0, tokens=tokens)
        vals.append(v)
        heads_total += h
        spent_total += s
    value = statistics.mean(vals)
    sample = ("oracle decode of the first %d cached tokens of a KV head (of T=%d, G=%d query "
              "heads), %d times, from the %s workload; one decode per step"
              % (min(tokens, cfgd["T"]), cfgd["T"], cfgd["h_q"] // cfgd["h_kv"], heads_total,
                 cfgd["name"]))
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "ms_per_step": 1e3 * spent_total / max(1, args.steps), "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(cfgd, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------------ our arm
def build_workload(cfgd, rank, dev, stream):
    """Every layer's plan and packed cache (energy, greedy allocation,
    quantize-pack by the library), its queries and output buffers."""
    import torch

    import decode_attention_13_b200 as gtq
    from decode_attention_13_b200 import synth

    L, B, hq, hkv, T = cfgd["layers"], cfgd["B"], cfgd["h_q"], cfgd["h_kv"], cfgd["T"]
    kb, vb, gq = cfgd["k_bits"], cfgd["v_bits"], cfgd["h_q"] // cfgd["h_kv"]
    w = {"plans": [], "packed": [], "qs": [], "outs": [], "kv": []}
    for layer in range(L):
        k, v, q = synth.layer_torch(rank_seed(cfgd["index"], rank, layer), B, hkv, gq, T,
                                    theta=cfgd["theta"], decay=cfgd["decay"], device=dev)
        # the inputs were drawn on torch's stream: the library's stream waits for them
        stream.wait_stream(torch.cuda.current_stream(dev))
        cfg = gtq.make_config(B, hq, hkv, kb, vb, T)
        with torch.cuda.stream(stream):
            plan = gtq.gtq_alloc_bits(cfg, k, T, stream=stream)
            buf = torch.empty(plan.packed_bytes, dtype=torch.uint8, device=dev)
            gtq.gtq_quantize_pack(plan, k, v, 0, T, buf, stream=stream)
        w["plans"].append(plan)
        w["packed"].append(buf)
        w["qs"].append(q)
        w["outs"].append(torch.empty((B, hq, 128), dtype=torch.float32, device=dev))
        w["kv"].append((k, v))
    stream.synchronize()
    for p in w["plans"]:
        rc = gtq.gtq_status(p)
        if rc != gtq.GTQ_OK:
            raise RuntimeError("status after quantize: " + gtq.strerror(rc))
    g_k = []  # nonzero-width key groups of every head (norms read per token)
    for p in w["plans"]:
        bits = gtq.gtq_get_bits(p)
        g_k.append([[len(set(int(x) for x in bits[b, h] if x > 0)) for h in range(hkv)]
                    for b in range(B)])
    w["step_bytes"] = float(sum(T * packed_bytes_per_token_head(kb, vb, g_k[l][b][h])
                                for l in range(L) for b in range(B) for h in range(hkv)))
    # small caches: further copies, so that a timed loop reads cold data
    w["copies"] = cache_copies(w["step_bytes"])
    with torch.cuda.stream(stream):
        w["packed_copies"] = [w["packed"]] + [[p.clone() for p in w["packed"]]
                                              for _ in range(w["copies"] - 1)]
    stream.synchronize()
    w["fp16_bytes"] = float(L * B * hkv * T * 2 * 128 * 2)
    return w


def time_quantize(cfgd, w, stream):
    """CUDA-event time of one quantize-pack of every layer (ms) and its bytes."""
    import torch

    import decode_attention_13_b200 as gtq

    T = cfgd["T"]
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for layer, (k, v) in enumerate(w["kv"]):
            gtq.gtq_quantize_pack(w["plans"][layer], k, v, 0, T, w["packed"][layer], stream=stream)
        ev1.record(stream)
    stream.synchronize()
    ms = ev0.elapsed_time(ev1)
    nbytes = float(cfgd["layers"] * cfgd["B"] * cfgd["h_kv"] * T * 512) + w["step_bytes"]
    return ms, nbytes


def decode_graph(cfgd, w, stream):
    """The decode step (one gtq_decode_attn per layer) captured in CUDA graphs,
    one per copy of the packed cache (replayed in turn, one step each)."""
    import torch

    import decode_attention_13_b200 as gtq

    T = cfgd["T"]
    graphs = []
    for c in range(w["copies"]):
        def step(c=c):
            for layer in range(cfgd["layers"]):
                gtq.gtq_decode_attn(w["plans"][layer], w["packed_copies"][c][layer], T,
                                    w["qs"][layer], w["outs"][layer], stream=stream)

        for _ in range(2):
            with torch.cuda.stream(stream):
                step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        stream.synchronize()
        graphs.append(graph)
    return graphs, None


def time_graph(graph, steps, warmup, stream, barrier=lambda: None):
    """ms per step over exactly `steps` replays (a list of graphs is replayed in
    turn: one step each)."""
    import torch

    graphs = graph if isinstance(graph, list) else [graph]
    for i in range(max(3, warmup)):
        graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for i in range(steps):
            graphs[i % len(graphs)].replay()
        t1.record(stream)
    torch.cuda.synchronize()
    barrier()
    return t0.elapsed_time(t1) / steps


def mixed_length_line(cfgd, w, dev, stream, hbm, steps, seed=11):
    """The batch's sequences at their own lengths (uniform in [T/4, T], int32
    lengths on the device, gtq_decode_attn_ex): bytes = the tokens each
    sequence holds."""
    import numpy as np
    import torch

    import decode_attention_13_b200 as gtq

    L, B, hkv, T = cfgd["layers"], cfgd["B"], cfgd["h_kv"], cfgd["T"]
    kb, vb = cfgd["k_bits"], cfgd["v_bits"]
    lens = np.random.default_rng(seed).integers(T // 4, T + 1, size=B).astype(np.int32)
    lens_dev = torch.from_numpy(lens).to(dev)
    stream.wait_stream(torch.cuda.current_stream(dev))
    lay = gtq.seq_layout(lens_dev)
    per_tok = w["step_bytes"] / (L * B * hkv * T)  # mean packed bytes per (token, head)

    def step():
        for layer in range(L):
            gtq.gtq_decode_attn_ex(w["plans"][layer], w["packed"][layer], T, w["qs"][layer],
                                   w["outs"][layer], layout=lay, stream=stream)

    g = _graph_of(step, stream)
    ms = time_graph(g, steps, 3, stream)
    nbytes = float(L * hkv * int(lens.sum())) * per_tok
    gbs = nbytes / (ms * 1e-3) / 1e9
    del g
    return {"decode_ms_per_step": ms, "decode_gbs": gbs, "decode_frac": gbs / hbm,
            "bytes_per_step": nbytes, "ctx_tokens_per_s": float(lens.sum()) / (ms * 1e-3),
            "seq_lens": "uniform in [T/4, T], mean %.0f" % float(lens.mean())}


def per_config_line(cfgd, rank, dev, stream, hbm, steps):
    """Decode and quantize-pack of one more workload, for the per_config block."""
    import torch

    w = build_workload(cfgd, rank, dev, stream)
    q_ms, q_bytes = time_quantize(cfgd, w, stream)
    graph, _ = decode_graph(cfgd, w, stream)
    ms = time_graph(graph, steps, 3, stream)
    gbs = w["step_bytes"] / (ms * 1e-3) / 1e9
    out = {"workload": cfgd["name"], "decode_ms_per_step": ms, "decode_gbs": gbs,
           "decode_frac": gbs / hbm, "ctx_tokens_per_s": cfgd["B"] * cfgd["T"] / (ms * 1e-3),
           "bytes_per_step": w["step_bytes"], "quantize_pack_ms": q_ms,
           "quantize_pack_gbs": q_bytes / (q_ms * 1e-3) / 1e9,
           "quantize_pack_frac": q_bytes / (q_ms * 1e-3) / 1e9 / hbm,
           "timed_steps": steps, "cache_copies_cycled": w["copies"]}
    del graph
    if cfgd["B"] > 1:
        out["mixed_lengths"] = mixed_length_line(cfgd, w, dev, stream, hbm, steps)
    del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def _graph_of(fn, stream):
    import torch

    for _ in range(2):
        with torch.cuda.stream(stream):
            fn()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn()
    stream.synchronize()
    return g


def decode_variants(cfgd, w, dev, stream, hbm, steps, window=128, seed=7):
    """The decode step of the same workload in the library's other modes, each
    captured in a CUDA graph and timed like the headline: a paged pool (pages
    in shuffled order, gtq_decode_attn_ex with a block table), K-only plans
    (keys coded, values read in fp16, gtq_decode_attn_full) and an fp16 window
    of recent tokens beside the packed cache, and twice the query heads per KV
    head."""
    import numpy as np
    import torch

    import decode_attention_13_b200 as gtq

    L, B, hq, hkv, T = cfgd["layers"], cfgd["B"], cfgd["h_q"], cfgd["h_kv"], cfgd["T"]
    kb, vb = cfgd["k_bits"], cfgd["v_bits"]
    out = {}

    def line(ms, nbytes, **kw):
        gbs = nbytes / (ms * 1e-3) / 1e9
        d = {"decode_ms_per_step": ms, "decode_gbs": gbs, "decode_frac": gbs / hbm,
             "bytes_per_step": nbytes, "timed_steps": steps}
        d.update(kw)
        return d

    torch.cuda.current_stream(dev).wait_stream(stream)
    ref = [o.clone() for o in w["outs"]]
    # ---- paged pool
    tb = gtq.gtq_layout_tile_bytes(kb, vb)
    n_tiles = (T + 63) // 64
    rng = np.random.default_rng(seed)
    pools, tables = [], []
    for layer in range(L):
        perm = torch.from_numpy(rng.permutation(B * n_tiles).astype(np.int64)).to(dev)
        src = w["packed"][layer][:B * hkv * n_tiles * tb].view(B, hkv, n_tiles, tb)
        pool = torch.empty(B * n_tiles * hkv * tb, dtype=torch.uint8, device=dev)
        pool.view(B * n_tiles, hkv, tb)[perm] = src.permute(0, 2, 1, 3).reshape(B * n_tiles, hkv, tb)
        pools.append(pool)
        tables.append(perm.view(B, n_tiles).to(torch.int32).contiguous())
    stream.wait_stream(torch.cuda.current_stream(dev))  # pools and tables built on torch's stream
    lays = [gtq.seq_layout(None, t) for t in tables]

    def paged():
        for layer in range(L):
            gtq.gtq_decode_attn_ex(w["plans"][layer], pools[layer], T, w["qs"][layer],
                                   w["outs"][layer], layout=lays[layer], stream=stream)

    g = _graph_of(paged, stream)
    ms = time_graph(g, steps, 3, stream)
    diff = max(float((o - r).abs().max()) for o, r in zip(w["outs"], ref))
    out["paged"] = line(ms, w["step_bytes"], max_abs_diff_vs_contiguous=diff,
                        how="pages of one tile of every KV head, shuffled block table")
    del g, pools, tables, lays
    # ---- K-only plans (fp16 values)
    plans, packed, g_k = [], [], []
    for layer, (k, v) in enumerate(w["kv"]):
        cfg = gtq.make_config(B, hq, hkv, kb, 0, T)
        with torch.cuda.stream(stream):
            p = gtq.gtq_alloc_bits(cfg, k, T, stream=stream)
            buf = torch.empty(p.packed_bytes, dtype=torch.uint8, device=dev)
            gtq.gtq_quantize_pack(p, k, None, 0, T, buf, stream=stream)
        plans.append(p)
        packed.append(buf)
    stream.synchronize()
    for p in plans:
        bits = gtq.gtq_get_bits(p)
        g_k.append([[len(set(int(x) for x in bits[b, h] if x > 0)) for h in range(hkv)]
                    for b in range(B)])
    kvs = [gtq.fp16_kv(v=v) for (_, v) in w["kv"]]

    def konly():
        for layer in range(L):
            gtq.gtq_decode_attn_full(plans[layer], packed[layer], T, w["qs"][layer],
                                     w["outs"][layer], kv=kvs[layer], stream=stream)

    g = _graph_of(konly, stream)
    ms = time_graph(g, steps, 3, stream)
    nbytes = float(sum(T * packed_bytes_per_token_head(kb, 0, g_k[l][b][h])
                       for l in range(L) for b in range(B) for h in range(hkv)))
    out["key_only"] = line(ms, nbytes, k_bits=kb, v_bits=0,
                           how="keys coded at k_bits, values read in fp16 from the caller's "
                               "tensor (gtq_decode_attn_full)")
    del g, plans, packed, kvs
    # ---- fp16 window of recent tokens beside the packed cache
    gen = torch.Generator(device=dev).manual_seed(seed)
    rks = [torch.randn((B, hkv, window, 128), generator=gen, device=dev, dtype=torch.float16)
           for _ in range(L)]
    rvs = [torch.randn((B, hkv, window, 128), generator=gen, device=dev, dtype=torch.float16)
           for _ in range(L)]
    stream.wait_stream(torch.cuda.current_stream(dev))
    wkv = [gtq.fp16_kv(recent_k=a, recent_v=b) for a, b in zip(rks, rvs)]

    def windowed():
        for layer in range(L):
            gtq.gtq_decode_attn_full(w["plans"][layer], w["packed"][layer], T, w["qs"][layer],
                                     w["outs"][layer], kv=wkv[layer], stream=stream)

    g = _graph_of(windowed, stream)
    ms = time_graph(g, steps, 3, stream)
    out["window"] = line(ms, w["step_bytes"] + float(L * B * hkv * window * 512),
                         window_tokens=window,
                         how="K%dV%d cache plus %d fp16 recent tokens per head in one softmax"
                             % (kb, vb, window))
    del g, rks, rvs, wkv
    # ---- twice the query heads per KV head (two decode units of 8 per KV head)
    plans2, q2, o2 = [], [], []
    for layer, (k, _) in enumerate(w["kv"]):
        cfg = gtq.make_config(B, 2 * hq, hkv, kb, vb, T)
        with torch.cuda.stream(stream):
            plans2.append(gtq.gtq_alloc_bits(cfg, k, T, stream=stream))
        q2.append(w["qs"][layer].repeat(1, 2, 1))
        o2.append(torch.empty((B, 2 * hq, 128), dtype=torch.float32, device=dev))
    stream.wait_stream(torch.cuda.current_stream(dev))
    stream.synchronize()
    # same keys, so the same allocation: the packed caches serve these plans too
    same = all(np.array_equal(gtq.gtq_get_bits(p2), gtq.gtq_get_bits(p1))
               for p1, p2 in zip(w["plans"], plans2))

    def wide():
        for layer in range(L):
            gtq.gtq_decode_attn(plans2[layer], w["packed"][layer], T, q2[layer], o2[layer],
                                stream=stream)

    if same:
        g = _graph_of(wide, stream)
        ms = time_graph(g, steps, 3, stream)
        out["q_group_x2"] = line(ms, w["step_bytes"], q_heads=2 * hq,
                                 how="%d query heads per KV head (decode units of 8 query heads, "
                                     "each streaming the KV head's cache)" % (2 * hq // hkv))
        del g
    del plans2, q2, o2
    torch.cuda.synchronize()
    return out


def memory_report(cfgd, rank, dev, stream, seq_lens=(131072, 262144, 524288)):
    """Peak device memory of the packed-cache serving state of the stack at
    several context lengths: every layer's plan and packed cache built layer by
    layer (one layer's fp16 K/V alive at a time), then one decode step; against
    the size of the same cache in fp16."""
    import torch

    import decode_attention_13_b200 as gtq
    from decode_attention_13_b200 import synth

    L, B, hq, hkv = cfgd["layers"], cfgd["B"], cfgd["h_q"], cfgd["h_kv"]
    kb, vb, gq = cfgd["k_bits"], cfgd["v_bits"], cfgd["h_q"] // cfgd["h_kv"]
    rows = []
    for T in seq_lens:
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        plans, packed, qs, outs, plan_bytes = [], [], [], [], 0
        for layer in range(L):
            k, v, q = synth.layer_torch((cfgd["index"], rank, layer), B, hkv, gq, T,
                                        theta=cfgd["theta"], decay=cfgd["decay"], device=dev)
            stream.wait_stream(torch.cuda.current_stream(dev))
            cfg = gtq.make_config(B, hq, hkv, kb, vb, T)
            with torch.cuda.stream(stream):
                plan = gtq.gtq_alloc_bits(cfg, k, T, stream=stream)
                buf = torch.empty(plan.packed_bytes, dtype=torch.uint8, device=dev)
                gtq.gtq_quantize_pack(plan, k, v, 0, T, buf, stream=stream)
            stream.synchronize()
            plan_bytes += gtq.gtq_plan_device_bytes(plan)
            plans.append(plan)
            packed.append(buf)
            qs.append(q)
            outs.append(torch.empty((B, hq, 128), dtype=torch.float32, device=dev))
            del k, v
        with torch.cuda.stream(stream):
            for layer in range(L):
                gtq.gtq_decode_attn(plans[layer], packed[layer], T, qs[layer], outs[layer],
                                    stream=stream)
        stream.synchronize()
        peak = torch.cuda.max_memory_allocated(dev) - base + plan_bytes
        resident = sum(b.numel() for b in packed) + plan_bytes
        fp16 = L * B * hkv * T * 2 * 128 * 2
        rows.append({"seq_len": T, "peak_bytes": int(peak), "resident_cache_bytes": int(resident),
                     "fp16_cache_bytes": int(fp16), "fp16_over_resident": fp16 / resident})
        del plans, packed, qs, outs
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return {"workload": cfgd["name"] + " (context varied)", "rows": rows,
            "how": "torch.cuda.max_memory_allocated over building the stack layer by layer "
                   "(one layer's fp16 K/V alive at a time) and one decode step, plus the plans' "
                   "own device memory (gtq_plan_device_bytes); fp16 = the same K/V cache in fp16; "
                   "no model weights are involved"}


# ------------------------------------------------------------------ our arm
def run_ours(args, rank, world):
    import numpy as np
    import torch

    import decode_attention_13_b200 as gtq
    from decode_attention_13_b200 import synth

    cfgd = dict(synth.CONFIGS[args.config], index=args.config)
    if args.seq_len:
        cfgd["T"] = args.seq_len
        cfgd["name"] += " (context overridden to %d)" % args.seq_len
    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    L, B, hq, hkv, T = cfgd["layers"], cfgd["B"], cfgd["h_q"], cfgd["h_kv"], cfgd["T"]
    assert cfgd["dtype"] == "fp16"
    stream = torch.cuda.Stream(device=dev)
    hbm, peak_kind = peaks()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    w = build_workload(cfgd, rank, dev, stream)
    step_bytes = w["step_bytes"]
    # ---- prefill timing: quantize-pack of every layer (A3-A6)
    quant_ms, quant_bytes = time_quantize(cfgd, w, stream)

    # ---- decode-time append: one new token into every layer's packed cache
    # (the allocation stays the one computed at prefill), captured in a graph
    def append_step():
        for layer, (k, v) in enumerate(w["kv"]):
            gtq.gtq_quantize_pack(w["plans"][layer], k, v, T - 1, 1, w["packed"][layer],
                                  stream=stream)

    with torch.cuda.stream(stream):
        append_step()
    stream.synchronize()
    agraph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(agraph, stream=stream):
        append_step()
    append_ms = time_graph(agraph, 50, 3, stream)
    del agraph

    # ---- the decode step, captured in a CUDA graph (only decode_kernel runs in it)
    graph, _ = decode_graph(cfgd, w, stream)
    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    # warm-up after the sampler's start, so the timed steps begin at full clocks
    for i in range(max(3, args.warmup)):
        graph[i % len(graph)].replay()
    torch.cuda.synchronize()
    copies = w["copies"]  # graphs over different copies of the cache, replayed in turn
    ms_local = time_graph(graph, args.steps, 0, stream, barrier)
    timed_steps = args.steps
    clk = clocks.stop()
    ms = max_over_ranks(ms_local, world, dev)

    # ---- latency of one eager gtq_decode_attn call (events around each call)
    call_ms = []
    with torch.cuda.stream(stream):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(L)]
        for _ in range(2):
            for layer in range(L):
                a, b = evs[layer]
                a.record(stream)
                gtq.gtq_decode_attn(w["plans"][layer], w["packed"][layer], T, w["qs"][layer],
                                    w["outs"][layer], stream=stream)
                b.record(stream)
            stream.synchronize()
            call_ms.append([a.elapsed_time(b) for a, b in evs])
    eager_call_ms = statistics.mean(call_ms[-1])

    # ---- end to end through the ABI with host buffers
    q_host = torch.stack(w["qs"]).cpu().pin_memory()
    out_host = torch.empty((L, B, hq, 128), dtype=torch.float32).pin_memory()
    q_dev = torch.empty_like(q_host, device=dev)
    out_dev = torch.empty((L, B, hq, 128), dtype=torch.float32, device=dev)

    def e2e_step(i):
        q_dev.copy_(q_host, non_blocking=True)
        packed = w["packed_copies"][i % copies]
        for layer in range(L):
            gtq.gtq_decode_attn(w["plans"][layer], packed[layer], T, q_dev[layer],
                                out_dev[layer], stream=stream)
        out_host.copy_(out_dev, non_blocking=True)

    e2e_steps = max(20, min(args.steps, 200))
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            e2e_step(i)
    stream.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        for i in range(e2e_steps):
            e2e_step(i)
        e1.record(stream)
    stream.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world, dev)
    ref_check = np.isfinite(out_host.numpy()).all()
    del graph
    variants = None
    if rank == 0 and world == 1 and not args.no_extra and not args.seq_len:
        variants = decode_variants(cfgd, w, dev, stream, hbm, min(args.steps, 400))
    del w
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # ---- CPU baseline (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, heads, spent, _ = oracle_decode_sample(cfgd, oracle_pool(cfgd), args.cpu_seconds)
        threads = oracle_threads()
        cpu = {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
               "sample": "fp64 oracle decode of %d whole KV heads (T=%d, %d query heads "
                         "each), %.1f s of CPU work" % (heads, T, hq // hkv, spent)}

    # ---- the other workloads and the memory report (rank 0 at N = 1)
    extra = {}
    if rank == 0 and world == 1 and not args.no_extra and not args.seq_len:
        pc = {}
        for c in (1, 3, 4):
            if c == args.config:
                continue
            d = dict(synth.CONFIGS[c], index=c)
            pc[str(c)] = per_config_line(d, rank, dev, stream, hbm, 100 if c == 3 else 400)
        extra["per_config"] = pc
        if args.config == 2:
            extra["memory"] = memory_report(cfgd, rank, dev, stream)

    value = world * step_bytes / (ms * 1e-3) / 1e9
    launch_ms = ms / L  # the graph step runs only decode_kernel, L launches back to back
    achieved = (step_bytes / L) / (launch_ms * 1e-3) / 1e9
    traffic = profile_traffic(os.path.join(ROOT, "decode_attention_13_b200", "csrc",
                                           "gtq_decode.cu"))
    n_launch = L * timed_steps  # one decode_kernel launch per layer per step (graph nodes)
    res = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": timed_steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16 operands / f32 accumulate", "data": "synthetic",
        "config": workload_config(cfgd, world),
        "pct_hbm_peak": 100.0 * value / world / hbm, "hbm_peak_gbs": hbm,
        "pct_hbm_nominal_8tbs": 100.0 * value / world / 8000.0,
        "ctx_tokens_per_s": world * B * T / (ms * 1e-3),
        "bytes_per_step": step_bytes,
        "fp16_bytes_per_step": float(L * B * hkv * T * 512),
        "compression_vs_fp16": float(L * B * hkv * T * 512) / step_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "kernel": "decode_kernel: one launch per layer (query rotation, split-K "
                               "decode and split merge fused); average launch duration = the "
                               "graph-timed step (CUDA events on the launching stream, only "
                               "decode_kernel inside) divided by its %d launches" % L,
                     "bytes_per_launch": step_bytes / L, "launch_us": 1e3 * launch_ms,
                     "eager_call_us": 1e3 * eager_call_ms,
                     "peak_kind": peak_kind},
        "prefill": {"quantize_pack_ms_all_layers": quant_ms,
                    "quantize_pack_gbs": quant_bytes / (quant_ms * 1e-3) / 1e9,
                    "quantize_pack_frac": quant_bytes / (quant_ms * 1e-3) / 1e9 / hbm,
                    "bytes": quant_bytes,
                    "kernels": "quantize_tc_kernel (full 128-token tiles) + quantize_kernel "
                               "(ragged edges, none at this T); one gtq_quantize_pack call "
                               "per layer, CUDA events around all layers"},
        "append": {"tokens_per_layer": 1, "layers": L, "ms_per_step": append_ms,
                   "us_per_layer_token": 1e3 * append_ms / L,
                   "how": "gtq_quantize_pack(t0 = T - 1, n = 1) on every layer, captured in a "
                          "CUDA graph, under the allocation computed at prefill"},
        "e2e": {"value": world * step_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
                "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": int(q_host.numel() * q_host.element_size()),
                "d2h_bytes_per_step": int(out_host.numel() * out_host.element_size()),
                "path": "pinned host q -> gtq_decode_attn per layer (eager) -> pinned host out; "
                        "the packed cache stays resident"},
        "gpu_launches": n_launch,
        "clocks": clk,
        "outputs_finite": bool(ref_check),
    }
    res.update(extra)
    if variants:
        res["variants"] = variants
    if cpu:
        res["cpu_baseline"] = cpu
    if rank == 0:
        print(json.dumps(res), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
