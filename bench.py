"""Benchmark of the mixed-precision KV decode step on B200.

One step = for every layer of the stack: append one new token per sequence
and decode attention for every query head (kvq_decode_step: one fused kernel
per layer-step), over a cache prefilled to the workload's context with one
full-context kvq_append per layer (timed too: append tokens/s). Default
workload, the largest: the long-context ragged Llama-3.1-8B-shaped stack
(32 layers, layers 0 and 31 bf16, the rest K8V8, 32 query / 8 KV heads,
head_dim 128, batch 4, per-sequence context 8K-32K). The same line carries the
uniform K4V4 (batch 16 x 4K), mixed 3.25-bit (batch 64, short contexts) and
Qwen2.5-7B-shaped 4.0-bit (batch 32 x 8K) stacks under `per_config`.

value = algorithmic HBM bytes per step (packed codes, fp16 scales/zeros, bf16
window of every layer at the step's context) / device time per step, in GB/s.
Every cache is far larger than the 126 MB L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from layer_wise_mixed_kvq_b200 import replicas, synth  # noqa: E402

METRIC = "quantized-KV decode attention HBM GB/s (% of B200 peak) and decode steps/s"
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="ragged_long", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' lines (llama_k4v4, llama_mixed325, qwen_mixed40)")
    ap.add_argument("--no-extras", action="store_true",
                    help="time the step only (no isolated-launch, end-to-end or graph pass; for profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=16.0)
    ap.add_argument("--layers", type=int, default=0,
                    help="profile a truncated stack (N layers from --first-layer); 0 = the workload's full stack")
    ap.add_argument("--first-layer", type=int, default=0, help="first layer of a truncated stack")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of the sources the decode step kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "layer_wise_mixed_kvq_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if (name.startswith("kvq_decode") and name.endswith(".cu")) or name.endswith(".cuh"):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(workload):
    """The committed ncu DRAM counters of one decode launch of the workload's
    shapes, only if they were taken on the current kernel source (else None):
    the entry's traffic_ratio is DRAM bytes / algorithmic bytes of that launch."""
    path = os.path.join(PROFILES, "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("counters_taken_at") != kernel_source_hash():
        return None
    return e


# --------------------------------------------------------------- clocks --
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------- CPU oracle --
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_baseline(w, seconds, threads=(1,)):
    """The oracle, as it stands, timed on this host on a bounded sample of the
    workload. One oracle layer per distinct pair of the layer map, holding the
    workload's whole batch at its context (+1, the step's token; prefill appends
    untimed); each is attended repeatedly with fresh queries for its share of
    `seconds` per thread count, the (sequence, KV head) units shared out over
    that many host threads. The stack's rate weights every pair by its layer
    count: GB/s = sum of layer bytes / sum of layer times. One result per entry
    of `threads`."""
    import oracle
    oracle.build()
    lens = synth.context_lengths(w) + 1
    pairs = []
    for layer, pair in enumerate(w.layer_map):
        if pair not in [p for p, _, _ in pairs]:
            pairs.append((pair, layer, sum(1 for q in w.layer_map if q == pair)))
    per_pair = seconds / len(pairs) / len(threads)
    acc = {n: {"stack_s": 0.0, "reps": 0, "t": 0.0} for n in threads}
    stack_bytes = 0.0
    for pair, layer, count in pairs:
        key_mode = pair[2] if len(pair) > 2 else 0
        fmt = pair[3] if len(pair) > 3 else 0
        scales = w.fp8_scales if fmt else (None, None)
        L = oracle.OracleLayer(pair[0], pair[1], w.batch, w.n_kv_heads, w.head_dim, key_mode=key_mode, fmt=fmt,
                               k_scales=scales[0], v_scales=scales[1])
        K, V = synth.kv_tokens(w, layer, int(lens.sum()))
        L.append(K, V, [int(x) for x in lens])
        del K, V
        page = oracle.page_bytes(pair[0], pair[1], w.head_dim, key_mode, fmt)
        stack_bytes += count * w.n_kv_heads * sum((int(T) // 32) * page + (int(T) % 32) * w.head_dim * 4
                                                  for T in lens)
        for n in threads:
            t, reps = 0.0, 0
            while reps == 0 or t < per_pair:
                Q = synth.queries(w, layer, salt=100 + reps)
                t0 = time.perf_counter()
                L.attend(Q, threads=n)
                t += time.perf_counter() - t0
                reps += 1
            acc[n]["stack_s"] += count * t / reps
            acc[n]["reps"] += reps
            acc[n]["t"] += t
        del L
    out = []
    for n in threads:
        a = acc[n]
        out.append({"value": stack_bytes / a["stack_s"] / 1e9, "unit": "GB/s", "cores": n, "kind": "oracle",
                    "sample": f"{a['reps']} whole-layer attention(s) of {w.name} (batch {w.batch}, all "
                              f"{w.n_q_heads} query heads, context {int(lens.min())}-{int(lens.max())}), one "
                              f"oracle layer per distinct pair ({len(pairs)}), fp64 attention on {n} host "
                              f"thread(s), {a['t']:.1f} s of attention; the stack rate weights the pairs by "
                              f"layer count",
                    "ms_per_step": a["stack_s"] * 1e3})
    return out


def cpu_baselines(w, seconds):
    """All host cores (the reported baseline) with one thread beside it."""
    allc, one = cpu_baseline(w, seconds, threads=(host_cores(), 1))
    allc["single_thread"] = {k: one[k] for k in ("value", "unit", "cores", "sample", "ms_per_step")}
    return allc


def workload_config(w, equiv_bits, world):
    """The `config` object both arms print (the GPU arm's workload, whatever the arm samples)."""
    return {"workload": w.name, "layers": w.n_layers, "layer_map_equiv_bits": equiv_bits, "batch": w.batch,
            "n_q_heads": w.n_q_heads, "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
            "context": int(synth.context_lengths(w).max()),
            "context_min": int(synth.context_lengths(w).min()), "parallelism": f"replicas x{world}",
            "l2": "cache larger than L2 (no flush)"}


def oracle_equiv_bits(w):
    import oracle
    return oracle.equiv_bits([p[:2] for p in w.layer_map])


def run_reference(args, w):
    rank, world, _ = replicas.world()
    if rank != 0:
        return 0
    cb = cpu_baseline(w, args.cpu_seconds, threads=(host_cores(),))[0]
    value = cb["value"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup,
        # one step = every layer of the stack over the whole batch (the GPU arm's step)
        "ms_per_step": cb["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, oracle_equiv_bits(w), 1),
        "cpu_baseline": {k: cb[k] for k in ("kind", "cores", "sample")} | {"value": value, "unit": "GB/s"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ GPU --
PER_CONFIG = ("llama_k4v4", "llama_mixed325", "qwen_mixed40")


def prefill_bytes(w, kvq, lens):
    """Algorithmic bytes of prefilling every layer from empty with one kvq_append:
    the bf16 keys and values read, the pages and window rows written."""
    total = 0
    for pair in w.layer_map:
        pb = kvq.kvq_page_bytes(pair, w.head_dim)
        for T in lens:
            T = int(T)
            total += w.n_kv_heads * (T * 4 * w.head_dim + (T // 32) * pb + (T % 32) * 4 * w.head_dim)
    return total


def measure(w, args, world, full):
    """Prefill the workload's cache, then time K decode steps (kvq_decode_step for
    every layer: one kernel per layer-step). `full` adds the event-per-launch pass,
    the end-to-end and CUDA-graph measurements and the clock record."""
    import torch
    from layer_wise_mixed_kvq_b200 import kvq
    dev = torch.device("cuda", torch.cuda.current_device())
    rank = replicas.world()[0]
    B, Hq, Hkv, D, NL = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim, w.n_layers
    lens = synth.context_lengths(w)
    total_steps = args.warmup + args.steps
    graph_steps = max(3, min(args.steps, 20))
    extra = (args.steps + graph_steps + 2) if full else 0
    max_tokens = int(lens.max()) + total_steps + extra + 32
    cache = kvq.kvq_cache_create(list(w.layer_map), Hq, Hkv, D, B, max_tokens)
    for layer, pair in enumerate(w.layer_map):
        if len(pair) > 3 and pair[3]:
            kvq.kvq_set_fp8_scales(cache, layer, w.fp8_scales[0], w.fp8_scales[1])
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.seed * 1000 + rank)
    stream = torch.cuda.current_stream()
    peak, peak_kind = peaks()

    # ---- every append kernel the prefill uses is launched once on a scratch cache
    # first: a kernel's first launch also loads it, which must not be timed
    warm = kvq.kvq_cache_create(list(w.layer_map), Hq, Hkv, D, 1, 64)
    for layer, pair in enumerate(w.layer_map):
        if len(pair) > 3 and pair[3]:
            kvq.kvq_set_fp8_scales(warm, layer, w.fp8_scales[0], w.fp8_scales[1])
    Kw = torch.zeros((40, Hkv, D), device=dev, dtype=torch.bfloat16)
    for layer in range(NL):
        kvq.kvq_append(warm, layer, Kw, Kw, [40], stream)
    torch.cuda.synchronize()
    kvq.kvq_cache_destroy(warm)
    del Kw

    # ---- prefill: one kvq_append of the full context per layer (append tokens/s).
    # A ~1 ms device-side sleep ahead of the start event keeps the stream busy
    # while the host prepares and launches the append, so the events time the
    # device work only.
    pre_ms = 0.0
    for layer in range(NL):
        K, V = synth.torch_kv_tokens(w, layer, int(lens.sum()), dev, gen)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        torch.cuda._sleep(2_000_000)
        e0.record(stream)
        kvq.kvq_append(cache, layer, K, V, [int(x) for x in lens], stream)
        e1.record(stream)
        torch.cuda.synchronize()
        pre_ms += e0.elapsed_time(e1)
        del K, V
    pre_bytes = prefill_bytes(w, kvq, lens)
    pre_gbs = pre_bytes / (pre_ms / 1e3) / 1e9
    append = {"tokens_per_s": int(lens.sum()) * NL / (pre_ms / 1e3), "unit": "token-layers/s",
              "roofline": {"bound": "hbm", "achieved": pre_gbs, "peak": peak, "unit": "GB/s", "frac": pre_gbs / peak,
                           "peak_kind": peak_kind, "bytes": pre_bytes,
                           "kernel": "append_kernel, full-context prefill of every layer (bf16 K, V in; pages "
                                     "and window rows out), CUDA events around each launch"}}

    # ---- per-step inputs resident in HBM
    steps_K, steps_V, steps_Q = [], [], []
    for s in range(total_steps):
        kl, vl, ql = [], [], []
        for layer in range(NL):
            k1, v1 = synth.torch_kv_tokens(w, layer, B, dev, gen)
            kl.append(k1)
            vl.append(v1)
            ql.append(torch.randn((B, Hq, D), device=dev, generator=gen).to(torch.bfloat16))
        steps_K.append(kl)
        steps_V.append(vl)
        steps_Q.append(ql)
    outs = [torch.empty((B, Hq, D), device=dev, dtype=torch.float32) for _ in range(NL)]

    def step(s, events=None):
        # one decode step per layer through the public call: kvq_decode_step appends
        # the layer's new token and attends, in one kernel
        for layer in range(NL):
            if events is not None:
                events[layer][0].record(stream)
            kvq.kvq_decode_step(cache, layer, steps_K[s][layer], steps_V[s][layer], steps_Q[s][layer],
                                outs[layer], stream)
            if events is not None:
                events[layer][1].record(stream)

    def step_bytes():
        return sum(kvq.kvq_bytes(cache, layer, B, True) for layer in range(NL))

    for s in range(args.warmup):
        step(s)
    torch.cuda.synchronize()
    bytes_before = step_bytes()
    launches0 = kvq.kvq_launch_count(cache)
    with ClockSampler(dev.index) as clk:
        # The timed region: K steps enqueued back to back with no event between
        # kernels (an event between two launches stops the next one from starting
        # under the tail of the previous one). Every launch is the fused decode kernel.
        replicas.barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for s in range(args.steps):
            step(args.warmup + s)
        t1.record(stream)
        torch.cuda.synchronize()
        replicas.barrier()
    launches = kvq.kvq_launch_count(cache) - launches0
    bytes_after = step_bytes()
    # the step at context c reads the cache after its own append
    bytes_per_step = (bytes_before + bytes_after) / 2.0
    local_ms = t0.elapsed_time(t1)
    total_bytes, max_ms, _ = replicas.aggregate(bytes_per_step * args.steps, local_ms)
    ms_per_step = max_ms / args.steps
    value = total_bytes / (max_ms / 1e3) / 1e9
    launch_us = local_ms * 1e3 / (args.steps * NL)
    # DRAM traffic of a launch: the captured launch's bytes per algorithmic byte
    # times this run's algorithmic bytes per launch (the capture ran a 2-layer
    # stack of the same shapes; the traffic grows with the units processed)
    prof = traffic_from_profile(w.name)
    traffic = prof["traffic_ratio"] * bytes_per_step / NL if prof else None
    res = {
        "value": value, "unit": "GB/s", "ms_per_step": ms_per_step, "decode_steps_per_s": 1e3 / ms_per_step,
        "tokens_per_s": B * world * 1e3 / ms_per_step, "bytes_per_step": bytes_per_step,
        "append_prefill_tokens_per_s": append["tokens_per_s"], "append": append,
        "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak, "unit": "GB/s",
                     "frac": value / world / peak, "traffic": traffic,
                     "traffic_ratio": prof["traffic_ratio"] if prof else None, "peak_kind": peak_kind,
                     "avg_launch_us": launch_us, "algorithmic_bytes_per_launch": bytes_per_step / NL,
                     "kernel": "fused decode step (decode_mma_kernel / decode_warp_kernel with the one-token "
                               "append): every launch of the timed region, average duration = region / launches"},
        "gpu_launches": launches, "clocks": clk.summary(),
    }
    if full:
        # each launch alone: an event pair around every decode step kernel (no
        # overlap with its neighbours), the same K steps one token later
        ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(NL)]
              for _ in range(args.steps)]
        b0 = step_bytes()
        torch.cuda.synchronize()
        for s in range(args.steps):
            step(args.warmup + s, ev[s])
        torch.cuda.synchronize()
        iso_us = float(np.mean([ev[s][l][0].elapsed_time(ev[s][l][1]) for s in range(args.steps)
                                for l in range(NL)])) * 1e3
        iso_gbs = ((b0 + step_bytes()) / 2.0 / NL) / (iso_us / 1e6) / 1e9
        res["roofline"]["isolated_launch"] = {"avg_us": iso_us, "achieved": iso_gbs, "frac": iso_gbs / peak}

        # ---- end to end through the public API with host buffers: every step copies
        # that step's K, V and Q for all layers from one pinned buffer to the device,
        # runs the layer-steps on views of it, and copies all outputs back
        e2e_steps = max(3, min(args.steps, 20))
        n_kv = B * Hkv * D
        row = 2 * n_kv + B * Hq * D
        dstage = torch.empty((NL, row), device=dev, dtype=torch.bfloat16)
        dK = [dstage[layer, :n_kv].view(B, Hkv, D) for layer in range(NL)]
        dV = [dstage[layer, n_kv:2 * n_kv].view(B, Hkv, D) for layer in range(NL)]
        dQ = [dstage[layer, 2 * n_kv:].view(B, Hq, D) for layer in range(NL)]
        hstage = []
        for s in range(e2e_steps):
            src = s % total_steps
            hs = torch.empty((NL, row), dtype=torch.bfloat16).pin_memory()
            for layer in range(NL):
                hs[layer, :n_kv].copy_(steps_K[src][layer].reshape(-1).cpu())
                hs[layer, n_kv:2 * n_kv].copy_(steps_V[src][layer].reshape(-1).cpu())
                hs[layer, 2 * n_kv:].copy_(steps_Q[src][layer].reshape(-1).cpu())
            hstage.append(hs)
        douts = torch.empty((NL, B, Hq, D), device=dev, dtype=torch.float32)
        hout = torch.empty((NL, B, Hq, D), dtype=torch.float32).pin_memory()
        h2d = hstage[0].numel() * hstage[0].element_size()
        d2h = hout.numel() * hout.element_size()
        e2e_bytes0 = step_bytes()
        replicas.barrier()
        torch.cuda.synchronize()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for s in range(e2e_steps):
            dstage.copy_(hstage[s], non_blocking=True)
            for layer in range(NL):
                kvq.kvq_decode_step(cache, layer, dK[layer], dV[layer], dQ[layer], douts[layer], stream)
            hout.copy_(douts, non_blocking=True)
        b_.record(stream)
        torch.cuda.synchronize()
        replicas.barrier()
        e2e_bytes = (e2e_bytes0 + step_bytes()) / 2.0
        e2e_total, e2e_max, _ = replicas.aggregate(e2e_bytes * e2e_steps, a.elapsed_time(b_))
        res["e2e"] = {"value": e2e_total / (e2e_max / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "steps": e2e_steps, "ms_per_step": e2e_max / e2e_steps}

        # ---- the same step captured once in a CUDA graph and replayed (device
        # lengths; inputs in static buffers)
        gK = [t.clone() for t in steps_K[0]]
        gV = [t.clone() for t in steps_V[0]]
        gQ = [t.clone() for t in steps_Q[0]]
        gstream = torch.cuda.Stream()
        gstream.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=gstream):
            for layer in range(NL):
                kvq.kvq_decode_step(cache, layer, gK[layer], gV[layer], gQ[layer], outs[layer])
        stream.wait_stream(gstream)
        graph.replay()                      # warm-up replay
        torch.cuda.synchronize()
        g_bytes0 = step_bytes()             # host mirror: includes the step recorded at capture
        replicas.barrier()
        torch.cuda.synchronize()
        ga, gb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ga.record(stream)
        for _ in range(graph_steps):
            graph.replay()
        gb.record(stream)
        torch.cuda.synchronize()
        replicas.barrier()
        kvq.kvq_refresh_lengths(cache)
        g_bytes = (g_bytes0 + step_bytes()) / 2.0
        g_total, g_max, _ = replicas.aggregate(g_bytes * graph_steps, ga.elapsed_time(gb))
        kvq.kvq_sync(cache)
        del graph
        res["graph"] = {"value": g_total / (g_max / 1e3) / 1e9, "unit": "GB/s", "steps": graph_steps,
                        "ms_per_step": g_max / graph_steps, "decode_steps_per_s": graph_steps / (g_max / 1e3) * world,
                        "note": "same step (kvq_decode_step per layer) captured in one CUDA graph, inputs resident"}
    kvq.kvq_sync(cache)
    kvq.kvq_cache_destroy(cache)
    return res


def run_gpu(args, w):
    import torch
    import torch.distributed as dist
    rank, world, local = replicas.world()
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", init_method="env://",
                                timeout=__import__("datetime").timedelta(seconds=120))
    from layer_wise_mixed_kvq_b200 import kvq

    head = measure(w, args, world, full=not args.no_extras)
    per_config = {}
    if not args.no_per_config and not args.layers:
        for name in PER_CONFIG:
            if name == w.name:
                continue
            r = measure(synth.WORKLOADS[name], args, world, full=False)
            per_config[name] = {k: r[k] for k in ("value", "unit", "ms_per_step", "decode_steps_per_s",
                                                  "append_prefill_tokens_per_s", "bytes_per_step", "gpu_launches")}
            per_config[name]["roofline"] = {k: r["roofline"][k] for k in ("achieved", "frac", "traffic",
                                                                          "traffic_ratio", "avg_launch_us")}
            per_config[name]["append_roofline_frac"] = r["append"]["roofline"]["frac"]
            per_config[name]["clocks"] = r["clocks"]
            per_config[name]["config"] = workload_config(synth.WORKLOADS[name],
                                                         kvq.kvq_equiv_bits(list(synth.WORKLOADS[name].layer_map)),
                                                         world)

    cb = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cb = cpu_baselines(w, args.cpu_seconds)

    result = {
        "metric": METRIC,
        "value": head["value"],
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": head["ms_per_step"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "operands": "f16 tensor-core operands (integer codes and e4m3 as exact f16, q * scale and p as exact or "
                    "hi+lo f16 pairs)",
        "data": "synthetic",
        "config": workload_config(w, kvq.kvq_equiv_bits(list(w.layer_map)), world),
        "pct_of_peak": head["roofline"]["frac"],
        "decode_steps_per_s": head["decode_steps_per_s"],
        "tokens_per_s": head["tokens_per_s"],
        "append_prefill_tokens_per_s": head["append_prefill_tokens_per_s"],
        "append": head["append"],
        "bytes_per_step": head["bytes_per_step"],
        "roofline": head["roofline"],
        "cpu_baseline": cb,
        "e2e": head.get("e2e"),
        "graph": head.get("graph"),
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "per_config": per_config,
    }
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.warmup < 3:
        print("warmup must be >= 3", file=sys.stderr)
        return 2
    w = synth.WORKLOADS[args.workload]
    if args.layers:
        import dataclasses
        w = dataclasses.replace(w, layer_map=w.layer_map[args.first_layer:args.first_layer + args.layers])
    if args.impl == "reference":
        return run_reference(args, w)
    return run_gpu(args, w)


if __name__ == "__main__":
    sys.exit(main())
