#!/usr/bin/env python
"""Benchmark of the packed KV-cache decode path on B200.

Workload (default): Qwen2.5-3B-shaped stack, 36 layers, 16 query / 2 KV
heads, head size 128, RoPE theta 1e6, batch 1, 128K context, K3V3 Block-GTQ
plans. Synthetic seeded inputs (synth.keys_values_torch); caches are built by
the library itself (energy + greedy plans + bulk quantize-append) before the
timed region.

Step = one decode step of the whole stack: per layer, one kvq_append_decode
launch quantize-appends the new token's key and value (1 token x 2 KV heads)
and runs packed decode attention over the layer's cache, the split merge
included. The step is captured in a CUDA graph. ``value`` = packed cache bytes read by decode attention per step
/ step time (GB/s). The packed caches of the 36 layers (944 MB) exceed L2, and
each layer's cache is read once per step, so no L2 flush is needed.

Also reported: decode-kernel roofline (the timed region over its launches;
the isolated launch time, CUDA events around each layer's decode call outside
the graph, beside it), bulk quantize throughput (prefill), an e2e
step through host buffers, SM clocks during the timed region, and the CPU
oracle timed on a bounded sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
Under torchrun each rank runs the same per-GPU work (weak scaling, no
data-path collective); rank 0 prints one JSON line.
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

import synth  # noqa: E402

BYTES_PER_TOKEN_HEAD = lambda bk, bv: 16 * (bk + bv) + 4  # noqa: E731  codes + 2 fp16 norms


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="qwen3b_128k",
                    choices=["qwen3b_128k", "llama8b", "qwen7b_serve", "qwen3b_sweep"])
    ap.add_argument("--context", type=int, default=0,
                    help="override the context length (points of the qwen3b_sweep)")
    ap.add_argument("--alloc", default="greedy", choices=["greedy", "uniform"],
                    help="Block-GTQ greedy widths, or every block at the key budget")
    ap.add_argument("--paged", type=int, default=0,
                    help="paged caches with this many 32-token tiles per page (pages handed "
                         "out in a shuffled order); 0: one contiguous cache per sequence")
    ap.add_argument("--rotate-keys", action="store_true",
                    help="plans with the per-width-group key rotation (KVQ_ALLOC_ROTATE_KEYS)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--layers", type=int, default=0,
                    help="override the layer count (small cases for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the timed oracle sample (sweep points)")
    ap.add_argument("--no-bf16", action="store_true",
                    help="skip the bf16 comparator (dense decode over an unquantized cache)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the other workloads (llama8b layer, qwen7b serving step, context "
                         "sweep with greedy and uniform plans, 512K x 36-layer prefill)")
    ap.add_argument("--dist-steps", type=int, default=0,
                    help="replays timed one by one for the step-time distribution "
                         "(default: >= 100 and >= 1 s)")
    return ap.parse_args()


# ------------------------------------------------------------------ helpers
def rank_max(x, dist, device="cpu"):
    """Max over ranks of a per-rank number (a job's time is its slowest
    rank's); x itself without a process group."""
    if dist is None:
        return float(x)
    import torch

    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, world, ms):
    """Whole-job throughput: the units all ranks processed over the slowest
    rank's time (weak scaling: every rank has the same per-GPU work)."""
    return world * units_per_rank / (ms / 1e3)


def rank_seed(seed, rank, b):
    """Synthetic-data seed of sequence b on a rank: ranks hold different
    sequences of the same shapes."""
    return seed * 1000 + rank * 100 + b


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def code_only(text):
    """C++ source without comments and blank space: what the compiler sees,
    so a comment edit does not retire counters taken on the same code."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def decode_source_hash():
    """Hash of the decode kernel's code (its source files, comments left out)."""
    h = hashlib.sha256()
    for f in ("decode.cu", "common.cuh", "splitk.cuh", "quant_dev.cuh"):
        with open(os.path.join(ROOT, "bit_kv_cache_19_b200", "csrc", f)) as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def profiled(workload, key):
    """A per-launch counter of the decode kernel (DRAM bytes, warp
    instructions) from a committed ncu summary, only if it was taken on the
    current decode source."""
    p = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(workload)
    if not e or e.get("source_hash") != decode_source_hash():
        return None
    return e.get(key)


def profiled_traffic(workload):
    return profiled(workload, "dram_bytes_per_launch")


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- CPU oracle
def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def oracle_sample(wl, seconds_target=12.0, seed=0, threads=None):
    """Time the oracle's decode (unpack + dequantize + exact attention) on a
    bounded sample: one layer, one KV head and its G query heads, over
    contexts of 8K tokens, repeated until ~seconds_target of CPU work.
    threads: BLAS threads (None: as the process has them)."""
    if threads is not None:
        from threadpoolctl import threadpool_limits
        with threadpool_limits(limits=threads):
            r = oracle_sample(wl, seconds_target, seed, None)
        r["cores"] = threads
        return r
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle_pipeline as op  # noqa: F401
    from oracle import alloc, attn, energy, layout, quant

    T = 8192
    G = wl.n_q_heads // wl.n_kv_heads
    kb, vb = synth.keys_values(wl, seed, 0, 0, T)
    k, v = synth.bf16_bits_to_f64(kb), synth.bf16_bits_to_f64(vb)
    E, _ = energy.block_energy(k[:, None, :])
    plan = alloc.make_plan(E[0], wl.bits_k, wl.bits_v, 1, 0, 0)
    kc, kn, _ = quant.quantize_keys(k, plan)
    vc, vn, _ = quant.quantize_values(v, plan)
    rec = layout.pack(kc, vc, kn, vn, plan, T)
    q = synth.bf16_bits_to_f64(synth.queries(wl, seed, 0, 0, T))[:G]
    reps, t0 = 0, time.perf_counter()
    while True:
        kc2, vc2, kn2, vn2 = layout.unpack(rec, plan, T)
        kh = attn.dequant_keys(kc2, kn2, plan)
        vh = attn.dequant_values(vc2, vn2, plan)
        attn.attention(q, kh, vh)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds_target:
            break
    bytes_done = reps * T * BYTES_PER_TOKEN_HEAD(wl.bits_k, wl.bits_v)
    try:
        from threadpoolctl import threadpool_info
        cores = max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:
        cores = 1
    return {"value": bytes_done / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{reps} x (1 layer, 1 KV head + {G} query heads, {T} tokens, "
                      f"K{wl.bits_k}V{wl.bits_v}): unpack + dequantize + exact fp64 attention",
            "seconds": el, "cpu_model": cpu_model(), "host_cpus": os.cpu_count()}


def cpu_baselines(wl, seed):
    """The oracle on all host cores (the line's cpu_baseline) and on one core."""
    allc = oracle_sample(wl, seconds_target=8.0, seed=seed)
    one = oracle_sample(wl, seconds_target=8.0, seed=seed, threads=1)
    allc["one_core"] = {k: one[k] for k in ("value", "unit", "cores", "sample", "seconds")}
    return allc


# --------------------------------------------------------------- main paths
def run_reference(args, wl, rank, world):
    if rank != 0:
        return
    steps, warmup = args.steps, args.warmup
    times = []
    per = max(1.0, min(10.0, 120.0 / max(1, steps + warmup)))
    for i in range(warmup + steps):
        r = oracle_sample(wl, seconds_target=per, seed=args.seed)
        if i >= warmup:
            times.append(r)
    val = statistics.mean(r["value"] for r in times)
    line = {
        "impl": "reference", "metric": f"packed K{wl.bits_k}V{wl.bits_v} decode-attn HBM GB/s",
        "value": val, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": wl.name, "layers": wl.n_layers, "q_heads": wl.n_q_heads,
                   "kv_heads": wl.n_kv_heads, "context": wl.context, "batch": wl.batch,
                   "budget": f"K{wl.bits_k}V{wl.bits_v}"},
        "cpu_baseline": {"value": val, "unit": "GB/s", "cores": times[0]["cores"],
                         "kind": "oracle", "sample": times[0]["sample"]},
        "e2e": {"value": val, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)


def build_stack(args, wl, T, n_layers, cfg, cap, rank, dev, dense, paged=0):
    """Per layer: energies + greedy (or uniform) plans from the layer's own
    keys and the bulk quantize-append of its T tokens (timed with events);
    optionally the same keys / values as a bf16 cache for the comparator
    ([batch][n_kv][cap][128] per layer). Returns the layers, the dense
    caches, the seconds of plan building and of quantize-append."""
    import torch

    from bit_kv_cache_19_b200.runtime import PackedLayer, PagedLayer

    B = wl.batch
    layers, dense_k, dense_v = [], [], []
    t_alloc = t_quant = 0.0
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for li in range(n_layers):
        if paged:
            per_seq = -(-cap // (32 * paged))
            L = PagedLayer(cfg, B, B * per_seq, paged, per_seq, device=dev, layer=li)
            order = [int(x) for x in np.random.default_rng(li).permutation(B * per_seq)]
            for b in range(B):
                L.reserve(b, cap, order=order)
        else:
            L = PackedLayer(cfg, B, cap, device=dev, layer=li)
        ks, vs = [], []
        for b in range(B):
            k, v = synth.keys_values_torch(wl, rank_seed(args.seed, rank, b), li, T, dev)
            ks.append(k)
            vs.append(v)
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        L.alloc_bits(ks[0])
        t_alloc += time.perf_counter() - t0
        kall = torch.stack(ks)
        vall = torch.stack(vs)
        del ks, vs
        if dense:
            dk = torch.zeros(B, wl.n_kv_heads, cap, 128, dtype=torch.bfloat16, device=dev)
            dv = torch.zeros_like(dk)
            dk[:, :, :T].copy_(kall.permute(0, 2, 1, 3))
            dv[:, :, :T].copy_(vall.permute(0, 2, 1, 3))
            dense_k.append(dk)
            dense_v.append(dv)
        ev0.record()
        L.append(kall, vall)
        ev1.record()
        torch.cuda.synchronize()
        t_quant += ev0.elapsed_time(ev1) / 1e3
        assert L.flags() == 0, f"layer {li}: status flags {L.flags()}"
        del kall, vall
        layers.append(L)
    torch.cuda.empty_cache()
    return layers, dense_k, dense_v, t_alloc, t_quant


def step_buffers(wl, n_layers, n_step, T, seed, dev):
    """The step's inputs (q, new k, new v of every layer) in one device
    buffer and its outputs in another, so that an end-to-end step moves them
    with one host-to-device and one device-to-host copy."""
    import torch

    B = wl.batch
    nq_el, nkv_el = B * wl.n_q_heads * 128, B * n_step * wl.n_kv_heads * 128
    per_layer = nq_el + 2 * nkv_el
    step_in = torch.empty(n_layers * per_layer, dtype=torch.bfloat16, device=dev)
    step_out = torch.empty(n_layers, B, wl.n_q_heads, 128, dtype=torch.float32, device=dev)
    qs, knew, vnew = [], [], []
    for li in range(n_layers):
        base = li * per_layer
        q = step_in[base:base + nq_el].view(B, wl.n_q_heads, 128)
        k = step_in[base + nq_el:base + nq_el + nkv_el].view(B, n_step, wl.n_kv_heads, 128)
        v = step_in[base + nq_el + nkv_el:base + per_layer].view(B, n_step, wl.n_kv_heads, 128)
        q.copy_(synth.queries_torch(wl, seed, li, B, T, dev))
        k.copy_(torch.randn(B, n_step, wl.n_kv_heads, 128, device=dev).to(torch.bfloat16))
        v.copy_(torch.randn(B, n_step, wl.n_kv_heads, 128, device=dev).to(torch.bfloat16))
        qs.append(q)
        knew.append(k)
        vnew.append(v)
    return step_in, step_out, qs, knew, vnew


def time_replays(run, stream, steps, flush):
    """Mean ms of `steps` runs on `stream`: two events around all of them, or,
    with an L2 flush buffer, events around each run after its flush."""
    import torch

    if flush is None:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            run()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b_ in evs:
        flush.add_(1)
        a.record(stream)
        run()
        b_.record(stream)
    stream.synchronize()
    return sum(a.elapsed_time(b_) for a, b_ in evs) / steps


def per_step_ms(run, stream, n, flush, reset=None, every=0):
    """Per-run ms of n runs, events around each (after the flush, if any);
    reset() (outside the events) before every `every` runs."""
    import torch

    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(n)]
    for i, (a, b_) in enumerate(evs):
        if reset is not None and every and i % every == 0:
            reset()
        if flush is not None:
            flush.add_(1)
        a.record(stream)
        run()
        b_.record(stream)
    stream.synchronize()
    return [a.elapsed_time(b_) for a, b_ in evs]


def percentiles(xs):
    ys = sorted(xs)

    def q(f):
        return ys[min(len(ys) - 1, int(round(f * (len(ys) - 1))))]
    return {"n": len(ys), "mean": statistics.mean(ys), "p10": q(0.1), "p50": q(0.5),
            "p90": q(0.9), "min": ys[0], "max": ys[-1]}


def fused_step_fn(kvq, args, cfg, layers, knew, vnew, qs, outs, ws, cap):
    def step():
        # one launch per layer: quantize-append the new token(s), then decode
        for li, L in enumerate(layers):
            if args.paged:
                kvq.paged_append_decode(cfg, L.plan_ptrs, knew[li], vnew[li], L.pages, L.lens,
                                        cap, qs[li], outs[li], ws, L.status, kvq.STEP_EARLY)
            else:
                kvq.append_decode(cfg, L.plan_ptrs, knew[li], vnew[li], L.cache_ptrs, L.lens,
                                  cap, cap, qs[li], outs[li], ws, L.status, kvq.STEP_EARLY)
    return step


def run_kvq(args, wl, rank, world, dist):
    import torch

    from bit_kv_cache_19_b200 import kvq

    dev = torch.device("cuda", torch.cuda.current_device())
    n_layers, B, T = args.layers or wl.n_layers, wl.batch, args.context or wl.context
    steps, warmup = args.steps, args.warmup
    n_step = max(1, wl.n_new)  # tokens appended per sequence and layer in a step
    n_dist = args.dist_steps
    n_dist_max = max(n_dist, 4000)
    cap = T + (steps + warmup + max(3, steps // 2) + 4) * n_step + 64
    mode = kvq.ALLOC_UNIFORM if args.alloc == "uniform" else kvq.ALLOC_GREEDY
    if args.rotate_keys:
        mode |= kvq.ALLOC_ROTATE_KEYS
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=1234, alloc_mode=mode)
    bpth = BYTES_PER_TOKEN_HEAD(wl.bits_k, wl.bits_v)

    # ---- prefill: energies + greedy plans, bulk quantize-append (timed)
    layers, dense_k, dense_v, t_alloc, t_quant = build_stack(
        args, wl, T, n_layers, cfg, cap, rank, dev, dense=not args.no_bf16, paged=args.paged)

    # ---- decode inputs (device resident) and static new-token buffers
    step_in, step_out, qs, knew, vnew = step_buffers(wl, n_layers, n_step, T, args.seed, dev)
    outs = [step_out[li] for li in range(n_layers)]
    ws = layers[0].workspace(wl.n_q_heads, cap)
    step = fused_step_fn(kvq, args, cfg, layers, knew, vnew, qs, outs, ws, cap)

    stream = torch.cuda.Stream(device=dev)
    graph = None
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        if not args.no_graph:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()

        def run():
            graph.replay() if graph is not None else step()

        len_before = int(layers[0].lens[0].item())
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        stack_bytes = n_layers * B * wl.n_kv_heads * bpth * T
        flush = (torch.zeros(2 * l2 // 4, dtype=torch.int32, device=dev)
                 if stack_bytes < 4 * l2 else None)
        sampler = ClockSampler(dev.index)
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        sampler.start()
        time.sleep(0.3)
        ms = time_replays(run, stream, steps, flush)
        torch.cuda.synchronize()
        # the step-time distribution: >= 100 replays and >= 2 s (at most
        # 4000), one by one (events between replays), inside the same clock
        # record; every `steps` replays the lengths go back to where the
        # timed region started, so the same lengths are replayed
        n_d = n_dist or min(n_dist_max, max(100, int(2000.0 / max(ms, 1e-3)) + 1))
        lens_end = [L.lens.clone() for L in layers]
        lens_start = [l1 - steps * n_step for l1 in lens_end]

        def reset_lens():
            for L, l0 in zip(layers, lens_start):
                L.lens.copy_(l0)
        dist_ms = per_step_ms(run, stream, n_d, flush, reset_lens, steps)
        for L, l1 in zip(layers, lens_end):  # where the timed region ended
            L.lens.copy_(l1)
        torch.cuda.synchronize()
        clocks = sampler.stop()
    ms = rank_max(ms, dist, dev)
    # packed bytes read per step: length grows by n_step per step
    lens_timed = [len_before + (i + 1) * n_step for i in range(steps)]
    bytes_step = n_layers * B * wl.n_kv_heads * bpth * statistics.mean(lens_timed)
    flags = 0
    for L in layers:
        flags |= L.flags()
    assert flags == 0, f"status flags {flags}"
    value = job_rate(bytes_step, world, ms) / 1e9
    stats = percentiles(dist_ms)
    stats["unit"] = "ms per step"
    stats["note"] = ("the step replayed one by one after the timed region (events around each, "
                     "same clock record); the line's ms_per_step is the timed region's mean")

    # ---- bf16 comparator: the same decode over the unquantized caches (one
    #      dense launch per layer, lengths as in the packed step, graph)
    peak, peak_kind = measured_peaks()
    bf16 = None
    fa2 = None
    if not args.no_bf16:
        dlen = torch.full((B,), int(layers[0].lens[0].item()), dtype=torch.int32, device=dev)
        dws = torch.zeros(kvq.bf16_decode_workspace_bytes(B, wl.n_kv_heads, wl.n_q_heads, cap),
                          dtype=torch.uint8, device=dev)
        dstatus = torch.zeros(1, dtype=torch.int32, device=dev)
        dout = torch.empty(n_layers, B, wl.n_q_heads, 128, dtype=torch.float32, device=dev)

        def dense_step():
            for li in range(n_layers):
                kvq.bf16_decode_attn(dense_k[li], dense_v[li], dlen, cap, qs[li], dout[li], dws,
                                     dstatus)

        with torch.cuda.stream(stream):
            for _ in range(warmup):
                dense_step()
            stream.synchronize()
            if dist is not None:
                dist.barrier()
            dgraph = None
            if not args.no_graph:
                dgraph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(dgraph, stream=stream):
                    dense_step()
            dms = time_replays(lambda: dgraph.replay() if dgraph is not None else dense_step(),
                               stream, steps, None)
        dms = rank_max(dms, dist, dev)
        assert int(dstatus.item()) == 0, "bf16 comparator status"
        dbytes = n_layers * B * wl.n_kv_heads * 512 * int(dlen[0].item())
        dense_floor_ms = dbytes / (peak * 1e9) * 1e3
        bf16 = {"kernel": "dense_decode_kernel (kvq_bf16_decode_attn, one launch per layer)",
                "ms_per_step": dms, "value": job_rate(dbytes, world, dms) / 1e9, "unit": "GB/s",
                "frac": dbytes / (dms / 1e3) / 1e9 / peak,
                "bytes_per_step": dbytes, "cache_bytes": "512 B per token-head (bf16 K + V)",
                "packed_step_speedup": dms / ms,
                "dense_step_at_copy_bw_ms": dense_floor_ms,
                "packed_step_speedup_vs_dense_at_copy_bw": dense_floor_ms / ms,
                "note": "decode only (no append); dense_step_at_copy_bw_ms = the bf16 cache "
                        "bytes at the measured copy bandwidth, the time any dense decode of "
                        "this step needs at least"}
        fa2 = fa2_comparator(dense_k, dense_v, dlen, cap, qs, n_layers, stream, steps, warmup,
                             ms, peak, dist, dev, world, dout)
        del dense_k, dense_v
        torch.cuda.empty_cache()

    # ---- decode kernel alone: events around each layer's decode call
    per_launch = []
    with torch.cuda.stream(stream):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n_layers * 3)]
        for r in range(3):
            for li, L in enumerate(layers):
                a, b = evs[r * n_layers + li]
                a.record(stream)
                if args.paged:
                    kvq.paged_decode_attn(cfg, L.plan_ptrs, L.pages, L.lens, cap, qs[li],
                                          outs[li], ws, L.status)
                else:
                    kvq.decode_attn(cfg, L.plan_ptrs, L.cache_ptrs, L.lens, cap, qs[li],
                                    outs[li], ws, L.status)
                b.record(stream)
        stream.synchronize()
        per_launch = [a.elapsed_time(b) for a, b in evs[n_layers:]]  # skip first pass
    iso_launch_ms = statistics.mean(per_launch)
    # decode_kernel is the only kernel of the step: its average launch
    # duration inside the timed region is the step time over the launches
    # (consecutive launches overlap by their prologue and merge tail)
    launch_ms = ms / n_layers
    bytes_launch = bytes_step / n_layers
    achieved = bytes_launch / (launch_ms / 1e3) / 1e9

    # ---- e2e: host buffers, H2D of the step's inputs and D2H of its outputs
    in_host = step_in.cpu().pin_memory()
    out_host = torch.empty_like(step_out, device="cpu").pin_memory()
    h2d = in_host.numel() * in_host.element_size()
    d2h = out_host.numel() * out_host.element_size()
    with torch.cuda.stream(stream):
        def e2e_step():
            step_in.copy_(in_host, non_blocking=True)
            graph.replay() if graph is not None else step()
            out_host.copy_(step_out, non_blocking=True)
        for _ in range(2):
            e2e_step()
        stream.synchronize()
        if dist is not None:
            dist.barrier()
        e2e_steps = max(3, steps // 2)
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        f1.record(stream)
        f1.synchronize()
        e2e_ms = f0.elapsed_time(f1) / e2e_steps
    e2e_len = int(layers[0].lens[0].item())
    e2e_bytes = n_layers * B * wl.n_kv_heads * bpth * (e2e_len - n_step * (e2e_steps - 1) / 2)
    e2e_ms = rank_max(e2e_ms, dist, dev)
    e2e_val = job_rate(e2e_bytes, world, e2e_ms) / 1e9
    graph = None
    del layers, step_in, step_out, qs, knew, vnew, outs, ws
    torch.cuda.empty_cache()

    # ---- the other workloads (1 GPU, default workload only)
    extras = None
    if world == 1 and not args.no_extras and wl.name == "qwen3b_128k" and not args.layers \
            and not args.context and not args.paged and args.alloc == "greedy" \
            and not args.rotate_keys:
        extras = run_extras(args, rank, dev, stream, peak)

    if rank != 0:
        return
    cpu = (cpu_baselines(wl, seed=args.seed)
           if world == 1 and not args.no_cpu_baseline else None)
    n_tok_quant = n_layers * B * T
    line = {
        "metric": f"packed K{wl.bits_k}V{wl.bits_v} decode-attn HBM GB/s",
        "value": value, "unit": "GB/s", "n_gpus": world, "steps": steps, "warmup": warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 mma, f32 accumulate (codes u8/u32)", "data": "synthetic",
        "config": {"workload": wl.name, "layers": n_layers, "q_heads": wl.n_q_heads,
                   "kv_heads": wl.n_kv_heads, "head_dim": 128, "context": T, "batch": B,
                   "budget": f"K{wl.bits_k}V{wl.bits_v}",
                   "alloc": ("Block-GTQ greedy" if args.alloc == "greedy" else "uniform")
                            + (", width-group key rotation" if args.rotate_keys else ""),
                   "appended_per_step": n_step,
                   "cache": (f"paged: {args.paged} tiles ({32 * args.paged} tokens) per page, "
                             "pages in shuffled order" if args.paged
                             else "one contiguous cache per sequence"),
                   "step": f"per layer, one fused launch: quantize-append {n_step} token(s) "
                           "per sequence + packed decode attention",
                   "l2": (f"inputs larger than L2 ({n_layers}-layer packed cache "
                          f"{stack_bytes / 1e6:.0f} MB, each layer read once per step)"
                          if flush is None else
                          f"L2 flushed before each timed step ({n_layers}-layer packed cache "
                          f"{stack_bytes / 1e6:.0f} MB < 4x L2)"),
                   "graph": not args.no_graph},
        "pct_of_8TBs": value / 8000.0 * 100,
        "tokens_per_s": job_rate(B, world, ms),
        "step_ms": stats,
        "quantize_prefill": {"layer_tokens_per_s": n_tok_quant / t_quant,
                             "token_heads_per_s": n_tok_quant * wl.n_kv_heads / t_quant,
                             "seconds": t_quant, "alloc_bits_seconds": t_alloc},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "traffic": profiled_traffic(wl.name),
                     "kernel": "decode_kernel (kvq_append_decode, one launch per layer)",
                     "bytes_per_launch": bytes_launch, "launch_us": launch_ms * 1e3,
                     "launch_timing": "timed region / launches in it",
                     "isolated_launch_us": iso_launch_ms * 1e3},
        "issue_roofline": issue_roofline(wl.name, launch_ms, clocks),
        "cpu_baseline": cpu,
        "e2e": {"value": e2e_val, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "bf16_comparator": bf16,
        "flash_attn_comparator": fa2,
        "workloads": extras,
        "gpu_launches": steps * n_layers,
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def fa2_comparator(dense_k, dense_v, dlen, cap, qs, n_layers, stream, steps, warmup, packed_ms,
                   peak, dist, dev, world, ref_out):
    """The pages' own yardstick: FlashAttention-2 decode (flash_attn's
    flash_attn_with_kvcache, library code) over the same unquantized caches,
    bf16 (the pages name fp16; same bytes), one call per layer, graph-captured.
    Its caches are [batch][cap][n_kv][128] copies of the comparator's. Returns
    None if flash_attn is not importable, or an "unavailable" record if its
    kernels do not run here."""
    import torch

    try:
        from flash_attn import flash_attn_with_kvcache
        import flash_attn
    except Exception:
        return None
    try:
        kf = [k.permute(0, 2, 1, 3).contiguous() for k in dense_k]
        vf = [v.permute(0, 2, 1, 3).contiguous() for v in dense_v]
        B, n_q = qs[0].shape[0], qs[0].shape[1]
        fout = [None] * n_layers

        def step():
            for li in range(n_layers):
                fout[li] = flash_attn_with_kvcache(qs[li].view(B, 1, n_q, 128), kf[li], vf[li],
                                                   cache_seqlens=dlen,
                                                   softmax_scale=128 ** -0.5)
        with torch.cuda.stream(stream):
            for _ in range(warmup):
                step()
            stream.synchronize()
            if dist is not None:
                dist.barrier()
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph, stream=stream):
                step()
            fms = time_replays(graph.replay, stream, steps, None)
            stream.synchronize()
        fms = rank_max(fms, dist, dev)
        # agreement with the bf16 comparator's output of the last layer
        a = fout[n_layers - 1].float().view(B, n_q, 128)
        b = ref_out[n_layers - 1]
        rel = float(((a - b).abs().amax() / b.abs().amax()).item())
        fbytes = n_layers * B * kf[0].shape[2] * 512 * int(dlen[0].item())
        del kf, vf, graph
        torch.cuda.empty_cache()
        return {"kernel": f"flash_attn {flash_attn.__version__} flash_attn_with_kvcache (library)",
                "ms_per_step": fms, "value": job_rate(fbytes, world, fms) / 1e9, "unit": "GB/s",
                "frac": fbytes / (fms / 1e3) / 1e9 / peak, "bytes_per_step": fbytes,
                "packed_step_speedup": fms / packed_ms,
                "max_rel_diff_vs_bf16_comparator": rel,
                "note": "bf16 K/V caches (the pages compare against fp16 FlashAttention-2 at "
                        "128K); decode only, one call per layer, graph-captured"}
    except Exception as e:  # e.g. no kernel image for this GPU
        torch.cuda.synchronize()
        return {"unavailable": str(e).splitlines()[0][:200]}


def measure_point(args, wl, T, alloc, n_layers, rank, dev, stream, peak, steps):
    """One workload point: build its stack (plans from its own keys, bulk
    quantize-append, timed), then time `steps` graph replays of its fused
    step (append n_new + decode per layer; L2 flushed before each step when
    the stack is within 4x L2). Returns the point's numbers."""
    import torch

    from bit_kv_cache_19_b200 import kvq

    B = wl.batch
    n_step = max(1, wl.n_new)
    warmup = 3
    cap = T + (steps + warmup + 2) * n_step + 64
    mode = kvq.ALLOC_UNIFORM if alloc == "uniform" else kvq.ALLOC_GREEDY
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=1234, alloc_mode=mode)
    bpth = BYTES_PER_TOKEN_HEAD(wl.bits_k, wl.bits_v)
    layers, _, _, _, t_quant = build_stack(args, wl, T, n_layers, cfg, cap, rank, dev, False)
    _, _, qs, knew, vnew = step_buffers(wl, n_layers, n_step, T, args.seed, dev)
    outs = [torch.empty(B, wl.n_q_heads, 128, dtype=torch.float32, device=dev)
            for _ in range(n_layers)]
    ws = layers[0].workspace(wl.n_q_heads, cap)

    class _A:
        paged = 0
    step = fused_step_fn(kvq, _A, cfg, layers, knew, vnew, qs, outs, ws, cap)
    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        len_before = int(layers[0].lens[0].item())
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        stack_bytes = n_layers * B * wl.n_kv_heads * bpth * T
        flush = (torch.zeros(2 * l2 // 4, dtype=torch.int32, device=dev)
                 if stack_bytes < 4 * l2 else None)
        ms = time_replays(graph.replay, stream, steps, flush)
        torch.cuda.synchronize()
    flags = 0
    for L in layers:
        flags |= L.flags()
    assert flags == 0, f"{wl.name} {T} {alloc}: status flags {flags}"
    mean_len = len_before + n_step * (steps + 1) / 2
    bytes_step = n_layers * B * wl.n_kv_heads * bpth * mean_len
    gbs = bytes_step / (ms / 1e3) / 1e9
    out = {"layers": n_layers, "batch": B, "context": T, "q_heads": wl.n_q_heads,
           "kv_heads": wl.n_kv_heads, "budget": f"K{wl.bits_k}V{wl.bits_v}", "alloc": alloc,
           "appended_per_step": n_step, "steps": steps, "ms_per_step": ms,
           "launch_us": ms / n_layers * 1e3, "GB_per_s": gbs, "frac": gbs / peak,
           "tokens_per_s": B / (ms / 1e3),
           "l2": ("stack larger than 4x L2" if flush is None else "L2 flushed before each step"),
           "prefill_seconds": t_quant,
           "prefill_token_heads_per_s": n_layers * B * T * wl.n_kv_heads / t_quant}
    graph = None
    del layers, qs, knew, vnew, outs, ws
    torch.cuda.empty_cache()
    return out


def measure_window(args, wl, T, R, n_layers, rank, dev, stream, peak, steps):
    """The recent-token window on a workload point: per layer a cache whose R
    most recent tokens stay exact (the prefill goes through the window, so
    the oldest T - R tokens are packed), and a step of
    kvq_append_decode_window per layer (one token: one launch that
    quantize-appends the token leaving the window, writes the new one to the
    ring and decodes over the packed and the window tokens); `steps` graph
    replays timed."""
    import torch

    from bit_kv_cache_19_b200 import kvq
    from bit_kv_cache_19_b200.runtime import PackedLayer

    B, n_step, warmup = wl.batch, max(1, wl.n_new), 3
    cap = T + (steps + warmup + 2) * n_step + 64
    cfg = kvq.make_cfg(wl.n_kv_heads, wl.bits_k, wl.bits_v, v_seed=1234)
    bpth = BYTES_PER_TOKEN_HEAD(wl.bits_k, wl.bits_v)
    layers = []
    for li in range(n_layers):
        L = PackedLayer(cfg, B, cap, device=dev, layer=li, window=R)
        ks, vs = zip(*[synth.keys_values_torch(wl, rank_seed(args.seed, rank, b), li, T, dev)
                       for b in range(B)])
        L.alloc_bits(ks[0])
        L.append_window(torch.stack(ks), torch.stack(vs))
        del ks, vs
        layers.append(L)
    torch.cuda.synchronize()
    _, _, qs, knew, vnew = step_buffers(wl, n_layers, n_step, T, args.seed, dev)
    outs = [torch.empty(B, wl.n_q_heads, 128, dtype=torch.float32, device=dev)
            for _ in range(n_layers)]
    ws = torch.zeros(kvq.window_decode_workspace_bytes(cfg, B, wl.n_q_heads, cap),
                     dtype=torch.uint8, device=dev)

    def step():
        for li, L in enumerate(layers):
            L.append_decode_window(knew[li], vnew[li], qs[li], out=outs[li], ws=ws,
                                   step_flags=kvq.STEP_EARLY)

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        stream.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            step()
        len_before = int(layers[0].lens[0].item())
        ms = time_replays(graph.replay, stream, steps, None)
        torch.cuda.synchronize()
    flags = 0
    for L in layers:
        flags |= L.flags()
    assert flags == 0, f"window {T} {R}: status flags {flags}"
    mean_packed = len_before + n_step * (steps + 1) / 2
    packed_bytes = n_layers * B * wl.n_kv_heads * bpth * mean_packed
    ring_bytes = n_layers * B * wl.n_kv_heads * R * 2 * 128 * 4
    out = {"layers": n_layers, "batch": B, "context": T, "window": R,
           "budget": f"K{wl.bits_k}V{wl.bits_v}", "appended_per_step": n_step, "steps": steps,
           "ms_per_step": ms, "GB_per_s": (packed_bytes + ring_bytes) / (ms / 1e3) / 1e9,
           "frac": (packed_bytes + ring_bytes) / (ms / 1e3) / 1e9 / peak,
           "launches_per_layer": 1,
           "note": "bytes = packed tokens read by the decode + the fp32 window ring; the step "
                   "is one kvq_append_decode_window launch per layer"}
    graph = None
    del layers, qs, knew, vnew, outs, ws
    torch.cuda.empty_cache()
    return out


def run_extras(args, rank, dev, stream, peak):
    """The other workloads of the build: one Llama-3.1-8B-shaped layer at 32K
    (K2V2), the 7B-Qwen-shaped serving step (16 x 32K, append 16 + decode,
    28 layers, K3V2), the Qwen2.5-3B-shaped context sweep 8K..512K with
    Block-GTQ (greedy) and uniform plans of the same bytes, the 36-layer
    128K step with a 128-token recent-token window, and the bulk prefill of
    512K tokens x 36 layers (its roofline: bf16 K/V in plus the packed bytes
    out at the measured copy bandwidth)."""
    steps = 20
    out = {}
    W = synth.WORKLOADS
    t0 = time.perf_counter()
    out["llama8b"] = measure_point(args, W["llama8b"], W["llama8b"].context, "greedy", 1, rank,
                                   dev, stream, peak, steps)
    sv = W["qwen7b_serve"]
    out["qwen7b_serve"] = measure_point(args, sv, sv.context, "greedy", sv.n_layers, rank, dev,
                                        stream, peak, steps)
    sw = W["qwen3b_sweep"]
    sweep = []
    for T in sw.contexts:
        for alloc in ("greedy", "uniform"):
            sweep.append(measure_point(args, sw, T, alloc, sw.n_layers, rank, dev, stream, peak,
                                       steps))
    out["qwen3b_sweep"] = sweep
    wq = W["qwen3b_128k"]
    out["qwen3b_128k_window128"] = measure_window(args, wq, wq.context, 128, wq.n_layers, rank,
                                                  dev, stream, peak, steps)
    big = [p for p in sweep if p["context"] == max(sw.contexts) and p["alloc"] == "greedy"][0]
    tok_heads = big["layers"] * big["context"] * sw.n_kv_heads
    moved = tok_heads * (512 + BYTES_PER_TOKEN_HEAD(sw.bits_k, sw.bits_v))
    floor_s = moved / (peak * 1e9)
    out["prefill_512k_x36"] = {"seconds": big["prefill_seconds"],
                               "token_heads_per_s": big["prefill_token_heads_per_s"],
                               "bytes_moved": moved, "roofline_seconds": floor_s,
                               "frac": floor_s / big["prefill_seconds"],
                               "note": "bulk quantize-append, one launch per layer; bytes = "
                                       "bf16 K + V in + packed codes and norms out"}
    out["seconds"] = time.perf_counter() - t0
    return out


def issue_roofline(workload, launch_ms, clocks):
    """The decode kernel against the instruction-issue ceiling (it is bound by
    issue, not by HBM): warp instructions per launch (ncu, same source) over
    the launch time, against 148 SMs x 4 schedulers x 1 warp instruction per
    cycle at the SM clock sampled during the timed region."""
    import torch
    inst = profiled(workload, "warp_inst_per_launch")
    if inst is None or not clocks or not clocks.get("sm_mhz"):
        return None
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    peak = n_sm * 4 * clocks["sm_mhz"] * 1e6 / 1e9
    achieved = inst / (launch_ms * 1e-3) / 1e9
    return {"bound": "issue", "achieved": achieved, "peak": peak, "unit": "G warp-inst/s",
            "frac": achieved / peak, "warp_inst_per_launch": inst,
            "peak_basis": f"{n_sm} SMs x 4 schedulers x 1 inst/cycle x {clocks['sm_mhz']:.0f} MHz"}


def main():
    args = parse()
    wl = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    dist = None
    if args.impl == "reference":
        run_reference(args, wl, rank, world)
        return
    import torch

    if world > 1:
        import torch.distributed as tdist
        from datetime import timedelta

        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        tdist.init_process_group("nccl", timeout=timedelta(seconds=120))
        dist = tdist
    else:
        torch.cuda.set_device(0)
    try:
        run_kvq(args, wl, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
