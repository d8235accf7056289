#!/usr/bin/env python
"""Benchmark of the MoE decode hot path on B200 (one JSON line on rank 0).

Workload (default): the 30-layer stack of the Gemma-like MoE layer (hidden
2816, 128 routed experts, top-8, expert intermediate 704, shared intermediate
2112, 4-bit group-64 experts, int8 router, per-expert router bias N(0, 1.5)),
decoding 256 consecutive tokens at batch 1 with an fp16 residual stream and
RMSNorm between layers; all experts resident in HBM (13.2 GB).  One step is
the decode of all 256 tokens through the 30 layers.  Inputs are synthetic and
seeded; the weights are larger than L2 and each token touches ~1.1 GB.

Multi-GPU: the path does not shard (one decode stream per GPU); --gpus N runs
N independent replicas, timed as the max over ranks.

--impl reference times the CPU oracle on the host cores on a bounded sample
of the same workload (one token-layer per step) and reports the same metric.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE decode tokens/s per layer-stack; achieved HBM GB/s vs B200 peak (1 GPU)"
UNIT = "tokens/s"
N_LAYERS = 30
N_TOKENS = 256
SEED = 0
BIAS_STD = 1.5
REPEATS = 5          # timed runs per step size of the batched sweep (median reported)


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--layers", type=int, default=N_LAYERS)
    p.add_argument("--tokens", type=int, default=N_TOKENS)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=15.0)
    p.add_argument("--batch-sizes", default="1,8,32,64,128,256",
                   help="tokens per step of the batched sweep (comma-separated)")
    p.add_argument("--chunk", type=int, default=128, help="prefill chunk (tokens)")
    p.add_argument("--store-dir", default=tempfile.gettempdir(), help="directory of the expert file")
    p.add_argument("--store-layers", type=int, default=8, help="layers in the expert file")
    p.add_argument("--store-threads", type=int, default=16, help="pread threads")
    p.add_argument("--workload", choices=("stack", "streaming", "batched", "prefill", "storage", "direct"),
                   default="stack",
                   help="stack (default, the headline line), streaming (experts in pinned host "
                        "memory behind the LFU cache), batched (one layer, T tokens per step) or "
                        "prefill (streaming, the prompt in chunks) or storage (misses read "
                        "from an expert file)")
    return p.parse_args()


def env_rank():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def max_over_ranks(value, world, device):
    """The largest value over all ranks (a time: the job ends with its slowest
    rank).  With one rank, the value itself."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(world, tokens_per_rank, ms_max):
    """Whole-job throughput: every rank decodes its own tokens (replicas), the
    job takes as long as its slowest rank."""
    return world * tokens_per_rank / (ms_max / 1000.0)


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def tensor_peak():
    """Dense 16-bit tensor peak in TFLOP/s (burst) and where it comes from;
    fp16 and bf16 share the rate."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index: int):
        import torch
        self.proc = None
        self.tmp = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        sel = str(device_index)
        try:
            pr = torch.cuda.get_device_properties(device_index)
            sel = f"{pr.pci_domain_id:08x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0"
        except Exception:
            pass
        self.cmd = ["nvidia-smi", "-i", sel, f"--query-gpu={self.FIELDS}",
                    "--format=csv,noheader,nounits", "-lms", "200"]

    def start(self):
        try:
            self.proc = subprocess.Popen(self.cmd, stdout=self.tmp, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.tmp.flush()
        rows = []
        with open(self.tmp.name) as f:
            for line in f:
                parts = [v.strip() for v in line.split(",")]
                if len(parts) >= 8:
                    rows.append(parts)
        os.unlink(self.tmp.name)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        reasons = set()
        for r in rows:
            for name, v in zip(self.NAMES, r[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------------ workload ----
def build_stack(device, n_layers):
    from bit_quantized_expert_int8_b200 import synth
    from bit_quantized_expert_int8_b200.config import LAYER
    return [synth.layer_weights(LAYER, SEED, l, device, bias_std=BIAS_STD)
            for l in range(n_layers)]


def kernel_launches_per_token(n_layers):
    # per token: load + store kernels and one fused kernel per layer
    return 2 + n_layers


def run_ours(args):
    import torch
    import torch.distributed as dist

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER

    rank, local_rank, world = env_rank()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=dev)
    moeq4.load()
    cfg = LAYER
    L, T = args.layers, args.tokens
    layers = build_stack(dev, L)
    objs = [moeq4.Layer.from_dict(d) for d in layers]
    h0 = synth.tokens(T, cfg.H, SEED + 1 + rank, dev)
    h = h0.clone()
    y_last = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
    ctx = moeq4.Context(cfg, 1)
    stream = torch.cuda.current_stream()

    def step():
        h.copy_(h0)
        moeq4.moe_stack_decode(ctx, objs, h, T, y_last)

    def barrier():
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    clocks = ClockSampler(local_rank)
    clocks.start()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.profiler.start()          # a profiler started with capture off records this region
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    torch.cuda.profiler.stop()
    clk = clocks.stop()
    ms = e0.elapsed_time(e1) / args.steps
    ms_max = max_over_ranks(ms, world, dev)
    value = job_tokens_per_s(world, T, ms_max)

    # ---- end to end through the C ABI with host buffers
    h_host = h0.cpu().pin_memory()
    h_back = torch.empty_like(h_host).pin_memory()

    def step_e2e():
        h.copy_(h_host, non_blocking=True)
        moeq4.moe_stack_decode(ctx, objs, h, T, y_last)
        h_back.copy_(h, non_blocking=True)

    for _ in range(max(1, args.warmup)):
        step_e2e()
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        step_e2e()
    e1.record(stream)
    barrier()
    ms_e2e = e0.elapsed_time(e1) / args.steps
    e2e_value = job_tokens_per_s(world, T, max_over_ranks(ms_e2e, world, dev))

    moeq4.moe_ctx_check(ctx)
    # ---- dominant kernel: the fused layer kernel of one token-layer
    roof = roofline(ctx, layers, cfg, dev, stream)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(layers, cfg, args.cpu_seconds, h0)
    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "q4 x fixed16 -> i32 (DP4A), f32 epilogue", "data": "synthetic (seeded; N(0,0.02) weights quantised to "
                                     "4-bit group-64 and int8 router; N(0,1) fp16 tokens)",
            "config": {"workload": f"stack{L}x{T}: {L}-layer MoE stack, {T} tokens decoded "
                                   "one after another at batch 1",
                       "hidden": cfg.H, "experts": cfg.E, "top_k": cfg.k,
                       "inter": cfg.I, "inter_shared": cfg.Is, "group": 64,
                       "router_bias_std": BIAS_STD, "tokens_per_step": T, "layers": L,
                       "parallelism": f"replicas{world}",
                       "l2": "inputs larger than L2 (13.2 GB resident weights; "
                             "~1.1 GB touched per token)"},
            "e2e": {"value": round(e2e_value, 3), "unit": UNIT,
                    "h2d_bytes_per_step": T * cfg.H * 2, "d2h_bytes_per_step": T * cfg.H * 2},
            "gpu_launches": kernel_launches_per_token(L) * T * args.steps,
            "roofline": roof,
            "clocks": clk,
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    ctx.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# DRAM bytes (read + write) of one launch of the fused layer kernel, from an
# ncu capture of the kernel built from the source with this SHA-256; any other
# source reports null (the counters describe a different kernel).
KERNEL_SRC = os.path.join(ROOT, "bit_quantized_expert_int8_b200", "csrc", "layer_fused.cuh")
TRAFFIC_BY_SOURCE = {
    # ncu --set full, one launch of the bench layers (hidden 2816, top-8),
    # 16-bit x digits: dram__bytes_read.sum 37,284,864 + write 43,008
    "ab523b1bf6c48f302f20a8d0fa33bdea867f6816a4e0a6fbc4a69b12422ad079": 37327872,
    # the same capture with 24-bit x digits: read 37,290,496 + write 114,432
    "c31f5378bd41ff1c3afc7da62ad3dfbbf79f3cba4022471fda56907f7fdcafba": 37404928,
    # status word read only by waits longer than 20 us: read 37,290,240 + write 140,544
    "315e1cae13a9292cedfd34824b3dfbd1020a3c725007f273bb51283915d59fcb": 37430784,
    # pre-norm with the down items' residual rows loaded beside x: read 37,289,984 + write 34,048
    "48bcc63c17dd9b2c08b20c7ddc1217797a982fe5d4bfbf3c4657e479a352f572": 37324032,
}


def kernel_traffic():
    import hashlib
    with open(KERNEL_SRC, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    return TRAFFIC_BY_SOURCE.get(digest), digest


def roofline(ctx, layers, cfg, dev, stream):
    """Average duration of the dominant kernel, the fused single-token layer
    kernel (router + shared and 8 routed expert FFNs + combine), over graph
    replays of one launch per layer of the stack, so no weight is
    L2-resident between its uses; algorithmic bytes = the router plus the 9
    experts' blobs the token reads."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    hbm, kind = peaks()
    n = len(layers)
    reps = 20
    # a distinct token for every launch of the graph, so no launch can profit
    # from the routing (or the weights) of an earlier replay
    xs = synth.tokens(n * reps, cfg.H, SEED + 77, dev)
    y = torch.empty((1, cfg.H), dtype=torch.float32, device=dev)
    objs = [moeq4.Layer.from_dict(d) for d in layers]
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for i, o in enumerate(objs):                          # warm up
            moeq4.moe_layer_decode(ctx, o, xs[i:i + 1], 1, y, stream=side)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for r in range(reps):
                for i, o in enumerate(objs):
                    j = r * n + i
                    moeq4.moe_layer_decode(ctx, o, xs[j:j + 1], 1, y, stream=side)
        for _ in range(2):
            g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(side)
        g.replay()
        e1.record(side)
    torch.cuda.synchronize()
    moeq4.moe_ctx_check(ctx)
    us = e0.elapsed_time(e1) * 1000.0 / (reps * n)
    algo = (cfg.k * synth.blob_bytes(cfg.H, cfg.I) + synth.blob_bytes(cfg.H, cfg.Is)
            + cfg.E * cfg.H + 2 * cfg.E)
    achieved = algo / (us * 1e-6) / 1e9
    return {"bound": "hbm", "kernel": "k_moe_layer_fused (one token, one layer)",
            "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "peak_kind": f"{kind} (hbm_gbs)",
            "algorithmic_bytes_per_launch": algo, "us_per_launch": round(us, 3),
            "traffic": kernel_traffic()[0]}


def cpu_baseline(layers, cfg, seconds, h0=None, n_sample_layers=2):
    """The CPU oracle as it stands on the host cores: full MoE layers of this
    workload, one token at a time, for about `seconds`; tokens/s of the whole
    stack = 1 / (layers * mean seconds per token-layer)."""
    import numpy as np
    import torch

    import oracle
    from bit_quantized_expert_int8_b200 import synth
    cores = oracle.set_threads(0)
    lns = []
    for d in layers[:n_sample_layers]:
        lns.append({k: (None if v is None else
                        (v.cpu().view(torch.int16).numpy().view(np.uint16)
                         if v.dtype == torch.float16 else v.cpu().numpy()))
                    for k, v in d.items()})
    x = synth.tokens(64, cfg.H, SEED + 5, "cpu").view(torch.int16).numpy().view(np.uint16)
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle.moe_layer(cfg, lns[n % len(lns)], x[n % x.shape[0]])
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per = el / n
    return {"value": round(1.0 / (N_LAYERS * per), 5), "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"{n} token-layers of the stack workload (layers 0-{len(lns) - 1}), "
                      f"{per * 1e3:.1f} ms each; tokens/s = 1/({N_LAYERS} x that)"}


def run_reference(args):
    rank, _, world = env_rank()
    if rank != 0:
        return
    import torch

    import oracle
    from bit_quantized_expert_int8_b200.config import LAYER
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    layers = build_stack(dev, 2)
    cfg = LAYER
    per_step = []
    cores = oracle.set_threads(0)
    import numpy as np

    from bit_quantized_expert_int8_b200 import synth
    lns = [{k: (None if v is None else
                (v.cpu().view(torch.int16).numpy().view(np.uint16)
                 if v.dtype == torch.float16 else v.cpu().numpy()))
            for k, v in d.items()} for d in layers]
    x = synth.tokens(64, cfg.H, SEED + 5, "cpu").view(torch.int16).numpy().view(np.uint16)
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        oracle.moe_layer(cfg, lns[i % 2], x[i % 64])
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            per_step.append(dt)
    per = sum(per_step) / len(per_step)
    value = 1.0 / (N_LAYERS * per)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(per * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (same recipe as ours)",
            "config": {"workload": f"stack{args.layers}x{args.tokens} (one token-layer "
                                   "sampled per step)", "hidden": cfg.H, "experts": cfg.E,
                       "top_k": cfg.k, "inter": cfg.I, "inter_shared": cfg.Is},
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": cores,
                             "kind": "oracle",
                             "sample": f"{args.steps} token-layers (layers 0-1), "
                                       f"{per * 1e3:.1f} ms each"},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_streaming(args):
    """Expert streaming: the stack over 512 tokens with every routed expert in
    pinned host memory, a 16-slot LFU cache per layer in HBM (cold at the
    start of each step), misses fetched while the shared expert runs.  Two
    lines: misses copied by host-issued cudaMemcpyAsync after one host wait
    per layer-token, and misses pulled by a device-side gather kernel
    (MOE_DEVICE_FILL, no host wait).  One GPU."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER
    cfg = LAYER
    L, T = args.layers, 512 if args.tokens == N_TOKENS else args.tokens
    dev = torch.device("cuda", 0)
    moeq4.load()
    nb = synth.blob_bytes(cfg.H, cfg.I)
    layers, keep = [], []
    for l in range(L):
        d = synth.layer_weights(cfg, SEED, l, dev, bias_std=BIAS_STD)
        store = torch.empty((cfg.E, nb), dtype=torch.uint8, pin_memory=True)
        store.copy_(d["experts"])
        del d["experts"]
        slots = torch.zeros((cfg.S, nb), dtype=torch.uint8, device=dev)
        table = moeq4.new_lfu_table()
        layers.append(moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"], d["shared"],
                                  None, store, slots, table))
        keep.append((d, store, slots, table))
    torch.cuda.empty_cache()
    ctx = moeq4.Context(cfg, 1)
    copy_stream = torch.cuda.Stream()
    h0 = synth.tokens(T, cfg.H, SEED + 1, dev)
    h = h0.clone()
    y = torch.empty((1, cfg.H), dtype=torch.float32, device=dev)
    # the link itself: one pinned host -> device copy of 1 GiB
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    src = torch.empty(1 << 30, dtype=torch.uint8, pin_memory=True)
    dst = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
    dst.copy_(src, non_blocking=True)
    torch.cuda.synchronize()
    e0.record()
    dst.copy_(src, non_blocking=True)
    e1.record()
    torch.cuda.synchronize()
    link = (1 << 30) / (e0.elapsed_time(e1) * 1e-3) / 1e9
    del src, dst
    for fill in ("host", "device"):
        flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)

        def step():
            for (_, _, _, table) in keep:
                moeq4.moe_lfu_init(ctx, table, cfg.S)
            h.copy_(h0)
            for t in range(T):
                for lay in layers:
                    moeq4.moe_layer_decode(ctx, lay, h[t:t + 1], 1, y, flags=flags,
                                           copy_stream=copy_stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        hits = misses = 0
        times = []
        clocks = ClockSampler(0)
        clocks.start()
        for _ in range(args.steps):
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
            for (_, _, _, table) in keep:
                tb = moeq4.read_lfu_table(table)
                hits += tb.hits
                misses += tb.misses
        clk = clocks.stop()
        moeq4.moe_ctx_check(ctx)
        ms = statistics.median(times)
        h2d = misses / args.steps * nb
        print(json.dumps({
            "metric": METRIC, "workload": f"streaming{L}x{T}", "fill": fill,
            "value": round(T / (ms / 1000.0), 3), "unit": UNIT, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "ms_per_step_min_max": [round(min(times), 3), round(max(times), 3)],
            "timing": f"median of {len(times)} steps", "higher_is_better": True,
            "config": {"layers": L, "tokens": T, "slots": cfg.S, "cache": "cold at each step",
                       "expert_store": "pinned host memory",
                       "fill": "host-issued cudaMemcpyAsync after a host wait per layer-token"
                               if fill == "host" else
                               "device gather kernel from pinned host memory, no host wait"},
            "clocks": clk,
            "hit_rate": round(hits / max(1, hits + misses), 4),
            "h2d_bytes_per_step": int(h2d), "h2d_gbs_over_step": round(h2d / (ms * 1e-3) / 1e9, 2),
            "h2d_link_gbs_measured": round(link, 2)}), flush=True)


def run_prefill(args):
    """Chunked prefill in streaming mode: a 512-token prompt through the 30-layer
    stack in chunks of 128 tokens (chunk-major: each chunk through every layer),
    every routed expert in pinned host memory behind a 16-slot LFU cache per
    layer (cold at the start of each step).  A chunk is one cache lookup and
    one copy per missing expert per unit of tokens whose experts fit the
    slots.  Reports prompt tokens/s, bytes copied per prompt token and the
    hit rate (distinct experts per unit), for host- and device-issued fills."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER
    cfg = LAYER
    L = args.layers
    P = 512 if args.tokens == N_TOKENS else args.tokens
    C = args.chunk
    dev = torch.device("cuda", 0)
    moeq4.load()
    nb = synth.blob_bytes(cfg.H, cfg.I)
    layers, keep = [], []
    for l in range(L):
        d = synth.layer_weights(cfg, SEED, l, dev, bias_std=BIAS_STD)
        store = torch.empty((cfg.E, nb), dtype=torch.uint8, pin_memory=True)
        store.copy_(d["experts"])
        del d["experts"]
        slots = torch.zeros((cfg.S, nb), dtype=torch.uint8, device=dev)
        table = moeq4.new_lfu_table()
        layers.append(moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"], d["shared"],
                                  None, store, slots, table))
        keep.append((d, store, slots, table))
    torch.cuda.empty_cache()
    ctx = moeq4.Context(cfg, C)
    copy_stream = torch.cuda.Stream()
    h0 = synth.tokens(P, cfg.H, SEED + 1, dev)
    h = h0.clone()
    y = torch.empty((C, cfg.H), dtype=torch.float32, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for fill in ("host", "device"):
        flags = moeq4.MOE_PRENORM | (moeq4.MOE_DEVICE_FILL if fill == "device" else 0)

        def step():
            for (_, _, _, table) in keep:
                moeq4.moe_lfu_init(ctx, table, cfg.S)
            h.copy_(h0)
            for c0 in range(0, P, C):
                n = min(C, P - c0)
                for lay in layers:
                    moeq4.moe_layer_decode(ctx, lay, h[c0:c0 + n], n, y[:n], flags=flags,
                                           copy_stream=copy_stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        hits = misses = 0
        times = []
        clocks = ClockSampler(0)
        clocks.start()
        for _ in range(args.steps):
            e0.record()
            step()
            e1.record()
            torch.cuda.synchronize()
            times.append(e0.elapsed_time(e1))
            for (_, _, _, table) in keep:
                tb = moeq4.read_lfu_table(table)
                hits += tb.hits
                misses += tb.misses
        clk = clocks.stop()
        moeq4.moe_ctx_check(ctx)
        ms = statistics.median(times)
        h2d = misses / args.steps * nb
        print(json.dumps({
            "metric": METRIC, "workload": f"prefill{L}x{P}/chunk{C}", "fill": fill,
            "value": round(P / (ms / 1000.0), 3), "unit": "prompt tokens/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 3),
            "ms_per_step_min_max": [round(min(times), 3), round(max(times), 3)],
            "timing": f"median of {len(times)} steps", "higher_is_better": True,
            "config": {"layers": L, "prompt_tokens": P, "chunk": C, "slots": cfg.S,
                       "order": "each chunk through every layer", "cache": "cold at each step",
                       "expert_store": "pinned host memory"},
            "clocks": clk,
            "hit_rate_distinct_experts": round(hits / max(1, hits + misses), 4),
            "copies_per_step": int(misses / args.steps),
            "h2d_bytes_per_step": int(h2d),
            "h2d_bytes_per_prompt_token": int(h2d / P),
            "h2d_gbs_over_step": round(h2d / (ms * 1e-3) / 1e9, 2)}), flush=True)


def _fs_of(path):
    """File system type of the mount holding path (from /proc/mounts)."""
    best, fs = "", "unknown"
    try:
        with open("/proc/mounts") as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and os.path.abspath(path).startswith(parts[1]) and len(parts[1]) > len(best):
                    best, fs = parts[1], parts[2]
    except OSError:
        pass
    return fs


def run_storage(args):
    """The storage tier: the stack's routed experts in an expert file (blobs
    padded to 4 KiB, read with parallel pread, O_DIRECT where the file system
    allows), misses read into pinned staging and copied to the 16 slots per
    layer.  Two lines: decode (tokens one after another) and prefill (the
    prompt in chunks, each chunk through every layer), cold cache each step."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER
    cfg = LAYER
    L = args.store_layers
    dev = torch.device("cuda", 0)
    moeq4.load()
    nb = synth.blob_bytes(cfg.H, cfg.I)
    d_all = [synth.layer_weights(cfg, SEED, l, dev, bias_std=BIAS_STD) for l in range(L)]
    path = os.path.join(args.store_dir, f"moeq4_experts_{os.getpid()}.bin")
    t0 = time.perf_counter()
    moeq4.write_expert_file(path, [d["experts"].cpu() for d in d_all], nb)
    os.sync()
    write_s = time.perf_counter() - t0
    fst = moeq4.Store(path, L, cfg.E, nb, n_threads=args.store_threads, n_staging=cfg.S)
    layers = []
    for l, d in enumerate(d_all):
        del d["experts"]
        slots = torch.zeros((cfg.S, nb), dtype=torch.uint8, device=dev)
        table = moeq4.new_lfu_table()
        layers.append((moeq4.Layer(d["router_w"], d["router_scale"], d["router_bias"], d["shared"],
                                   None, None, slots, table, store=fst, store_layer=l), slots, table))
    torch.cuda.empty_cache()
    C = args.chunk
    ctx = moeq4.Context(cfg, C)
    copy_stream = torch.cuda.Stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    try:
        for mode, P in (("decode", 128), ("prefill", 512)):
            h0 = synth.tokens(P, cfg.H, SEED + 1, dev)
            h = h0.clone()
            y = torch.empty((C, cfg.H), dtype=torch.float32, device=dev)

            def step():
                for (_, _, table) in layers:
                    moeq4.moe_lfu_init(ctx, table, cfg.S)
                h.copy_(h0)
                if mode == "decode":
                    for t in range(P):
                        for (lay, _, _) in layers:
                            moeq4.moe_layer_decode(ctx, lay, h[t:t + 1], 1, y[:1], flags=moeq4.MOE_PRENORM,
                                                   copy_stream=copy_stream)
                else:
                    for c0 in range(0, P, C):
                        n = min(C, P - c0)
                        for (lay, _, _) in layers:
                            moeq4.moe_layer_decode(ctx, lay, h[c0:c0 + n], n, y[:n], flags=moeq4.MOE_PRENORM,
                                                   copy_stream=copy_stream)

            for _ in range(args.warmup):
                step()
            torch.cuda.synchronize()
            b0, s0, direct = fst.stats()
            misses = 0
            times = []
            clocks = ClockSampler(0)
            clocks.start()
            for _ in range(args.steps):
                e0.record()
                step()
                e1.record()
                torch.cuda.synchronize()
                times.append(e0.elapsed_time(e1))
                misses += sum(moeq4.read_lfu_table(t).misses for (_, _, t) in layers)
            clk = clocks.stop()
            moeq4.moe_ctx_check(ctx)
            b1, s1, direct = fst.stats()
            ms = statistics.median(times)
            print(json.dumps({
                "metric": METRIC, "workload": f"storage-{mode}{L}x{P}", "value": round(P / (ms / 1000.0), 3),
                "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": round(ms, 3), "ms_per_step_min_max": [round(min(times), 3), round(max(times), 3)],
                "timing": f"median of {len(times)} steps", "higher_is_better": True,
                "config": {"layers": L, "tokens": P, "chunk": C if mode == "prefill" else 1, "slots": cfg.S,
                           "expert_store": "file", "file_system": _fs_of(path), "o_direct": bool(direct),
                           "reader_threads": args.store_threads, "cache": "cold at each step",
                           "file_bytes": os.path.getsize(path), "file_write_s": round(write_s, 2)},
                "clocks": clk,
                "copies_per_step": int(misses / args.steps),
                "read_bytes_per_step": int((b1 - b0) / args.steps),
                "read_gbs_while_reading": round((b1 - b0) / max(1e-9, s1 - s0) / 1e9, 2),
                "read_gbs_over_step": round((b1 - b0) / args.steps / (ms * 1e-3) / 1e9, 2),
                "read_bytes_per_token": int((b1 - b0) / args.steps / P)}), flush=True)
    finally:
        fst.close()
        os.unlink(path)


def bucket_split(counts, T, min_tokens=1, min_step=2):
    """Experts of one step by the kernel that serves them: `counts` holds the
    pairs routed to each expert.  In steps of at least `min_step` tokens a
    bucket of `min_tokens` or more pairs runs on tcgen05; every other used
    expert on the CUDA-core grouped kernels.  Returns (tcgen05, grouped)."""
    used = [c for c in counts if c > 0]
    if T < min_step or min_tokens <= 0:
        return 0, len(used)
    tc = sum(1 for c in used if c >= min_tokens)
    return tc, len(used) - tc


def run_batched(args):
    """Batched decode: one layer of the stack configuration (no router bias,
    independent routings) at T tokens per step; 8 weight copies rotated so the
    experts a step touches are not L2-resident from the step before."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER
    cfg = LAYER
    dev = torch.device("cuda", 0)
    moeq4.load()
    hbm, kind = peaks()
    tpk, tkind = tensor_peak()
    copies = [synth.layer_weights(cfg, SEED, l, dev) for l in range(8)]
    objs = [moeq4.Layer.from_dict(d) for d in copies]
    nb, nbs = synth.blob_bytes(cfg.H, cfg.I), synth.blob_bytes(cfg.H, cfg.Is)
    sizes = [int(v) for v in args.batch_sizes.split(",")]
    ctx = moeq4.Context(cfg, max(sizes))
    lines = []
    clocks = ClockSampler(0)
    clocks.start()
    for T in sizes:
        x = synth.tokens(T, cfg.H, SEED + 3, dev)
        y = torch.empty((T, cfg.H), dtype=torch.float32, device=dev)
        idx = torch.empty((T, cfg.k), dtype=torch.int32, device=dev)
        touched = 0
        n_tc = n_grp = 0
        for o in objs:
            moeq4.moe_layer_decode(ctx, o, x, T, y, idx)
            touched += torch.unique(idx).numel()
            if T > 1:
                counts = torch.bincount(idx.flatten().long(), minlength=cfg.E).tolist()
                a, b = bucket_split(counts, T)
                n_tc += a
                n_grp += b
        touched /= len(objs)
        reps = max(8, min(400, int(4000 / T)))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        runs = []
        for _ in range(REPEATS):
            torch.cuda.synchronize()
            e0.record()
            for r in range(reps):
                moeq4.moe_layer_decode(ctx, objs[r % len(objs)], x, T, y)
            e1.record()
            torch.cuda.synchronize()
            runs.append(e0.elapsed_time(e1) * 1000.0 / reps)
        us = statistics.median(runs)
        algo = touched * nb + nbs + cfg.E * cfg.H + 2 * cfg.E
        # useful multiply-adds of the FFNs: gate, up and down of k routed and the shared expert
        flop = 2.0 * T * 3 * cfg.H * (cfg.k * cfg.I + cfg.Is)
        if T == 1:
            path = "fused single-token kernel"
        else:
            path = "tcgen05 kernels (shared expert and every routed bucket, one persistent launch per FFN half)"
        lines.append({"tokens": T, "us_per_step": round(us, 2),
                      "us_min_max": [round(min(runs), 2), round(max(runs), 2)],
                      "tokens_per_s": round(T / (us * 1e-6), 1),
                      "distinct_experts": round(touched, 1), "algorithmic_bytes": int(algo),
                      "achieved_gbs": round(algo / (us * 1e-6) / 1e9, 1),
                      "frac_of_hbm": round(algo / (us * 1e-6) / 1e9 / hbm, 4),
                      "ffn_tflops": round(flop / (us * 1e-6) / 1e12, 2),
                      "frac_of_tensor": round(flop / (us * 1e-6) / 1e12 / tpk, 4),
                      # max(bytes / HBM peak, flops / tensor peak) over the measured time
                      "frac_of_roofline": round(max(algo / (hbm * 1e9), flop / (tpk * 1e12)) /
                                                (us * 1e-6), 4),
                      "experts_tcgen05": round(n_tc / len(objs), 1),
                      "experts_grouped": round(n_grp / len(objs), 1),
                      "path": path})
    clk = clocks.stop()
    moeq4.moe_ctx_check(ctx)
    print(json.dumps({"metric": METRIC, "workload": "batched sweep, one layer", "unit": UNIT,
                      "timing": f"median of {REPEATS} runs of each step size", "clocks": clk,
                      "peak_gbs": hbm, "peak_kind": kind, "tensor_peak_tflops": tpk,
                      "tensor_peak_kind": tkind, "mma_min_tokens": 1, "sweep": lines}), flush=True)


def run_direct(args):
    """The granular expert-FFN entry point (moe_expert_ffn_q4, direct
    per-pair kernels) on one token's pairs of the stack configuration: the
    shared expert and 8 routed experts, each blob read once per call; 8
    weight copies rotated so no call finds its blobs in L2."""
    import torch

    from bit_quantized_expert_int8_b200 import moeq4, synth
    from bit_quantized_expert_int8_b200.config import LAYER
    cfg = LAYER
    dev = torch.device("cuda", 0)
    moeq4.load()
    hbm, kind = peaks()
    copies = [synth.layer_weights(cfg, SEED, l, dev) for l in range(8)]
    nb, nbs = synth.blob_bytes(cfg.H, cfg.I), synth.blob_bytes(cfg.H, cfg.Is)
    ctx = moeq4.Context(cfg, 1)
    x = synth.tokens(1, cfg.H, SEED + 3, dev)
    y = torch.empty((cfg.k + 1, cfg.H), dtype=torch.float32, device=dev)
    pair_sets = []
    for d in copies:
        base = d["experts"].data_ptr()
        ent = [(d["shared"].data_ptr(), cfg.Is, 0)]
        ent += [(base + e * 16 * nb, cfg.I, 0) for e in range(cfg.k)]     # experts 0, 16, ..., 112
        pair_sets.append(moeq4.make_pairs(ent, dev))
    for p in pair_sets:                                                     # warm up
        moeq4.moe_expert_ffn_q4(ctx, p, cfg.k + 1, x, 1, y)
    reps = 200
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(0)
    clocks.start()
    runs = []
    for _ in range(REPEATS):
        torch.cuda.synchronize()
        e0.record()
        for r in range(reps):
            moeq4.moe_expert_ffn_q4(ctx, pair_sets[r % len(pair_sets)], cfg.k + 1, x, 1, y)
        e1.record()
        torch.cuda.synchronize()
        runs.append(e0.elapsed_time(e1) * 1000.0 / reps)
    clk = clocks.stop()
    moeq4.moe_ctx_check(ctx)
    us = statistics.median(runs)
    algo = cfg.k * nb + nbs
    print(json.dumps({"metric": METRIC, "workload": "direct: moe_expert_ffn_q4, one token, "
                                                    "shared + 8 routed experts",
                      "unit": "us per call", "value": round(us, 2),
                      "us_min_max": [round(min(runs), 2), round(max(runs), 2)],
                      "timing": f"median of {REPEATS} runs of {reps} calls", "clocks": clk,
                      "algorithmic_bytes": algo, "achieved_gbs": round(algo / (us * 1e-6) / 1e9, 1),
                      "frac_of_hbm": round(algo / (us * 1e-6) / 1e9 / hbm, 4), "peak_kind": kind,
                      "kernels": "k_ffn_gateup_simple + k_ffn_down_simple"}), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "streaming":
        run_streaming(args)
    elif args.workload == "batched":
        run_batched(args)
    elif args.workload == "prefill":
        run_prefill(args)
    elif args.workload == "storage":
        run_storage(args)
    elif args.workload == "direct":
        run_direct(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
