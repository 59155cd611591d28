"""Benchmark of the fine-grained MoE layer on B200.

One step = one whole-layer call (moe_forward: router + top-6, dispatch,
grouped SwiGLU experts + shared expert, combine) over one batch of N tokens
whose inputs already sit in HBM. The headline workload is the Kolibri-shaped
decode layer (N = 32, d = 2560, E = 384, top-6 + 1 shared, I = 512, BF16
expert weights, FP32 router); the prefill layer (N = 8192) is reported in the
same line under "prefill".

Launch: python bench.py [--gpus N --steps K --warmup W] [--impl reference]
With N > 1 (torchrun), every rank runs an independent replica on its own
tokens: tokens are independent, so the layer shards with no collective
(weak scaling); rank 0 prints the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from fine_grained_sparse_fp32_b200 import _build, kmoe  # noqa: E402
from fine_grained_sparse_fp32_b200.inputs import (CONFIGS, expected_distinct_experts, make_block_inputs,  # noqa: E402
                                                  make_inputs, make_x)

METRIC = "MoE-layer tokens/s at 1 B200 (decode N=32, prefill N=8192); % of HBM/tensor roofline"
ROTATE = 8           # distinct token batches cycled through the timed steps


# DRAM bytes (read + write) per launch of each workload's FFN kernel(s), from
# one ncu capture of `bench.py --capture <workload> --calls 4` (metrics
# dram__bytes_read.sum and dram__bytes_write.sum, -k regex:ffn_, mean over the
# 4 launches). They hold only for the kernel sources they were measured on:
# each entry is keyed by a hash of those files, and a changed kernel reports
# no traffic until it is measured again.
TRAFFIC_SOURCES = {
    "swap": ('fine_grained_sparse_fp32_b200/csrc/ffn_swap.cu', 'fine_grained_sparse_fp32_b200/csrc/swap_units.cuh', 'fine_grained_sparse_fp32_b200/csrc/sm100.cuh', 'fine_grained_sparse_fp32_b200/csrc/common.cuh'),
    "a8": ('fine_grained_sparse_fp32_b200/csrc/ffn_a8.cu', 'fine_grained_sparse_fp32_b200/csrc/swap_units.cuh', 'fine_grained_sparse_fp32_b200/csrc/sm100.cuh', 'fine_grained_sparse_fp32_b200/csrc/common.cuh'),
    "tc": ('fine_grained_sparse_fp32_b200/csrc/ffn_tc.cu', 'fine_grained_sparse_fp32_b200/csrc/sm100.cuh', 'fine_grained_sparse_fp32_b200/csrc/common.cuh'),
}
TRAFFIC = {
    "decode": ("swap", "b6401135bdb7745e", 1197.4e6),
    "fp8_decode": ("a8", "1dd307aeb0673877", 599.3e6),
    "fp8a8_decode": ("a8", "1dd307aeb0673877", 599.2e6),
    "fp8a8_prefill": ("a8", "1dd307aeb0673877", 1699.2e6),
    "prefill": ("tc", "696ba858c73ac825", 3689.9e6),   # up + down kernel
    "fp8_prefill": ("tc", "696ba858c73ac825", 1756.0e6),   # up + down kernel
    "skew": ("tc", "696ba858c73ac825", 8471.2e6),   # up + down kernel
}


def kernel_traffic(layer):
    import hashlib
    entry = TRAFFIC.get(layer)
    if entry is None:
        return None
    group, key, value = entry
    h = hashlib.sha256()
    try:
        for f in TRAFFIC_SOURCES[group]:
            with open(os.path.join(ROOT, f), "rb") as fh:
                h.update(fh.read())
    except OSError:
        return None
    return value if h.hexdigest()[:16] == key else None


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as fh:
            p = json.load(fh)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ helpers
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def bytes_per_weight(cfg):
    return {"f32": 4, "bf16": 2, "e4m3": 1, "e4m3_a8": 1}[cfg.w_dtype]


def algorithmic(cfg, distinct_routed: float):
    """Algorithmic bytes and FLOPs of one layer call (intermediates excluded)."""
    per_expert = cfg.expert_weights * bytes_per_weight(cfg)
    if cfg.fp8_weights:
        per_expert += 3 * (cfg.d // 128) * (cfg.I // 128) * 4
    xb = 4 if cfg.x_dtype == "f32" else 2
    weights = (distinct_routed + 1) * per_expert
    act = cfg.N * cfg.d * xb + cfg.N * cfg.d * 2
    router = cfg.E * cfg.d * 4 + cfg.E * 4
    flops = 2 * cfg.N * cfg.d * cfg.E + 2 * cfg.N * (cfg.K + 1) * 3 * cfg.d * cfg.I
    ffn_bytes = weights + cfg.N * cfg.d * xb + (cfg.N * cfg.K + cfg.N) * cfg.d * 2
    return {"layer_bytes": weights + act + router, "ffn_bytes": ffn_bytes, "flops": flops,
            "expert_weight_bytes": weights}


def fp8_mma(cfg):
    """Whether the layer's expert GEMMs run as FP8 x FP8 MMAs: FP8 activations, or E4M3 weights
    with two-term BF16 activations below 256 tokens (mirrors abi.cu's dispatch)."""
    return cfg.w_dtype == "e4m3_a8" or (cfg.w_dtype == "e4m3" and cfg.x_dtype == "bf16" and cfg.N < 256)


def launches_per_step(cfg):
    """Kernels of this library that one moe_forward launches (mirrors abi.cu's dispatch)."""
    if fp8_mma(cfg):
        ffn = 2             # x quantiser (one or two terms), FP8 tensor-core FFN (up and down units, one launch)
    elif cfg.x_dtype == "bf16" and cfg.w_dtype == "bf16" and cfg.N < 256:
        ffn = 1             # swap-AB FFN (up and down units, one launch)
    else:
        ffn = 2             # ffn up, ffn down
    if cfg.N <= 256:
        return 3 + ffn + 1  # router logits, top-K, permute, FFN, combine
    router = 2 if (cfg.x_dtype == "bf16" and cfg.N >= 512) else 1   # split + tcgen05 router | SIMT router
    chunks = (cfg.N + 255) // 256
    permute = 1 if chunks <= 64 else 2      # scatter with the scan folded in | scan, scatter (top-K counts)
    return router + 1 + permute + ffn + 1   # + top-K, permute, FFN, combine


# --------------------------------------------------------------- GPU arm
def run_config(cfg, steps, warmup, rank, world, seed=0, use_graph=True, cpu_sample=0):
    dev = torch.device("cuda", torch.cuda.current_device())
    layer = make_inputs(cfg, seed=seed, device=dev)
    # the oracle on the same layer, on a bounded token sample (host cores; rank 0 of a 1-GPU run only)
    cpu = oracle_rates(cfg, layer, cpu_sample) if cpu_sample else None
    lay = kmoe.Layer(layer, cfg.N)
    xs = [make_x(cfg, seed=1000 * rank + 17 * i + 1, device=dev) for i in range(ROTATE)]
    ys = [torch.empty((cfg.N, cfg.d), dtype=torch.bfloat16, device=dev) for _ in range(ROTATE)]
    counts = [torch.empty(cfg.E, dtype=torch.int32, device=dev) for _ in range(ROTATE)]
    stream = torch.cuda.Stream(device=dev)
    with torch.cuda.stream(stream):
        for i in range(ROTATE):
            lay.forward(xs[i], y=ys[i], counts=counts[i], stream=stream)
    stream.synchronize()
    distinct = float(np.mean([(c > 0).sum().item() for c in counts]))

    # One graph per step, and one graph holding a whole cycle of ROTATE
    # consecutive steps (the way a model's forward pass replays many layer
    # calls from a single graph); the timed loop replays cycles and fills any
    # remainder with single steps, so it runs exactly `steps` layer calls.
    graphs = []
    cycle = None
    if use_graph:
        for i in range(ROTATE):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                lay.forward(xs[i], y=ys[i], counts=counts[i], stream=stream)
            graphs.append(g)
        cycle = torch.cuda.CUDAGraph()
        with torch.cuda.graph(cycle, stream=stream):
            for i in range(ROTATE):
                lay.forward(xs[i], y=ys[i], counts=counts[i], stream=stream)

    def step(i):
        if use_graph:
            graphs[i % ROTATE].replay()
        else:
            lay.forward(xs[i % ROTATE], y=ys[i % ROTATE], counts=counts[i % ROTATE], stream=stream)

    def run_steps(n, single=False):
        i = 0
        while i < n:
            if cycle is not None and not single and n - i >= ROTATE:
                cycle.replay()
                i += ROTATE
            else:
                step(i)
                i += 1

    with torch.cuda.stream(stream):
        run_steps(warmup)
    torch.cuda.synchronize()
    barrier(world)
    clocks = ClockSampler(torch.cuda.current_device()) if rank == 0 else None
    time.sleep(0.3 if clocks else 0)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    with torch.cuda.stream(stream):
        t0.record(stream)
        run_steps(steps)
        t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1)
    clk = clocks.stop() if clocks else None
    ms_max = all_max(ms, world)

    # the same steps replayed one graph per step (reported beside the main number)
    single_ms = None
    if cycle is not None:
        barrier(world)
        with torch.cuda.stream(stream):
            t0.record(stream)
            run_steps(steps, single=True)
            t1.record(stream)
        torch.cuda.synchronize()
        single_ms = all_max(t0.elapsed_time(t1), world) / steps

    # per-kernel-group timing of the dominant step (grouped FFN), decomposed calls
    ffn_ms = time_grouped_ffn(layer, xs, stream, steps=max(20, min(steps, 400)))

    # end to end: pinned host x -> device, layer, device y -> pinned host
    e2e_ms = time_e2e(lay, cfg, xs, stream, steps=max(20, min(steps, 400)), warmup=max(3, warmup // 4))
    alg = algorithmic(cfg, distinct)
    return {"ms_per_step": ms_max / steps, "single_graph_ms": single_ms, "clocks": clk, "distinct": distinct, "alg": alg,
            "ffn_ms": ffn_ms, "e2e_ms": e2e_ms, "cpu": cpu}


def time_block(cfg, steps, warmup, seed=0):
    """Average step of the sandwich block (pre-norm, layer, post-norm + residual) on
    rotating residual streams, in CUDA graphs; h_out is written in place."""
    dev = torch.device("cuda", torch.cuda.current_device())
    layer = make_inputs(cfg, seed=seed, device=dev)
    lay = kmoe.Layer(layer, cfg.N, block=True)
    blks = [make_block_inputs(cfg, seed=31 * i + 7, device=dev) for i in range(ROTATE)]
    stream = torch.cuda.Stream(device=dev)
    eps = 1e-6

    def call(i):
        b = blks[i % ROTATE]
        lay.block_forward(b["h"], b["gamma_pre"], b["gamma_post"], eps, h_out=b["h"], stream=stream)

    with torch.cuda.stream(stream):
        call(0)
    stream.synchronize()
    graphs = []
    for i in range(ROTATE):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            call(i)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            graphs[i % ROTATE].replay()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        t0.record(stream)
        for i in range(steps):
            graphs[i % ROTATE].replay()
        t1.record(stream)
    torch.cuda.synchronize()
    status = kmoe.moe_device_status(lay.ws)
    return {"ms_per_step": t0.elapsed_time(t1) / steps, "status": status}


def time_grouped_ffn(layer, xs, stream, steps):
    """Average duration of one moe_grouped_ffn call (the expert FFN kernels)."""
    cfg = layer["cfg"]
    dev = xs[0].device
    preps = []
    with torch.cuda.stream(stream):
        for x in xs:
            idx, w = kmoe.moe_router_topk(x, layer["w_router"], layer["bias"], cfg.K, stream=stream)
            _, offsets, perm, _ = kmoe.moe_permute(idx, cfg.E, stream=stream)
            preps.append((x, perm, offsets))
    ws = kmoe.workspace(cfg.N, cfg.d, cfg.E, cfg.K, cfg.I, kmoe.dtype_code(xs[0].dtype), kmoe.w_dtype_code(cfg.w_dtype),
                        dev)
    adt = kmoe.act_dtype_for(cfg.w_dtype)
    y_perm = torch.empty((cfg.N * cfg.K, cfg.d), dtype=adt, device=dev)
    y_shared = torch.empty((cfg.N, cfg.d), dtype=adt, device=dev)
    for x, p, o in preps:
        kmoe.moe_grouped_ffn(x, layer, p, o, ws=ws, stream=stream, out=(y_perm, y_shared))
    stream.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    with torch.cuda.stream(stream):
        for i in range(steps):
            x, p, o = preps[i % len(preps)]
            ev[i][0].record(stream)
            kmoe.moe_grouped_ffn(x, layer, p, o, ws=ws, stream=stream, out=(y_perm, y_shared))
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ev]))


def time_e2e(lay, cfg, xs, stream, steps, warmup):
    """End to end through Layer.forward: every step copies its token batch from pinned host memory
    to the device, runs the layer and copies y back to pinned host memory, all inside the timed
    region. Timed twice: with eager launches, and with each step (copy in, layer, copy out) replayed
    from a CUDA graph, the way a serving loop replays a step. The graph figure is the reported one."""
    xb = 4 if cfg.x_dtype == "f32" else 2
    hx = [x.cpu().pin_memory() for x in xs]
    hy = torch.empty((cfg.N, cfg.d), dtype=torch.bfloat16).pin_memory()
    dx = torch.empty_like(xs[0])
    dy = torch.empty((cfg.N, cfg.d), dtype=torch.bfloat16, device=xs[0].device)

    def one(i):
        dx.copy_(hx[i % len(hx)], non_blocking=True)
        lay.forward(dx, y=dy, stream=stream)
        hy.copy_(dy, non_blocking=True)

    def timed(run):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            for i in range(steps):
                run(i)
            t1.record(stream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / steps

    with torch.cuda.stream(stream):
        for i in range(warmup):
            one(i)
    torch.cuda.synchronize()
    eager = timed(one)
    graphs = []
    for i in range(len(hx)):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            one(i)
        graphs.append(g)
    with torch.cuda.stream(stream):
        for i in range(warmup):
            graphs[i % len(graphs)].replay()
    torch.cuda.synchronize()
    graphed = timed(lambda i: graphs[i % len(graphs)].replay())
    return {"ms": graphed, "ms_eager": eager, "h2d": cfg.N * cfg.d * xb, "d2h": cfg.N * cfg.d * 2}


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def all_max(v, world):
    """Max of a per-rank value over all ranks (NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return v
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def whole_job_tokens_per_s(tokens_per_rank, world, ms_max):
    """Replicas: every rank processes its own tokens; the job's throughput is all
    ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / (ms_max / 1e3)


# --------------------------------------------------------------- CPU oracle
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_rates(cfg, layer, n_tokens):
    """The oracle as it stands on the first n_tokens tokens of this workload, timed with all host
    cores and with one thread (a quarter of the sample), in tokens/s. The skewed layer's sample
    stands in for its 65,536 tokens: the rate is per token, and the full-layer time it implies is
    an extrapolation, labelled so."""
    import oracle
    from fine_grained_sparse_fp32_b200.inputs import to_host
    host = to_host(layer)
    fn = oracle.layer_a8 if cfg.w_dtype == "e4m3_a8" else oracle.layer
    nt = oracle.max_threads()
    rows = np.arange(min(n_tokens, cfg.N), dtype=np.int32)
    t = time.perf_counter()
    fn(host, rows=rows, nthreads=nt)
    all_cores = len(rows) / (time.perf_counter() - t)
    rows1 = rows[: max(1, len(rows) // 4)]
    t = time.perf_counter()
    fn(host, rows=rows1, nthreads=1)
    one = len(rows1) / (time.perf_counter() - t)
    out = {"tokens_per_s_all_cores": all_cores, "tokens_per_s_1_thread": one, "cores": nt,
           "sample": f"{len(rows)} of {cfg.N} tokens (all cores), {len(rows1)} (1 thread)"}
    if cfg.N > len(rows):
        out["full_layer_s_extrapolated"] = cfg.N / all_cores
    return out


# ------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", default="kmoe", choices=["kmoe", "reference"])
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the FP8 and skewed-routing layers")
    ap.add_argument("--cpu-tokens", type=int, default=32)
    ap.add_argument("--capture", default=None, metavar="LAYER",
                    help="untimed: run --calls whole-layer calls of one workload (for ncu captures) and exit")
    ap.add_argument("--calls", type=int, default=4)
    args = ap.parse_args()
    world, rank, local = dist_env()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.capture:
        return run_capture(args.capture, args.calls)

    if world > 1:
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    _build.build()
    kmoe.load()

    hbm, tflops, tflops_sus, peak_kind = peaks()
    dec = CONFIGS["decode"]
    cpu_n = args.cpu_tokens if (world == 1 and rank == 0) else 0
    r = run_config(dec, args.steps, args.warmup, rank, world, use_graph=not args.no_graph, cpu_sample=cpu_n)
    pre = None
    extras = {}
    blocks = {}
    if not args.no_prefill:
        pcfg = CONFIGS["prefill"]
        psteps = max(10, min(args.steps // 10, 200))
        pre = run_config(pcfg, psteps, max(3, args.warmup // 10), rank, world, use_graph=not args.no_graph,
                         cpu_sample=cpu_n)
        torch.cuda.empty_cache()
        if not args.no_extra:
            for name, n_steps in (("fp8_decode", max(20, min(args.steps, 1000))), ("fp8_prefill", 50),
                                  ("fp8a8_decode", max(20, min(args.steps, 1000))), ("fp8a8_prefill", 50),
                                  ("skew", 10)):
                extras[name] = run_config(CONFIGS[name], n_steps, 3, rank, world, use_graph=not args.no_graph,
                                          cpu_sample=cpu_n)
                torch.cuda.empty_cache()
            if not args.no_graph:
                blocks = {"decode": time_block(dec, max(20, min(args.steps, 1000)), 10),
                          "prefill": time_block(CONFIGS["prefill"], 50, 3)}
                torch.cuda.empty_cache()

    if rank == 0:
        ms = r["ms_per_step"]
        value = whole_job_tokens_per_s(dec.N, world, ms)
        alg = r["alg"]
        ffn_gbs = alg["ffn_bytes"] / (r["ffn_ms"] / 1e3) / 1e9
        layer_gbs = alg["layer_bytes"] / (ms / 1e3) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": decode_config(world, args.no_graph),
            "roofline": {"bound": "hbm", "kernel": "moe_grouped_ffn: ffn_swap_kernel (up and down units, one launch)",
                         "achieved": ffn_gbs, "peak": hbm, "unit": "GB/s", "frac": ffn_gbs / hbm,
                         "traffic": kernel_traffic("decode"), "peak_kind": peak_kind + " burst",
                         "layer_achieved": layer_gbs, "layer_frac": layer_gbs / hbm,
                         "algorithmic_bytes_per_launch": alg["ffn_bytes"], "launch_ms": r["ffn_ms"]},
            "e2e": {"value": dec.N * world / (r["e2e_ms"]["ms"] / 1e3), "unit": "tokens/s",
                    "how": "pinned host x -> device, layer, device y -> pinned host, each step one CUDA graph replay",
                    "value_eager_launches": dec.N * world / (r["e2e_ms"]["ms_eager"] / 1e3),
                    "h2d_bytes_per_step": r["e2e_ms"]["h2d"], "d2h_bytes_per_step": r["e2e_ms"]["d2h"]},
            "gpu_launches": launches_per_step(dec) * args.steps,
            "clocks": r["clocks"],
            "ms_per_step_one_graph_per_step": r["single_graph_ms"],
            "distinct_experts_per_step": r["distinct"],
        }
        if pre is not None:
            pcfg = CONFIGS["prefill"]
            pms = pre["ms_per_step"]
            palg = pre["alg"]
            t_hbm = palg["layer_bytes"] / (hbm * 1e9)
            t_tc = palg["flops"] / (tflops * 1e12)
            line["prefill"] = {
                "value": pcfg.N * world / (pms / 1e3), "unit": "tokens/s", "ms_per_step": pms,
                "roofline_time_ms": max(t_hbm, t_tc) * 1e3, "bound": "hbm" if t_hbm >= t_tc else "tensor",
                "frac": max(t_hbm, t_tc) * 1e3 / pms,
                "tflops": palg["flops"] / (pms / 1e3) / 1e12, "tensor_frac": palg["flops"] / (pms / 1e3) / (tflops * 1e12),
                "ffn_ms": pre["ffn_ms"], "clocks": pre["clocks"], "gpu_launches_per_step": launches_per_step(pcfg),
                "e2e": {"value": pcfg.N * world / (pre["e2e_ms"]["ms"] / 1e3), "unit": "tokens/s"},
                "cpu_oracle": pre["cpu"],
                "traffic": kernel_traffic("prefill"),
                "ffn_algorithmic_bytes": palg["ffn_bytes"],
            }
        for name, r_x in extras.items():
            xcfg = CONFIGS[name]
            xms = r_x["ms_per_step"]
            xalg = r_x["alg"]
            # FP8 x FP8 MMAs: the measured BF16 peak times the nominal FP8 / BF16 ratio of 2
            tc_peak = tflops * (2.0 if fp8_mma(xcfg) else 1.0)
            t_hbm = xalg["layer_bytes"] / (hbm * 1e9)
            t_tc = xalg["flops"] / (tc_peak * 1e12)
            line[name] = {
                "value": whole_job_tokens_per_s(xcfg.N, world, xms), "unit": "tokens/s", "ms_per_step": xms,
                "N": xcfg.N, "weights": xcfg.w_dtype, "distinct_experts_per_step": r_x["distinct"],
                "roofline_time_ms": max(t_hbm, t_tc) * 1e3, "bound": "hbm" if t_hbm >= t_tc else "tensor",
                "frac": max(t_hbm, t_tc) * 1e3 / xms, "tflops": xalg["flops"] / (xms / 1e3) / 1e12,
                "tensor_peak_tflops": tc_peak,
                "ffn_frac": xalg["ffn_bytes"] / (r_x["ffn_ms"] / 1e3) / 1e9 / hbm,
                "ffn_ms": r_x["ffn_ms"], "ffn_gbs": xalg["ffn_bytes"] / (r_x["ffn_ms"] / 1e3) / 1e9,
                "gpu_launches_per_step": launches_per_step(xcfg), "clocks": r_x["clocks"],
                "traffic": kernel_traffic(name), "ffn_algorithmic_bytes": xalg["ffn_bytes"],
                "cpu_oracle": r_x["cpu"],
            }
        if blocks:
            base = {"decode": ms, "prefill": pre["ms_per_step"] if pre else None}
            line["block"] = {
                "what": "RMSNorm -> layer -> RMSNorm + residual, BF16 residual stream updated in place",
                **{k: {"ms_per_step": v["ms_per_step"], "layer_ms_per_step": base[k],
                       "value": CONFIGS[k].N * world / (v["ms_per_step"] / 1e3), "unit": "tokens/s",
                       "device_status": v["status"]} for k, v in blocks.items()},
            }
        if world == 1 and r["cpu"]:
            c = r["cpu"]
            line["cpu_baseline"] = {"value": c["tokens_per_s_all_cores"], "unit": "tokens/s", "cores": c["cores"],
                                    "kind": "oracle", "sample": c["sample"] + " of the decode layer, whole layer in double",
                                    "value_1_thread": c["tokens_per_s_1_thread"], "cpu_model": cpu_model()}
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


def run_capture(name, calls):
    """A few untimed whole-layer calls of one workload, on rotating token
    batches: the command that ncu profiles (no number is reported)."""
    _build.build()
    kmoe.load()
    cfg = CONFIGS[name]
    dev = torch.device("cuda", 0)
    layer = make_inputs(cfg, seed=0, device=dev)
    lay = kmoe.Layer(layer, cfg.N)
    xs = [make_x(cfg, seed=17 * i + 1, device=dev) for i in range(min(calls, ROTATE))]
    for i in range(calls):
        y = lay.forward(xs[i % len(xs)])
    torch.cuda.synchronize()
    status = kmoe.moe_device_status(lay.ws)
    print(json.dumps({"capture": name, "calls": calls, "device_status": status,
                      "y_abs_mean": float(y.float().abs().mean())}), flush=True)
    if status != 0:
        raise SystemExit(f"device status {status}")


def decode_config(world, no_graph=False):
    """The workload description both arms report (the GPU arm and the oracle)."""
    cfg = CONFIGS["decode"]
    w = algorithmic(cfg, expected_distinct_experts(cfg))["expert_weight_bytes"]
    return {"workload": "decode layer N=32 d=2560 E=384 top-6+1 shared I=512, BF16 experts, FP32 router",
            "tokens_per_gpu": cfg.N, "parallelism": f"replicas x{world} (no collective)",
            "l2": "inputs larger than L2: ~%.2f GB of expert weights per step (expected), %d rotating token "
                  "batches" % (w / 1e9, ROTATE),
            "cuda_graph": (f"{ROTATE} consecutive layer calls per graph" if not no_graph else False)}


def run_reference(args, world, rank):
    """The oracle on the host cores, on this arm's metric and workload."""
    if rank != 0:
        return
    import oracle
    from fine_grained_sparse_fp32_b200.inputs import to_host
    cfg = CONFIGS["decode"]
    host = to_host(make_inputs(cfg, seed=0, device="cuda" if torch.cuda.is_available() else "cpu"))
    # each step evaluates a bounded token sample so that K steps stay within a
    # couple of minutes of host time (about 1600 token evaluations in total)
    sample = max(1, min(cfg.N, 1600 // max(args.steps, 1)))
    rows = np.arange(sample, dtype=np.int32)
    nt = min(oracle.max_threads(), sample)
    for _ in range(args.warmup):
        oracle.layer(host, rows=rows, nthreads=nt)
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        oracle.layer(host, rows=rows, nthreads=nt)
        times.append(time.perf_counter() - t)
    per_token = float(np.sum(times)) / (sample * len(times))
    value = 1.0 / per_token
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": len(times), "warmup": args.warmup, "ms_per_step": per_token * cfg.N * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": decode_config(world, args.no_graph),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": nt, "kind": "oracle",
                             "sample": f"{sample} of the {cfg.N} decode tokens per step, whole layer in double"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
