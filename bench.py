#!/usr/bin/env python
"""Benchmark of the BitLinear W1.58A8 forward on B200.

Headline (``value``): decode GB/s of packed ternary weights streamed per
second for the 2B-class decode step (one token through BitLinear K=2560 ->
N=6912 and K=2560 -> N=2560, bf16 in/out), whole job over all ranks.  A step
is one pass of the inference forward over one batch: per-token activation
quantisation, ternary x int8 product with int32 accumulation and fused
dequantisation, for every layer of the workload.  The weights are packed once
at load time (absmean + ternarise + pack), as a deployed checkpoint is; that
offline path is timed separately under ``pack``.

Also reported in the same line: the 2B prefill GEMM (2048 tokens) in int8
TOPS against the tensor-core roofline, the 70B-class decode layer chain
at 1 and 8 tokens and the 3B-class decode layers at 1 to 16 tokens in GB/s.  Inputs are seeded and synthetic with the pages'
shapes and distributions; weights rotate over enough copies that every step
reads them from HBM (more than 4x the L2 size).

``--impl reference`` times the CPU oracle (plain scalar C, one core) on the
same workload, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "BitLinear decode GB/s (% HBM peak) + prefill int8 TOPS (% peak), 1 B200"
UNIT = "GB/s"
DECODE_LAYERS = [(2560, 6912), (2560, 2560)]  # (K in, N out)
PREFILL = dict(M=2048, K=2560, N=6912)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100000, help="timed decode steps")
    p.add_argument("--warmup", type=int, default=2000)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-extras", action="store_true", help="skip prefill / 70B chain / pack lines")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--only", choices=["prefill", "chain70b", "decode3b", "next"], default=None,
                   help="run one secondary workload alone and print its own line (a small case for profiling)")
    return p.parse_args()


# DRAM traffic per launch from the committed ncu summaries.  A figure is used
# only while the kernel's sources hash to what they were when it was taken.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")
KERNEL_SOURCES = {
    "gemv": ["ternary_weight_a8_b200/csrc/gemv.cu", "ternary_weight_a8_b200/csrc/common.cuh"],
    "gemm": ["ternary_weight_a8_b200/csrc/gemm_tcgen05.cu", "ternary_weight_a8_b200/csrc/common.cuh"],
}


def kernel_source_hash(kernel: str) -> str:
    import hashlib

    h = hashlib.sha1()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(key: str, kernel: str):
    """Bytes per launch recorded for `key`, or None if absent or taken on other sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            for line in f:
                parts = line.split()
                if len(parts) >= 3 and not line.startswith("#") and parts[0] == key:
                    return float(parts[1]) if parts[2] == kernel_source_hash(kernel) else None
    except OSError:
        pass
    return None


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            d = json.load(fh)
        return dict(hbm=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    except (OSError, KeyError, ValueError):
        return dict(hbm=FALLBACK_HBM_GBS, bf16=FALLBACK_BF16_TFLOPS, bf16_sustained=1400.0,
                    source="fallback")


# ----------------------------------------------------------------------------
# clocks sampled while the GPU is busy
# ----------------------------------------------------------------------------

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.QUERY, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [s.strip() for s in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        busy = sorted(sm)[len(sm) // 2:] if sm else []
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(smax) if smax else None, "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------
# distributed plumbing (replicas: no data-path collective)
# ----------------------------------------------------------------------------

_BACKEND = None  # process-group backend of this run (None: one rank)


def dist_init():
    """One process per GPU (NCCL); without a GPU (host-side tests) the ranks use gloo."""
    global _BACKEND
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist

        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
            _BACKEND = "nccl"
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
            _BACKEND = "gloo"
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device="cpu" if _BACKEND == "gloo" else "cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

def l2_bytes():
    import torch

    return torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size


def make_layer_sets(shapes, seed, min_bytes):
    """Packed weights for each (K, N) layer, plus byte-identical copies at other
    addresses until all sets together exceed ``min_bytes`` (cold L2 per step)."""
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    base = []
    for i, (K, N) in enumerate(shapes):
        W = torch.from_numpy(synth.latent_weights(N, K, seed=seed + i)).cuda()
        packed, gamma = tb.pack_weights(W)
        del W
        base.append((packed, gamma))
    set_bytes = sum(p.numel() for p, _ in base)
    nsets = max(1, math.ceil(min_bytes / set_bytes))
    sets = [base] + [[(p.clone(), g.clone()) for p, g in base] for _ in range(nsets - 1)]
    torch.cuda.synchronize()
    return sets, set_bytes


def make_inputs(shapes, M, seed, shared=None):
    import torch

    import synth

    xs = []
    for i, (K, N) in enumerate(shapes):
        if shared is not None and shared[i]:
            xs.append(xs[-1])
            continue
        bits, _ = synth.activations_bf16(M, K, seed=seed + 100 + i)
        xs.append(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
    ys = [torch.empty((M, N), dtype=torch.bfloat16, device="cuda") for (K, N) in shapes]
    return xs, ys


def capture(fn, steps):
    """A CUDA graph of `steps` calls fn(i)."""
    import torch

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(0)  # warm the launch paths outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                fn(i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def timed_graph_run(step_fn, steps, warmup, world, chunk=500, sampler=None):
    """Times exactly `steps` calls of step_fn, replayed as CUDA graphs; returns seconds (max over ranks)."""
    import torch

    chunk = max(1, min(chunk, steps))
    g_main = capture(lambda i: step_fn(i), chunk)
    rem = steps % chunk
    g_rem = capture(lambda i: step_fn(i), rem) if rem else None
    w_chunk = max(1, min(chunk, warmup))
    g_warm = capture(lambda i: step_fn(i), w_chunk)
    for _ in range(max(1, warmup // w_chunk)):
        g_warm.replay()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps // chunk):
        g_main.replay()
    if g_rem is not None:
        g_rem.replay()
    end.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    secs = start.elapsed_time(end) / 1e3
    del g_main, g_rem, g_warm
    return max_over_ranks(secs, world), clocks


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    import torch

    import ternary_weight_a8_b200 as tb

    torch.cuda.set_device(local)
    peaks = load_peaks()
    L2 = l2_bytes()
    out = {}

    # ---- decode 2B (headline) ----
    sets, set_bytes = make_layer_sets(DECODE_LAYERS, seed=0, min_bytes=4 * L2)
    nsets = len(sets)
    xs, ys = make_inputs(DECODE_LAYERS, 1, seed=0)
    layer_sets = [[tb.Layer(p, g, x, y) for (p, g), x, y in zip(S, xs, ys)] for S in sets]
    ws = tb.new_workspace(tb.chain_workspace_bytes(layer_sets[0], 1))

    def decode_step(i):
        # Both BitLinears of the step in one call; independent layers share one launch.
        tb.layer_chain(layer_sets[i % nsets], workspace=ws)

    sampler = ClockSampler(torch.cuda.current_device())
    secs, clocks = timed_graph_run(decode_step, args.steps, args.warmup, world, sampler=sampler)
    units = args.steps * set_bytes * world
    value = units / secs / 1e9
    launches = args.steps  # one decode kernel per step
    status = tb.device_status(ws)

    # Roofline of the dominant kernel: the decode kernel is the whole step, so its
    # average launch duration is the timed region over the launches in it.
    x_bytes = sum(K * 2 for K, N in DECODE_LAYERS)
    y_bytes = sum(N * 2 for K, N in DECODE_LAYERS)
    step_bytes = set_bytes + x_bytes + y_bytes + 8 * len(DECODE_LAYERS)
    per_launch = secs / world / launches * world  # seconds per launch on one GPU
    achieved = step_bytes / per_launch / 1e9
    roofline = {"bound": "hbm", "kernel": "gemv_group_kernel (decode 2B step: K=2560 -> N=6912 and N=2560, 1 token)",
                "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "peak_source": peaks["source"] + " HBM copy",
                "traffic": profiled_traffic("decode_2b", "gemv"), "algorithmic_bytes_per_launch": step_bytes,
                "launch_us_mean": round(per_launch * 1e6, 3)}

    # ---- e2e through the public API with host buffers ----
    # The step's inputs sit in one pinned host buffer and one device buffer (a
    # view per layer), its outputs likewise: one H2D and one D2H copy per step.
    x_numel = [x.numel() for x in xs]
    y_numel = [y.numel() for y in ys]
    x_dev = torch.empty(sum(x_numel), dtype=xs[0].dtype, device="cuda")
    y_dev = torch.empty(sum(y_numel), dtype=ys[0].dtype, device="cuda")
    x_views = [v.view(x.shape) for v, x in zip(torch.split(x_dev, x_numel), xs)]
    y_views = [v.view(y.shape) for v, y in zip(torch.split(y_dev, y_numel), ys)]
    for v, x in zip(x_views, xs):
        v.copy_(x)
    x_host = torch.empty(x_dev.shape, dtype=x_dev.dtype, pin_memory=True)
    x_host.copy_(x_dev.cpu())
    y_host = torch.empty(y_dev.shape, dtype=y_dev.dtype, pin_memory=True)
    e2e_sets = [[tb.Layer(L.packed, L.gamma, xv, yv) for L, xv, yv in zip(S, x_views, y_views)] for S in layer_sets]
    ne = min(args.steps, 2000)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(ne):
        x_dev.copy_(x_host, non_blocking=True)
        tb.layer_chain(e2e_sets[i % nsets], workspace=ws)
        y_host.copy_(y_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()  # the step's result is on the host
    e1.record()
    torch.cuda.synchronize()
    e2e_secs = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e = {"value": round(ne * set_bytes * world / e2e_secs / 1e9, 2), "unit": UNIT,
           "h2d_bytes_per_step": x_dev.numel() * x_dev.element_size(),
           "d2h_bytes_per_step": y_dev.numel() * y_dev.element_size(), "steps": ne,
           "ms_per_step": round(e2e_secs / ne * 1e3, 4)}
    del sets, layer_sets, e2e_sets

    if not args.no_extras:
        out["prefill"] = run_prefill(args, world, peaks, L2)
        out["chain_70b"] = run_chain(args, world, peaks, L2)
        out["decode_3b"] = run_decode_3b(args, world, peaks, L2)
        out["pack"] = run_pack(world)
        out["next"] = run_next(args, world, peaks, L2)

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(secs / args.steps * 1e3, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded N(0,0.02) latent weights, N(0,1) bf16 activations with 1% x20 outlier channels)",
        "config": {"workload": "decode_2b: BitLinear K=2560->N=6912 and K=2560->N=2560, 1 token, bf16 in/out, "
                               "packed 2-bit ternary weights",
                   "tokens": 1, "layers_k_n": DECODE_LAYERS, "weight_bytes_per_step": set_bytes,
                   "l2": "rotating %d byte-identical weight sets (%.0f MB > 4x L2), cold L2 every step"
                         % (nsets, nsets * set_bytes / 1e6),
                   "graph": "steps replayed as CUDA graphs of 500 steps", "parallelism": "replicas x%d" % world},
        "pct_hbm_measured": round(100 * value / world / peaks["hbm"], 2),
        "pct_hbm_nominal_8tbs": round(100 * value / world / 8000.0, 2),
        "roofline": roofline, "e2e": e2e, "gpu_launches": launches, "clocks": clocks,
        "device_status": status,
    }
    result.update(out)
    return result


def run_prefill(args, world, peaks, L2):
    import torch

    import ternary_weight_a8_b200 as tb

    M, K, N = PREFILL["M"], PREFILL["K"], PREFILL["N"]
    sets, set_bytes = make_layer_sets([(K, N)], seed=7, min_bytes=L2)
    xs = []
    import synth
    for i in range(4):
        bits, _ = synth.activations_bf16(M, K, seed=300 + i)
        xs.append(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = tb.new_workspace(tb.workspace_bytes(M, N, K))

    def step(i):
        packed, gamma = sets[i % len(sets)][0]
        tb.forward(packed, gamma, xs[i % len(xs)], y=y, workspace=ws)

    steps = 400
    secs, _ = timed_graph_run(step, steps, 20, world, chunk=100)
    ops = 2.0 * M * N * K
    tops = ops * steps * world / secs / 1e12
    # Roofline of the GEMM alone: a graph of back-to-back GEMM launches on quantised input.
    xq, sc, rs = tb.quant_act(xs[0])
    gsteps = 200
    gsecs, _ = timed_graph_run(
        lambda i: tb.forward_quantized(sets[i % len(sets)][0][0], sets[i % len(sets)][0][1], xq, sc, rs, y=y,
                                       workspace=ws), gsteps, 10, world, chunk=100)
    mean_s = gsecs / gsteps
    peak_int8 = peaks["bf16"] * INT8_PER_BF16
    k_tops = ops / mean_s / 1e12
    status = tb.device_status(ws)
    return {"metric": "prefill int8 TOPS", "value": round(tops, 1), "unit": "TOPS",
            "workload": "prefill_2b: BitLinear K=2560->N=6912 over 2048 tokens (act quant + tcgen05 GEMM)",
            "ms_per_step": round(secs / steps * 1e3, 5), "tokens_per_s": round(M * steps * world / secs, 0),
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel (tcgen05 kind::i8)", "achieved": round(k_tops, 1),
                         "peak": peak_int8, "unit": "TOPS", "frac": round(k_tops / peak_int8, 4),
                         "peak_source": "%s bf16 burst x %.0f (nominal int8/bf16 ratio)" % (peaks["source"], INT8_PER_BF16),
                         "launch_us_mean": round(mean_s * 1e6, 2),
                         "traffic": profiled_traffic("prefill_2b", "gemm"),
                         "algorithmic_bytes_per_launch": M * K + N * K // 4 + M * N * 2 + 8 * M},
            "pct_int8_nominal_4500": round(100 * tops / world / 4500.0, 2), "device_status": status}


DECODE_3B = [(3200, 8640), (8640, 3200)]  # (K in, N out)
DECODE_3B_TOKENS = (1, 2, 4, 8, 16)


def run_decode_3b(args, world, peaks, L2):
    """The 3B-class decode sweep: one BitLinear per step through the public
    single-layer call (quantisation and product), 1 to 16 tokens."""
    import torch

    import ternary_weight_a8_b200 as tb

    res = {"workload": "decode_3b: BitLinear K=3200->N=8640 and K=8640->N=3200 alone, bf16 in/out, "
                       "1/2/4/8/16 tokens, one forward call per step"}
    for li, (K, N) in enumerate(DECODE_3B):
        sets, set_bytes = make_layer_sets([(K, N)], seed=500 + li, min_bytes=4 * L2)
        for M in DECODE_3B_TOKENS:
            xs, ys = make_inputs([(K, N)], M, seed=500 + li)
            x, y = xs[0], ys[0]
            ws = tb.new_workspace(tb.workspace_bytes(M, N, K))

            def step(i):
                packed, gamma = sets[i % len(sets)][0]
                tb.forward(packed, gamma, x, y=y, workspace=ws)

            steps = min(args.steps, 4000)
            secs, _ = timed_graph_run(step, steps, min(args.warmup, 200), world, chunk=500)
            gbs = set_bytes * steps * world / secs / 1e9
            res["k%d_n%d_m%d" % (K, N, M)] = {
                "GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / world / peaks["hbm"], 2),
                "us_per_call": round(secs / steps * 1e6, 3), "tokens_per_s": round(M * steps * world / secs, 1),
                "device_status": tb.device_status(ws)}
        del sets
    return res


def run_chain(args, world, peaks, L2):
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    shapes = synth.CHAIN_70B
    sets, set_bytes = make_layer_sets(shapes, seed=1000, min_bytes=3 * L2)
    res = {"workload": "chain_70b: QKV 8192->10240, O 8192->8192, gate+up 8192->2x28672, down 28672->8192, "
                       "bf16, gate/up share one quantised input", "weight_bytes_per_step": set_bytes}
    for M in (1, 8):
        xs, ys = make_inputs(shapes, M, seed=1000, shared=synth.CHAIN_70B_SHARED_INPUT)
        layer_sets = [[tb.Layer(p, g, x, y) for (p, g), x, y in zip(S, xs, ys)] for S in sets]
        ws = tb.new_workspace(tb.chain_workspace_bytes(layer_sets[0], M))

        def step(i):
            tb.layer_chain(layer_sets[i % len(layer_sets)], workspace=ws)

        steps = min(args.steps, 300)
        secs, _ = timed_graph_run(step, steps, min(args.warmup, 10), world, chunk=100)
        gbs = set_bytes * steps * world / secs / 1e9
        res["tokens_%d" % M] = {"GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / world / peaks["hbm"], 2),
                                "us_per_chain": round(secs / steps * 1e6, 2),
                                "tokens_per_s": round(M * steps * world / secs, 1),
                                "device_status": tb.device_status(ws)}
    return res


def run_next(args, world, peaks, L2):
    """The rows beyond the forward: fused RMSNorm + quantisation (prefill and decode sizes)."""
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    out = {}
    for M, K in ((2048, 2560), (1, 8192)):
        n_in = max(4, int(4 * L2 // (M * K * 2)) + 1)  # inputs larger than L2 in total
        xs = []
        for i in range(min(n_in, 64)):
            bits, _ = synth.activations_bf16(M, K, seed=500 + i)
            xs.append(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
        g = torch.ones(K, dtype=torch.float32, device="cuda")
        xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        sc = torch.empty(M, dtype=torch.float32, device="cuda")
        rs = torch.empty(M, dtype=torch.int32, device="cuda")
        steps = 400
        secs, _ = timed_graph_run(lambda i: tb.rmsnorm_quant(xs[i % len(xs)], g, 1e-6, None, xq, sc, rs),
                                  steps, 20, world, chunk=100)
        nb = M * K * 3 + M * 8 + K * 4
        gbs = nb / (secs / steps) / 1e9
        res = {"us": round(secs / steps * 1e6, 3), "GB/s": round(gbs, 1),
               "pct_hbm_measured": round(100 * gbs / peaks["hbm"], 2), "bytes_per_call": nb}
        # Unfused comparison: the norm as separate torch ops writing bf16, then the quantisation kernel.
        def unfused(i):
            x = xs[i % len(xs)]
            xf = x.float()
            v = (xf * torch.rsqrt(xf.pow(2).mean(-1, keepdim=True) + 1e-6) * g).to(torch.bfloat16)
            tb.quant_act(v, xq, sc, rs)
        usecs, _ = timed_graph_run(unfused, steps, 20, world, chunk=100)
        res["unfused_torch_norm_then_quant_us"] = round(usecs / steps * 1e6, 3)
        out["rmsnorm_quant_%dx%d" % (M, K)] = res
    # The FFN's gated activation + quantisation of the down BitLinear's input.
    for M, N in ((2048, 6912), (1, 28672)):
        n_in = max(2, int(4 * L2 // (M * N * 4)) + 1)
        gs, us = [], []
        for i in range(min(n_in, 32)):
            gs.append(torch.from_numpy(synth.activations_bf16(M, N, seed=600 + i)[0].view("int16")).cuda()
                      .view(torch.bfloat16))
            us.append(torch.from_numpy(synth.activations_bf16(M, N, seed=700 + i)[0].view("int16")).cuda()
                      .view(torch.bfloat16))
        xq = torch.empty((M, N), dtype=torch.int8, device="cuda")
        sc = torch.empty(M, dtype=torch.float32, device="cuda")
        rs = torch.empty(M, dtype=torch.int32, device="cuda")
        steps = 400
        secs, _ = timed_graph_run(lambda i: tb.glu_quant(gs[i % len(gs)], us[i % len(us)], tb.GLU_RELU2, None, xq, sc,
                                                         rs), steps, 20, world, chunk=100)
        nb = M * N * 5 + M * 8
        gbs = nb / (secs / steps) / 1e9
        res = {"us": round(secs / steps * 1e6, 3), "GB/s": round(gbs, 1),
               "pct_hbm_measured": round(100 * gbs / peaks["hbm"], 2), "bytes_per_call": nb, "act": "relu2"}

        def unfused(i):
            g, u = gs[i % len(gs)], us[i % len(us)]
            h = (torch.relu(g.float()).square() * u.float()).to(torch.bfloat16)
            tb.quant_act(h, xq, sc, rs)
        usecs, _ = timed_graph_run(unfused, steps, 20, world, chunk=100)
        res["unfused_torch_glu_then_quant_us"] = round(usecs / steps * 1e6, 3)
        out["glu_quant_%dx%d" % (M, N)] = res
    # The lookup-table decode product against the tensor-core decode kernel, same codes, one token.
    for K, N in ((2560, 6912), (8192, 10240)):
        sets, set_bytes = make_layer_sets([(K, N)], seed=800, min_bytes=4 * L2)
        bits, _ = synth.activations_bf16(1, K, seed=801)
        xq, sc, rs = tb.quant_act(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
        y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        ws = tb.new_workspace(tb.workspace_bytes(1, N, K))
        steps = 400
        res = {"weight_bytes": set_bytes}
        for name, fn in (("lut", lambda i: tb.forward_lut(sets[i % len(sets)][0][0], sets[i % len(sets)][0][1], xq,
                                                           sc, rs, y=y)),
                         ("decode_kernel", lambda i: tb.forward_quantized(sets[i % len(sets)][0][0],
                                                                             sets[i % len(sets)][0][1], xq, sc, rs,
                                                                             y=y, workspace=ws))):
            secs, _ = timed_graph_run(fn, steps, 20, world, chunk=100)
            gbs = set_bytes / (secs / steps) / 1e9
            res[name] = {"us": round(secs / steps * 1e6, 3), "GB/s": round(gbs, 1),
                         "pct_hbm_measured": round(100 * gbs / peaks["hbm"], 2)}
        out["lut_vs_gemv_%dx%d" % (K, N)] = res
        del sets
    # The straight-through backward at the prefill shape: two bf16 tensor-core products.
    M, K, N = PREFILL["M"], PREFILL["K"], PREFILL["N"]
    codes = torch.randint(0, 3, (N, K // 4, 4), dtype=torch.int32, device="cuda")  # 2-bit codes 0..2
    packed = (codes[..., 0] | (codes[..., 1] << 2) | (codes[..., 2] << 4) | (codes[..., 3] << 6)).to(torch.uint8)
    gamma = torch.full((1,), 0.02, dtype=torch.float32, device="cuda")
    bits, _ = synth.activations_bf16(M, K, seed=900)
    xq, sc, _ = tb.quant_act(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
    dy = torch.from_numpy(synth.activations_bf16(M, N, seed=901)[0].view("int16")).cuda().view(torch.bfloat16)
    dx = torch.empty((M, K), dtype=torch.float32, device="cuda")
    dw = torch.empty((N, K), dtype=torch.float32, device="cuda")
    ws = tb.new_workspace(tb.ste_workspace_bytes(M, N, K))
    steps = 50
    secs, _ = timed_graph_run(lambda i: tb.ste_backward(packed, gamma, K, dy, xq, sc, dx=dx, dw=dw, workspace=ws),
                              steps, 5, world, chunk=50)
    flops = 2 * 2.0 * M * N * K
    tf = flops / (secs / steps) / 1e12
    out["ste_backward_2048x2560x6912"] = {"us": round(secs / steps * 1e6, 2), "TFLOP/s": round(tf, 1),
                                          "pct_bf16_measured": round(100 * tf / peaks["bf16"], 2),
                                          "flops_per_call": flops, "device_status": tb.device_status(ws)}
    return out


def run_pack(world):
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    K, N = 2560, 6912
    W = torch.from_numpy(synth.latent_weights(N, K, seed=0)).cuda()
    packed = torch.empty((N, K // 4), dtype=torch.uint8, device="cuda")
    gamma = torch.empty(1, dtype=torch.float32, device="cuda")
    ws = tb.new_workspace(tb.pack_workspace_bytes(N, K))
    for _ in range(3):
        tb.pack_weights(W, packed, gamma, ws)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    n = 20
    for _ in range(n):
        tb.pack_weights(W, packed, gamma, ws)
    b.record()
    torch.cuda.synchronize()
    s = a.elapsed_time(b) / 1e3 / n
    return {"workload": "pack K=2560, N=6912 fp32 latent -> 2-bit (gamma + ternarise + pack)",
            "us_per_call": round(s * 1e6, 1), "GB/s_latent_read": round(N * K * 4 / s / 1e9, 1)}


# ----------------------------------------------------------------------------
# the oracle (CPU) on the same workload
# ----------------------------------------------------------------------------

def oracle_decode_layers():
    """The decode_2b layers as the oracle takes them: (packed, gamma, K, x) per layer."""
    import oracle
    import synth

    layers = []
    for i, (K, N) in enumerate(DECODE_LAYERS):
        W = synth.latent_weights(N, K, seed=i)
        packed, gamma, _ = oracle.pack_weights(W)
        _, xf = synth.activations_bf16(1, K, seed=100 + i)
        layers.append((packed, gamma, K, xf))
    return layers, sum(p.size for p, *_ in layers)


def oracle_decode_steps(layers, reps):
    """reps decode steps of the oracle over `layers` (any subset of rows); returns seconds."""
    import oracle

    t0 = time.perf_counter()
    for _ in range(reps):
        for packed, gamma, K, xf in layers:
            T, ok = oracle.unpack(packed, K)
            acc, y, *_ = oracle.forward(T, gamma, xf)
            oracle.round_bf16(y)
    return time.perf_counter() - t0


def oracle_decode_setup():
    layers, set_bytes = oracle_decode_layers()
    return (lambda: oracle_decode_steps(layers, 1)), set_bytes


def row_slices(n_rows, parts):
    """Contiguous, disjoint [n0, n1) slices of n_rows rows, one per part, sizes within one."""
    return [(n_rows * c // parts, n_rows * (c + 1) // parts) for c in range(parts)]


def _oracle_rows_worker(task):
    layers, reps = task
    oracle_decode_steps(layers, 1)  # load the oracle library before timing
    return oracle_decode_steps(layers, reps)


def cpu_baseline(target_s=10.0):
    step, set_bytes = oracle_decode_setup()
    t0 = time.perf_counter()
    step()
    one = time.perf_counter() - t0
    reps = max(1, int(target_s / max(one, 1e-6)))
    t0 = time.perf_counter()
    for _ in range(reps):
        step()
    secs = time.perf_counter() - t0
    return {"value": round(reps * set_bytes / secs / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d full decode_2b steps (unpack + quantise + accumulate + dequantise + bf16 round, "
                      "both layers) on one host core, %.1f s" % (reps, secs)}


def cpu_baseline_all_cores(cpu_work_s=20.0):
    """The same oracle decode steps spread over the host's cores: each process
    takes a contiguous slice of every layer's output rows (rows are independent,
    so the slices together compute the whole step).  The pool is started with
    `spawn`, so no process inherits the CUDA context."""
    import multiprocessing

    layers, set_bytes = oracle_decode_layers()
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    cores = max(1, min(cores, 128))
    one = oracle_decode_steps(layers, 1)
    reps = max(2, int(cpu_work_s / max(one, 1e-6)))  # about cpu_work_s of CPU work in total
    tasks = []
    for c in range(cores):
        shard = []
        for packed, gamma, K, xf in layers:
            n0, n1 = row_slices(packed.shape[0], cores)[c]
            if n1 > n0:
                shard.append((packed[n0:n1], gamma, K, xf))
        tasks.append((shard, reps))
    with multiprocessing.get_context("spawn").Pool(cores) as pool:
        pool.map(_oracle_rows_worker, [(t[0], 1) for t in tasks])  # start every worker
        t0 = time.perf_counter()
        pool.map(_oracle_rows_worker, tasks, chunksize=1)
        secs = time.perf_counter() - t0
    return {"value": round(reps * set_bytes / secs / 1e9, 4), "unit": UNIT, "cores": cores, "kind": "oracle",
            "sample": "%d full decode_2b steps, each process of %d taking 1/%d of every layer's rows, %.2f s wall"
                      % (reps, cores, cores, secs)}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    step, set_bytes = oracle_decode_setup()
    steps = max(1, min(args.steps, 200))
    warm = max(0, min(args.warmup, 3))
    for _ in range(warm):
        step()
    t0 = time.perf_counter()
    for _ in range(steps):
        step()
    secs = time.perf_counter() - t0
    value = steps * set_bytes / secs / 1e9
    sample = "%d full decode_2b steps on one host core (steps capped at 200)" % steps
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": round(secs / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": "decode_2b: BitLinear K=2560->N=6912 and K=2560->N=2560, 1 token, bf16 in/out"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    args = parse_args()
    world, rank, local = dist_init() if args.impl == "ours" else (
        int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), 0)
    if args.impl == "reference":
        res = run_reference(args, world, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if args.only:
        import torch

        torch.cuda.set_device(local)
        fn = {"prefill": run_prefill, "chain70b": run_chain, "decode3b": run_decode_3b, "next": run_next}[args.only]
        res = fn(args, world, load_peaks(), l2_bytes())
        if rank == 0:
            print(json.dumps(res), flush=True)
        return
    res = run_ours(args, world, rank, local)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline()
        try:
            res["cpu_baseline_all_cores"] = cpu_baseline_all_cores()
        except Exception as e:  # a secondary figure: report why it is missing, keep the line
            res["cpu_baseline_all_cores"] = {"unavailable": "%s: %s" % (type(e).__name__, e)}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


if __name__ == "__main__":
    main()
