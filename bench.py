#!/usr/bin/env python
"""Benchmark of the BitLinear W1.58A8 forward on B200.

Headline (``value``): decode GB/s of packed ternary weights streamed per
second by the 70B-class decode layer chain at one token (QKV 8192->10240, O
8192->8192, gate and up 8192->28672 each, down 28672->8192; bf16 in/out;
gate and up share one input), whole job over all ranks.  A step is one pass
of the inference forward over one batch: per-token activation quantisation,
ternary x int8 product with int32 accumulation and fused dequantisation, for
every layer of the workload.  The weights are packed once at load time
(absmean + ternarise + pack), as a deployed checkpoint is; that offline path
is timed separately under ``pack``.

Timing: the K steps of a run are captured in CUDA graphs; those exact graphs
are replayed once or more before timing (warm-up), then the K steps are
timed as a block with CUDA events, repeated until the timed blocks cover a
minimum time; ``ms_per_step`` is the median block over K.  Decode weights
rotate over byte-identical copies that together exceed the L2 size several
times, so every step reads them from HBM (inputs larger than L2: no flush,
whose dirty lines would be written back inside the next block); the other
sections write a buffer of twice the L2 size before every block.

Also in the same line: ``decode`` (the same chain at 8 and 16 tokens, the
2B-class decode step and the 3B-class layers at 1 to 16 tokens), ``prefill``
(the 2B prefill GEMM over 2048 tokens in int8 TOPS, with the GEMM's own
roofline), ``pack`` and ``next`` (the rows beyond the forward).

``--impl reference`` times the CPU oracle (plain scalar C, one host core) on
the same workload, as the reference arm.
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
# The 70B-class layer chain (K in, N out); gate and up share one input.
CHAIN_70B = [(8192, 10240), (8192, 8192), (8192, 28672), (8192, 28672), (28672, 8192)]
CHAIN_70B_SHARED_INPUT = [False, False, False, True, False]
CHAIN_WORKLOAD = ("chain_70b: BitLinear QKV 8192->10240, O 8192->8192, gate 8192->28672, up 8192->28672, "
                  "down 28672->8192 as one decode step, bf16 in/out, gate and up share one quantised input, "
                  "packed 2-bit ternary weights")
DECODE_LAYERS = [(2560, 6912), (2560, 2560)]  # the 2B-class decode step (K in, N out)
PREFILL = dict(M=2048, K=2560, N=6912)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense ratio (4.5 POPS int8 / 2.25 PFLOPS bf16)
CPU_SAMPLE_ROWS = 8  # the CPU legs take the first 1/8 of every layer's output rows


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200, help="timed steps of the headline workload")
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-extras", action="store_true", help="headline only (no decode / prefill / pack / next)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--only", choices=["chain70b", "decode2b", "prefill", "decode3b", "next", "ffn"], default=None,
                   help="run one workload alone and print its own line (a small case for profiling)")
    p.add_argument("--tokens", type=str, default=None,
                   help="with --only chain70b / ffn / decode3b: the token counts to run, comma-separated")
    return p.parse_args(argv)


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
# timing
# ----------------------------------------------------------------------------

def l2_bytes():
    import torch

    return torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size


def capture(fn, steps, first=0):
    """A CUDA graph of the calls fn(first), ..., fn(first + steps - 1)."""
    import torch

    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn(first)  # warm the launch paths outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                fn(first + i)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def rep_plan(steps: int, est_block_s: float, min_region_s: float, max_reps: int = 5000) -> int:
    """Number of timed blocks of `steps` steps so that together they cover min_region_s."""
    if est_block_s <= 0:
        return max_reps
    return int(max(1, min(max_reps, math.ceil(min_region_s / est_block_s))))


class _L2Flush:
    """Writes a buffer of twice the L2 size (outside the timed blocks)."""

    def __init__(self):
        import torch

        self.buf = torch.empty(2 * l2_bytes() // 4 + 1024, dtype=torch.int32, device="cuda")

    def __call__(self):
        self.buf.fill_(1)


def timed_graph_run(step_fn, steps, warmup, world, chunk=500, sampler=None, min_region_s=0.05, flush=True):
    """Times `steps` consecutive calls of step_fn replayed as CUDA graphs.

    The graphs holding the `steps` calls are captured once and replayed (all of
    them) at least once and for at least `warmup` steps before timing.  Then
    the whole block of `steps` calls is timed with CUDA events (L2 flushed
    before each block unless `flush` is false: inputs larger than L2; the
    blocks are then enqueued back to back), repeated until the blocks cover
    `min_region_s`.
    Returns (median seconds per block of `steps` calls, max over ranks; info).
    """
    import torch

    chunk = max(1, min(chunk, steps))
    n_full, rem = divmod(steps, chunk)
    graphs = [capture(step_fn, chunk)] * n_full if n_full else []
    if rem:
        graphs.append(capture(step_fn, rem, first=n_full * chunk))

    def block():
        for g in graphs:
            g.replay()

    flush = _L2Flush() if flush else (lambda: None)
    for _ in range(max(1, math.ceil(warmup / steps))):
        block()
    torch.cuda.synchronize()
    # One block timed alone sizes the repetition count (every rank takes the largest).
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush()
    a.record()
    block()
    b.record()
    torch.cuda.synchronize()
    reps = rep_plan(steps, max_over_ranks(a.elapsed_time(b) / 1e3, world), min_region_s)
    reps = int(max_over_ranks(float(reps), world))
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    if sampler:
        sampler.start()
    barrier(world)
    torch.cuda.synchronize()
    for e0, e1 in ev:
        flush()
        e0.record()
        block()
        e1.record()
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    times = [e0.elapsed_time(e1) / 1e3 for e0, e1 in ev]
    med = max_over_ranks(statistics.median(times), world)
    info = {"repeats": reps, "block_steps": steps, "block_ms_median": round(med * 1e3, 4),
            "block_ms_min": round(min(times) * 1e3, 4), "block_ms_max": round(max(times) * 1e3, 4),
            "timed_region_s": round(sum(times), 4)}
    del graphs
    return med, clocks, info


# ----------------------------------------------------------------------------
# workloads
# ----------------------------------------------------------------------------

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
    nsets = max(2, math.ceil(min_bytes / set_bytes))
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


def chain_step_launches(M: int) -> int:
    """Kernel launches of one chain step: the grouped quantisation and the grouped decode launch."""
    return 2


def run_chain(args, world, peaks, L2, tokens=(1, 8, 16), steps=None, warmup=None, sampler=None,
              min_region_s=0.05):
    """The 70B-class layer chain as one decode step per call, at each token count."""
    import torch

    import ternary_weight_a8_b200 as tb

    sets, set_bytes = make_layer_sets(CHAIN_70B, seed=1000, min_bytes=3 * L2)
    steps = steps or 100
    warmup = warmup if warmup is not None else 10
    out = {"workload": CHAIN_WORKLOAD, "weight_bytes_per_step": set_bytes,
           "l2": "%d rotating byte-identical weight sets (%.0f MB > 3x L2): inputs larger than L2, every step "
                 "reads its weights from HBM; no flush"
                 % (len(sets), len(sets) * set_bytes / 1e6)}
    for M in tokens:
        xs, ys = make_inputs(CHAIN_70B, M, seed=1000, shared=CHAIN_70B_SHARED_INPUT)
        layer_sets = [[tb.Layer(p, g, x, y) for (p, g), x, y in zip(S, xs, ys)] for S in sets]
        ws = tb.new_workspace(tb.chain_workspace_bytes(layer_sets[0], M))

        def step(i):
            tb.layer_chain(layer_sets[i % len(layer_sets)], workspace=ws)

        secs, clocks, info = timed_graph_run(step, steps, warmup, world, chunk=100,
                                             sampler=sampler if M == tokens[0] else None,
                                             min_region_s=min_region_s, flush=False)
        per_step = secs / steps
        gbs = set_bytes * world / per_step / 1e9
        res = {"GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / world / peaks["hbm"], 2),
               "pct_hbm_nominal_8tbs": round(100 * gbs / world / 8000.0, 2),
               "us_per_step": round(per_step * 1e6, 3), "tokens_per_s": round(M * world / per_step, 1),
               "timing": info, "device_status": tb.device_status(ws),
               "launches_per_step": chain_step_launches(M)}
        if clocks is not None:
            res["clocks"] = clocks
        out["tokens_%d" % M] = res
        del layer_sets
    return out, sets, set_bytes


class _Rt:
    """The few CUDA runtime calls of the end-to-end loop, made directly (cuda-python) so that the
    host's per-step overhead stays below the GPU's step time; torch's equivalents as a fallback."""

    def __init__(self):
        try:
            from cuda.bindings import runtime as rt
        except ImportError:
            rt = None
        self.rt = rt

    def _ok(self, res):
        err = res[0] if isinstance(res, tuple) else res
        if err != self.rt.cudaError_t.cudaSuccess:
            raise RuntimeError("CUDA runtime call failed: %s" % (err,))
        return res[1] if isinstance(res, tuple) and len(res) > 1 else None

    def event(self):
        import torch

        if self.rt is None:
            return torch.cuda.Event()
        return self._ok(self.rt.cudaEventCreateWithFlags(self.rt.cudaEventDisableTiming))

    def record(self, ev, stream):
        if self.rt is None:
            ev.record(stream)
        else:
            self._ok(self.rt.cudaEventRecord(ev, stream.cuda_stream))

    def wait(self, stream, ev):
        if self.rt is None:
            stream.wait_event(ev)
        else:
            self._ok(self.rt.cudaStreamWaitEvent(stream.cuda_stream, ev, 0))

    def sync(self, ev):
        if self.rt is None:
            ev.synchronize()
        else:
            self._ok(self.rt.cudaEventSynchronize(ev))

    def copy(self, dst, src, stream):
        import torch

        if self.rt is None:
            with torch.cuda.stream(stream):
                dst.copy_(src, non_blocking=True)
        else:
            kind = (self.rt.cudaMemcpyKind.cudaMemcpyHostToDevice if dst.is_cuda else
                    self.rt.cudaMemcpyKind.cudaMemcpyDeviceToHost)
            self._ok(self.rt.cudaMemcpyAsync(dst.data_ptr(), src.data_ptr(), dst.numel() * dst.element_size(),
                                             kind, stream.cuda_stream))

    def destroy(self, ev):
        if self.rt is not None:
            self.rt.cudaEventDestroy(ev)


def chain_e2e(sets, set_bytes, M, steps, world, min_region_s=0.05):
    """The chain step end to end through the public API: every step copies its
    inputs from pinned host memory (one H2D copy), runs the chain (a prepared
    ``layer_chain``) and copies its outputs back to pinned host memory (one
    D2H copy).  The host waits for each step's outputs one step later: two
    sets of device and host buffers let it issue step i + 1 before it waits
    for step i, and the copies run on their own streams, ordered by events, so
    that they overlap the neighbouring steps' products — a decode loop that
    overlaps its host work and copies with the GPU."""
    import torch

    import ternary_weight_a8_b200 as tb

    rt = _Rt()
    xs, ys = make_inputs(CHAIN_70B, M, seed=1000, shared=CHAIN_70B_SHARED_INPUT)
    uniq = []
    for x in xs:
        if not any(x is u for u in uniq):
            uniq.append(x)
    x_numel = [x.numel() for x in uniq]
    y_numel = [y.numel() for y in ys]
    x_host = torch.empty(sum(x_numel), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(torch.cat([x.reshape(-1) for x in uniq]).cpu())
    main = torch.cuda.current_stream()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    bufs = []
    for _ in range(2):
        x_dev = torch.empty(sum(x_numel), dtype=torch.bfloat16, device="cuda")
        y_dev = torch.empty(sum(y_numel), dtype=torch.bfloat16, device="cuda")
        x_views = [v.view(x.shape) for v, x in zip(torch.split(x_dev, x_numel), uniq)]
        y_views = [v.view(y.shape) for v, y in zip(torch.split(y_dev, y_numel), ys)]
        x_of = [x_views[next(j for j, u in enumerate(uniq) if u is x)] for x in xs]
        y_host = torch.empty(y_dev.shape, dtype=y_dev.dtype, pin_memory=True)
        layer_sets = [[tb.Layer(p, g, xv, yv) for (p, g), xv, yv in zip(S, x_of, y_views)] for S in sets]
        ev = {k: rt.event() for k in ("in", "used", "out")}
        bufs.append([x_dev, y_dev, y_host, layer_sets, ev])
    ws = tb.new_workspace(tb.chain_workspace_bytes(bufs[0][3][0], M))
    for b in bufs:  # each buffer set's chains marshalled once (the public prepared-chain call)
        b[3] = [tb.prepare_chain(L, workspace=ws, stream=main) for L in b[3]]
        for e in b[4].values():  # every event recorded once, so the first waits pass
            rt.record(e, main)
    torch.cuda.synchronize()

    def issue(i):
        x_dev, y_dev, y_host, plans, ev = bufs[i % 2]
        rt.wait(h2d, ev["used"])            # the step two back has read this x buffer
        rt.copy(x_dev, x_host, h2d)
        rt.record(ev["in"], h2d)
        rt.wait(main, ev["in"])
        rt.wait(main, ev["out"])            # the step two back's outputs are copied out
        plans[i % len(plans)].run()
        rt.record(ev["used"], main)
        rt.wait(d2h, ev["used"])
        rt.copy(y_host, y_dev, d2h)
        rt.record(ev["out"], d2h)

    def run(n):
        issue(0)
        for i in range(1, n):
            issue(i)
            rt.sync(bufs[(i - 1) % 2][4]["out"])  # step i - 1's outputs are on the host
        rt.sync(bufs[(n - 1) % 2][4]["out"])

    run(6)
    t0 = time.perf_counter()
    run(4)
    est = (time.perf_counter() - t0) / 4
    ne = max(steps, int(math.ceil(min_region_s / max(est, 1e-6))))
    ne = int(max_over_ranks(float(ne), world))
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(main)
    h2d.wait_stream(main)  # the first copy comes after the start event
    t0 = time.perf_counter()
    run(ne)
    host_s = time.perf_counter() - t0
    main.wait_stream(d2h)
    e1.record(main)
    torch.cuda.synchronize()
    for b in bufs:
        for e in b[4].values():
            rt.destroy(e)
    e2e_secs = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    return {"value": round(ne * set_bytes * world / e2e_secs / 1e9, 2), "unit": UNIT,
            "h2d_bytes_per_step": x_host.numel() * x_host.element_size(),
            "d2h_bytes_per_step": bufs[0][2].numel() * bufs[0][2].element_size(), "steps": ne,
            "ms_per_step": round(e2e_secs / ne * 1e3, 4), "host_ms_per_step": round(host_s / ne * 1e3, 4),
            "api": "ternary_weight_a8_b200.prepare_chain(...).run() with pinned host x / y: per step one H2D "
                   "copy of the inputs, the chain and one D2H copy of the outputs, the copies on their own "
                   "streams; the host waits for each step's outputs one step later (two buffer sets)"}


def chain_algorithmic_bytes(M: int) -> int:
    """Bytes the chain's decode launch must move: packed weights, int8 codes of
    every distinct input, token scales and code sums, and the bf16 outputs."""
    w = sum(N * K // 4 for K, N in CHAIN_70B)
    x = sum(M * K for (K, N), sh in zip(CHAIN_70B, CHAIN_70B_SHARED_INPUT) if not sh)
    y = sum(M * N * 2 for K, N in CHAIN_70B)
    return w + x + y + 8 * M * 4


def run_decode_2b(args, world, peaks, L2):
    """The 2B-class decode step: both BitLinears of one token in one grouped launch."""
    import ternary_weight_a8_b200 as tb

    sets, set_bytes = make_layer_sets(DECODE_LAYERS, seed=0, min_bytes=4 * L2)
    xs, ys = make_inputs(DECODE_LAYERS, 1, seed=0)
    layer_sets = [[tb.Layer(p, g, x, y) for (p, g), x, y in zip(S, xs, ys)] for S in sets]
    ws = tb.new_workspace(tb.chain_workspace_bytes(layer_sets[0], 1))

    def step(i):
        tb.layer_chain(layer_sets[i % len(layer_sets)], workspace=ws)

    steps = 500
    secs, _, info = timed_graph_run(step, steps, 100, world, chunk=500, flush=False)
    per_step = secs / steps
    x_bytes = sum(K * 2 for K, N in DECODE_LAYERS)
    y_bytes = sum(N * 2 for K, N in DECODE_LAYERS)
    step_bytes = set_bytes + x_bytes + y_bytes + 8 * len(DECODE_LAYERS)
    achieved = step_bytes / per_step / 1e9
    gbs = set_bytes * world / per_step / 1e9
    return {"workload": "decode_2b: BitLinear K=2560->N=6912 and K=2560->N=2560, 1 token, bf16 in/out, one "
                        "grouped launch (activation quantisation inside the decode kernel)",
            "GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / world / peaks["hbm"], 2),
            "us_per_step": round(per_step * 1e6, 3), "tokens_per_s": round(world / per_step, 1),
            "weight_bytes_per_step": set_bytes, "timing": info,
            "l2": "%d rotating byte-identical weight sets (%.0f MB > 4x L2): inputs larger than L2; no flush"
                  % (len(sets), len(sets) * set_bytes / 1e6),
            "roofline": {"bound": "hbm", "kernel": "gemv_group_kernel (the whole step: one launch)",
                         "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                         "frac": round(achieved / peaks["hbm"], 4),
                         "peak_source": peaks["source"] + " HBM copy",
                         "traffic": profiled_traffic("decode_2b", "gemv"),
                         "algorithmic_bytes_per_launch": step_bytes, "launch_us_mean": round(per_step * 1e6, 3)},
            "device_status": tb.device_status(ws)}


def measure_int8_gemm(world, m, n, k, reps=30):
    """cuBLASLt's int8 GEMM (torch._int_mm, int32 accumulation) on [m][k] x [k][n],
    timed with CUDA events after warm-up."""
    import torch

    a = torch.randint(-127, 128, (m, k), dtype=torch.int8, device="cuda")
    b = torch.randint(-127, 128, (n, k), dtype=torch.int8, device="cuda").t()  # column-major operand
    for _ in range(5):
        torch._int_mm(a, b)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(reps):
        torch._int_mm(a, b)
    e1.record()
    torch.cuda.synchronize()
    secs = max_over_ranks(e0.elapsed_time(e1) / 1e3 / reps, world)
    del a, b
    return {"TOPS": round(2.0 * m * n * k / secs / 1e12, 1), "shape": "%dx%dx%d int8 x int8 -> int32" % (m, n, k),
            "library": "cuBLASLt via torch._int_mm", "us_per_call": round(secs * 1e6, 2), "calls": reps}


def measure_int8_peak(world, n=8192, reps=30):
    """Dense int8 tensor-core throughput measured on this GPU: cuBLASLt's int8
    GEMM on n x n x n.  The denominator of the prefill GEMM's roofline."""
    r = measure_int8_gemm(world, n, n, n, reps)
    r["shape"] = "%d^3 int8 x int8 -> int32" % n
    return r


def run_prefill(args, world, peaks, L2):
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    M, K, N = PREFILL["M"], PREFILL["K"], PREFILL["N"]
    sets, set_bytes = make_layer_sets([(K, N)], seed=7, min_bytes=L2)
    xs = []
    for i in range(4):
        bits, _ = synth.activations_bf16(M, K, seed=300 + i)
        xs.append(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
    y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ws = tb.new_workspace(tb.workspace_bytes(M, N, K))

    def step(i):
        packed, gamma = sets[i % len(sets)][0]
        tb.forward(packed, gamma, xs[i % len(xs)], y=y, workspace=ws)

    steps = 100
    secs, _, info = timed_graph_run(step, steps, 20, world, chunk=100)
    ops = 2.0 * M * N * K
    tops = ops * world / (secs / steps) / 1e12
    # Roofline of the GEMM alone: a graph of back-to-back GEMM launches on quantised input.
    xq, sc, rs = tb.quant_act(xs[0])
    gsteps = 100
    gsecs, _, ginfo = timed_graph_run(
        lambda i: tb.forward_quantized(sets[i % len(sets)][0][0], sets[i % len(sets)][0][1], xq, sc, rs, y=y,
                                       workspace=ws), gsteps, 10, world, chunk=100)
    mean_s = gsecs / gsteps
    try:
        int8_peak = measure_int8_peak(world)
        peak_int8, peak_src = int8_peak["TOPS"], "measured int8 dense: " + int8_peak["library"] + ", " + \
            int8_peak["shape"]
    except Exception as e:  # no int8 library GEMM: the nominal ratio over the measured bf16 figure
        int8_peak = {"unavailable": "%s: %s" % (type(e).__name__, e)}
        peak_int8 = peaks["bf16"] * INT8_PER_BF16
        peak_src = "%s bf16 burst x %.0f (nominal int8/bf16 ratio)" % (peaks["source"], INT8_PER_BF16)
    try:  # context: a library int8 GEMM of the same shape on int8 weights (no unpack, 4x the weight bytes)
        same_shape = measure_int8_gemm(world, M, N, K)
    except Exception as e:
        same_shape = {"unavailable": "%s: %s" % (type(e).__name__, e)}
    k_tops = ops / mean_s / 1e12
    status = tb.device_status(ws)
    return {"metric": "prefill int8 TOPS", "value": round(tops, 1), "unit": "TOPS",
            "workload": "prefill_2b: BitLinear K=2560->N=6912 over 2048 tokens (activation quantisation + "
                        "tcgen05 GEMM), bf16 in/out",
            "us_per_step": round(secs / steps * 1e6, 3), "tokens_per_s": round(M * world / (secs / steps), 0),
            "pct_int8_nominal_4500": round(100 * tops / world / 4500.0, 2), "timing": info,
            "int8_peak": int8_peak, "library_int8_same_shape": same_shape,
            "roofline": {"bound": "tensor", "kernel": "gemm_kernel (tcgen05 kind::i8), alone",
                         "achieved": round(k_tops, 1), "peak": peak_int8, "unit": "TOPS",
                         "frac": round(k_tops / peak_int8, 4),
                         "peak_source": peak_src,
                         "frac_of_2x_bf16": round(k_tops / (peaks["bf16"] * INT8_PER_BF16), 4),
                         "launch_us_mean": round(mean_s * 1e6, 3), "timing": ginfo,
                         "traffic": profiled_traffic("prefill_2b", "gemm"),
                         "algorithmic_ops_per_launch": ops,
                         "algorithmic_bytes_per_launch": M * K + N * K // 4 + M * N * 2 + 8 * M},
            "device_status": status}


DECODE_3B = [(3200, 8640), (8640, 3200)]  # (K in, N out)
DECODE_3B_TOKENS = (1, 2, 4, 8, 16)


def run_chain_tensor_core_form(args, world, peaks, L2, tokens=(8, 16)):
    """The same chain through the decode product's tensor-core form (chosen
    only on request), for comparison with the default CUDA-core form."""
    import ternary_weight_a8_b200 as tb

    tb.set_decode_form(tb.DECODE_FORM_TENSOR_CORES)
    try:
        res, _, _ = run_chain(args, world, peaks, L2, tokens=tokens, steps=20, warmup=5)
    finally:
        tb.set_decode_form(tb.DECODE_FORM_AUTO)
    res = {k: v for k, v in res.items() if k != "l2"}
    res["form"] = "tcgen05.mma kind::i8, unpacked codes in tensor memory (bitlinear_set_decode_form 2)"
    return res


def run_decode_3b(args, world, peaks, L2, tokens=None):
    """The 3B-class decode sweep: one BitLinear per step through the public
    single-layer call (quantisation and product), 1 to 16 tokens."""
    import ternary_weight_a8_b200 as tb

    res = {"workload": "decode_3b: BitLinear K=3200->N=8640 and K=8640->N=3200 alone, bf16 in/out, "
                       "1/2/4/8/16 tokens, one forward call per step"}
    for li, (K, N) in enumerate(DECODE_3B):
        sets, set_bytes = make_layer_sets([(K, N)], seed=500 + li, min_bytes=4 * L2)
        for M in (tokens or DECODE_3B_TOKENS):
            xs, ys = make_inputs([(K, N)], M, seed=500 + li)
            x, y = xs[0], ys[0]
            ws = tb.new_workspace(tb.workspace_bytes(M, N, K))

            def step(i):
                packed, gamma = sets[i % len(sets)][0]
                tb.forward(packed, gamma, x, y=y, workspace=ws)

            steps = 500
            secs, _, info = timed_graph_run(step, steps, 100, world, chunk=500, min_region_s=0.03, flush=False)
            per = secs / steps
            gbs = set_bytes * world / per / 1e9
            res["k%d_n%d_m%d" % (K, N, M)] = {
                "GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / world / peaks["hbm"], 2),
                "us_per_call": round(per * 1e6, 3), "tokens_per_s": round(M * world / per, 1),
                "repeats": info["repeats"], "device_status": tb.device_status(ws)}
        del sets
    return res


def run_ffn(args, world, peaks, L2, tokens=(1, 8, 2048)):
    """The FFN's gate and up BitLinears with the gated activation and the
    quantisation of h: one call (gate_up_glu) against the same work as the
    chain of the two products followed by the gated-activation kernel."""
    import torch

    import synth
    import ternary_weight_a8_b200 as tb

    out = {}
    # decode sizes at the 70B FFN width, many tokens at the 2B prefill shape
    for M, K, N in ((t, 8192, 28672) if t <= 16 else (t, 2560, 6912) for t in tokens):
        wsets, wbytes = make_layer_sets([(K, N), (K, N)], seed=1100, min_bytes=3 * L2)
        x = torch.from_numpy(synth.activations_bf16(M, K, seed=1101)[0].view("int16")).cuda().view(torch.bfloat16)
        yg = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        yu = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        xq = torch.empty((M, N), dtype=torch.int8, device="cuda")
        sc = torch.empty(M, dtype=torch.float32, device="cuda")
        rs = torch.empty(M, dtype=torch.int32, device="cuda")
        ws_f = tb.new_workspace(tb.gate_up_glu_workspace_bytes(M, N, K))
        lsets = [[tb.Layer(p, g, x, yg if j == 0 else yu) for j, (p, g) in enumerate(S)] for S in wsets]
        ws_c = tb.new_workspace(tb.chain_workspace_bytes(lsets[0], M))

        def fused(i):
            (pg, gg), (pu, gu) = wsets[i % len(wsets)]
            tb.gate_up_glu(pg, gg, pu, gu, x, tb.GLU_RELU2, xq=xq, scale=sc, rowsum=rs, workspace=ws_f)

        def unfused(i):
            tb.layer_chain(lsets[i % len(lsets)], workspace=ws_c)
            tb.glu_quant(yg, yu, tb.GLU_RELU2, None, xq, sc, rs)

        steps = 20
        res = {"weight_bytes": wbytes}
        for name, fn in (("fused_one_call", fused), ("chain_then_glu_quant", unfused)):
            secs, _, _ = timed_graph_run(fn, steps, 5, world, chunk=steps, min_region_s=0.05)
            us = secs / steps * 1e6
            res[name] = {"us": round(us, 3)}
            if M <= 16:
                gbs = wbytes / (us * 1e-6) / 1e9
                res[name].update({"GB/s": round(gbs, 1), "pct_hbm_measured": round(100 * gbs / peaks["hbm"], 2)})
            else:
                tops = 2 * 2.0 * M * N * K / (us * 1e-6) / 1e12
                res[name].update({"TOPS": round(tops, 1)})
        res["launches"] = {"fused_one_call": 2 if M <= 8 else 3, "chain_then_glu_quant": 3 if M <= 16 else 4}
        res["device_status"] = tb.device_status(ws_f)
        out["ffn_gate_up_glu_%dx%dx%d" % (M, K, N)] = res
        del wsets, lsets
    return out


def run_next(args, world, peaks, L2):
    """The rows beyond the forward: fused RMSNorm + quantisation, gated activation +
    quantisation, the lookup-table decode product and the straight-through backward."""
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
        steps = 200
        secs, _, _ = timed_graph_run(lambda i: tb.rmsnorm_quant(xs[i % len(xs)], g, 1e-6, None, xq, sc, rs),
                                     steps, 20, world, chunk=200, min_region_s=0.02)
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
        usecs, _, _ = timed_graph_run(unfused, steps, 20, world, chunk=200, min_region_s=0.02)
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
        steps = 200
        secs, _, _ = timed_graph_run(lambda i: tb.glu_quant(gs[i % len(gs)], us[i % len(us)], tb.GLU_RELU2, None,
                                                            xq, sc, rs), steps, 20, world, chunk=200,
                                     min_region_s=0.02)
        nb = M * N * 5 + M * 8
        gbs = nb / (secs / steps) / 1e9
        res = {"us": round(secs / steps * 1e6, 3), "GB/s": round(gbs, 1),
               "pct_hbm_measured": round(100 * gbs / peaks["hbm"], 2), "bytes_per_call": nb, "act": "relu2"}

        def unfused(i):
            g, u = gs[i % len(gs)], us[i % len(us)]
            h = (torch.relu(g.float()).square() * u.float()).to(torch.bfloat16)
            tb.quant_act(h, xq, sc, rs)
        usecs, _, _ = timed_graph_run(unfused, steps, 20, world, chunk=200, min_region_s=0.02)
        res["unfused_torch_glu_then_quant_us"] = round(usecs / steps * 1e6, 3)
        out["glu_quant_%dx%d" % (M, N)] = res
    out.update(run_ffn(args, world, peaks, L2))
    # The lookup-table decode product against the tensor-core decode kernel, same codes, one token.
    for K, N in ((2560, 6912), (8192, 10240)):
        sets, set_bytes = make_layer_sets([(K, N)], seed=800, min_bytes=4 * L2)
        bits, _ = synth.activations_bf16(1, K, seed=801)
        xq, sc, rs = tb.quant_act(torch.from_numpy(bits.view("int16")).cuda().view(torch.bfloat16))
        y = torch.empty((1, N), dtype=torch.bfloat16, device="cuda")
        ws = tb.new_workspace(tb.workspace_bytes(1, N, K))
        steps = 200
        res = {"weight_bytes": set_bytes}
        for name, fn in (("lut", lambda i: tb.forward_lut(sets[i % len(sets)][0][0], sets[i % len(sets)][0][1], xq,
                                                           sc, rs, y=y)),
                         ("decode_kernel", lambda i: tb.forward_quantized(sets[i % len(sets)][0][0],
                                                                             sets[i % len(sets)][0][1], xq, sc, rs,
                                                                             y=y, workspace=ws))):
            secs, _, _ = timed_graph_run(fn, steps, 20, world, chunk=200, min_region_s=0.02)
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
    steps = 20
    secs, _, _ = timed_graph_run(lambda i: tb.ste_backward(packed, gamma, K, dy, xq, sc, dx=dx, dw=dw, workspace=ws),
                                 steps, 5, world, chunk=20, min_region_s=0.02)
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
# our arm
# ----------------------------------------------------------------------------

def run_ours(args, world, rank, local):
    import torch

    torch.cuda.set_device(local)
    peaks = load_peaks()
    L2 = l2_bytes()

    # ---- headline: the 70B-class chain at one token ----
    sampler = ClockSampler(torch.cuda.current_device())
    tokens = (1,) if args.no_extras else (1, 8, 16)
    chain, sets, set_bytes = run_chain(args, world, peaks, L2, tokens=tokens, steps=args.steps,
                                       warmup=args.warmup, sampler=sampler, min_region_s=0.5)
    head = chain["tokens_1"]
    per_step = head["us_per_step"] / 1e6
    value = set_bytes * world / per_step / 1e9
    clocks = head.pop("clocks", None)
    reps = head["timing"]["repeats"]
    launches_per_step = head["launches_per_step"]
    # Roofline of the dominant kernel.  The step is the grouped quantisation
    # launch and the grouped decode launch, which starts streaming weights while
    # the quantisation runs; the decode launch's duration is taken as the whole
    # step's (an upper bound, so `achieved` is a lower bound).
    alg = chain_algorithmic_bytes(1)
    achieved = alg / per_step / 1e9
    roofline = {"bound": "hbm", "kernel": "gemv_group_kernel (70B chain, 1 token: all five BitLinears in one "
                                          "launch)",
                "achieved": round(achieved, 1), "peak": peaks["hbm"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm"], 4), "peak_source": peaks["source"] + " HBM copy",
                "traffic": profiled_traffic("chain_70b_m1", "gemv"), "algorithmic_bytes_per_launch": alg,
                "launch_us_mean": round(per_step * 1e6, 3),
                "launch_time_basis": "whole step (quantisation launch + decode launch), CUDA events"}
    e2e = chain_e2e(sets, set_bytes, 1, args.steps, world)
    del sets

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(per_step * 1e3, 6), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic (seeded N(0,0.02) latent weights packed to 2-bit ternary, N(0,1) bf16 activations "
                "with 1% x20 outlier channels)",
        "config": {"workload": CHAIN_WORKLOAD, "tokens": 1, "layers_k_n": CHAIN_70B,
                   "weight_bytes_per_step": set_bytes, "l2": chain["l2"],
                   "timing": "the %d steps replayed as CUDA graphs; the same graphs warmed first; the block of %d "
                             "steps timed %d times with CUDA events, blocks back to back (weights rotate over "
                             "more than L2: no flush); median block / %d"
                             % (args.steps, args.steps, reps, args.steps),
                   "parallelism": "replicas x%d" % world},
        "pct_hbm_measured": round(100 * value / world / peaks["hbm"], 2),
        "pct_hbm_nominal_8tbs": round(100 * value / world / 8000.0, 2),
        "roofline": roofline, "e2e": e2e,
        "gpu_launches": reps * args.steps * launches_per_step,
        "gpu_launches_per_step": launches_per_step, "clocks": clocks, "timing": head["timing"],
        "device_status": head["device_status"],
    }
    if not args.no_extras:
        result["prefill"] = run_prefill(args, world, peaks, L2)
        result["decode"] = {"chain_70b": {k: v for k, v in chain.items() if k != "l2"},
                            "chain_70b_tensor_core_form": run_chain_tensor_core_form(args, world, peaks, L2),
                            "decode_2b": run_decode_2b(args, world, peaks, L2),
                            "decode_3b": run_decode_3b(args, world, peaks, L2)}
        result["pack"] = run_pack(world)
        result["next"] = run_next(args, world, peaks, L2)
    return result


# ----------------------------------------------------------------------------
# the oracle (CPU) on the same workload
# ----------------------------------------------------------------------------

def oracle_chain_layers(rows_div=CPU_SAMPLE_ROWS):
    """The chain's layers as the oracle takes them, on a sample: the first
    ceil(N / rows_div) output rows of every layer (all of K), packed with the
    sample's own gamma.  Returns ([(packed, gamma, K, x)], packed bytes)."""
    import oracle
    import synth

    layers = []
    xf_prev = None
    for i, ((K, N), sh) in enumerate(zip(CHAIN_70B, CHAIN_70B_SHARED_INPUT)):
        n = -(-N // rows_div)
        W = synth.latent_weights(n, K, seed=1000 + i)  # the first n rows of the layer's weights
        packed, gamma, _ = oracle.pack_weights(W)
        del W
        xf = xf_prev if sh else synth.activations_bf16(1, K, seed=1000 + 100 + i)[1]
        xf_prev = xf
        layers.append((packed, gamma, K, xf))
    return layers, sum(p.size for p, *_ in layers)


def oracle_steps(layers, reps):
    """reps chain steps of the oracle over `layers` (any subset of rows); returns seconds."""
    import oracle

    t0 = time.perf_counter()
    for _ in range(reps):
        for packed, gamma, K, xf in layers:
            T, ok = oracle.unpack(packed, K)
            acc, y, *_ = oracle.forward(T, gamma, xf)
            oracle.round_bf16(y)
    return time.perf_counter() - t0


def row_slices(n_rows, parts):
    """Contiguous, disjoint [n0, n1) slices of n_rows rows, one per part, sizes within one."""
    return [(n_rows * c // parts, n_rows * (c + 1) // parts) for c in range(parts)]


def _oracle_rows_worker(task):
    layers, reps = task
    oracle_steps(layers, 1)  # load the oracle library before timing
    return oracle_steps(layers, reps)


CPU_SAMPLE_TEXT = ("the 70B chain at one token on the first 1/%d of every layer's output rows (all of K; gamma "
                   "of the sample), unpack + quantise + accumulate + dequantise + bf16 round" % CPU_SAMPLE_ROWS)


def cpu_baseline(target_s=10.0):
    layers, set_bytes = oracle_chain_layers()
    one = oracle_steps(layers, 1)
    reps = max(1, int(target_s / max(one, 1e-6)))
    secs = oracle_steps(layers, reps)
    return {"value": round(reps * set_bytes / secs / 1e9, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": "%d steps of %s, one host core, %.1f s" % (reps, CPU_SAMPLE_TEXT, secs)}


def cpu_baseline_all_cores(cpu_work_s=20.0):
    """The same oracle steps spread over the host's cores: each process takes a
    contiguous slice of every layer's output rows (rows are independent, so the
    slices together compute the whole step).  The pool is started with
    `spawn`, so no process inherits the CUDA context."""
    import multiprocessing

    layers, set_bytes = oracle_chain_layers()
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    cores = max(1, min(cores, 128))
    one = oracle_steps(layers, 1)
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
            "sample": "%d steps of %s, each of %d processes taking 1/%d of every layer's rows, %.2f s wall"
                      % (reps, CPU_SAMPLE_TEXT, cores, cores, secs)}


def run_reference(args, world, rank):
    """The reference arm: the CPU oracle, as it stands, on one host core, on
    this arm's workload (a row sample of every layer per step), exactly
    --warmup untimed and --steps timed steps."""
    if rank != 0:
        return None
    layers, set_bytes = oracle_chain_layers()
    steps = max(1, args.steps)
    warm = max(0, args.warmup)
    oracle_steps(layers, warm)
    secs = oracle_steps(layers, steps)
    value = steps * set_bytes / secs / 1e9
    sample = "%d steps of %s, one host core" % (steps, CPU_SAMPLE_TEXT)
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": steps, "warmup": warm, "ms_per_step": round(secs / steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": CHAIN_WORKLOAD, "tokens": 1, "layers_k_n": CHAIN_70B,
                       "sample_rows": "first 1/%d of every layer's output rows" % CPU_SAMPLE_ROWS,
                       "weight_bytes_per_step": set_bytes},
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
        peaks, L2 = load_peaks(), l2_bytes()
        tokens = tuple(int(t) for t in args.tokens.split(",")) if args.tokens else None
        if args.only == "chain70b":
            res, _, _ = run_chain(args, world, peaks, L2, steps=args.steps, warmup=args.warmup,
                                  **({"tokens": tokens} if tokens else {}))
        elif args.only == "ffn":
            res = run_ffn(args, world, peaks, L2, **({"tokens": tokens} if tokens else {}))
        elif args.only == "decode3b":
            res = run_decode_3b(args, world, peaks, L2, tokens=tokens)
        else:
            fn = {"decode2b": run_decode_2b, "prefill": run_prefill, "next": run_next}[args.only]
            res = fn(args, world, peaks, L2)
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
