#!/usr/bin/env python
"""Benchmark of the B200 W4A16 group-128 linear layer.

Default workload (one "step"): a LLaMA-7B-shaped decode step at N = 1 token --
32 layers x {fused QKV 12288x4096, O 4096x4096, fused gate/up 22016x4096,
down 4096x11008}, 128 distinct packed weight sets resident in HBM (3.37 GB, far
beyond the 126 MB L2, so no flush is needed), each projection one
w4a16_gemm_ws call on the automatic path (the decode kernel: weights streamed
from HBM into registers, warp-level MMAs on the exact dequant, the first
weight groups requested before the grid dependency wait under programmatic
dependent launch), the step captured once in a CUDA graph.  The metric is algorithmic HBM bytes per second (packed int4 weights +
2.5 B per group of metadata + fp16 X and Y), reported against the measured HBM
copy bandwidth.  `e2e` is the same step with every call's X copied in from
pinned host memory and every Y copied back each step, pipelined per layer
group on copy streams inside the step's graph (the serialised form beside
it).  The same JSON line carries, each with its own clock summary and median
/ p10 / p90 over its repeats: every projection alone, the fused-QKV N sweep
on every kernel, the LLaMA-3-8B batched-decode shapes, the fused forms and
secondary kernels, the two prefill GEMMs (TFLOP/s; last, since their power
draw slows the memory-bound points timed after them), and the CPU oracle at
all cores and at one thread.  Each secondary graph replays for 25 ms (250 ms
before the LLaMA-3 leg) before it is timed.

One JSON line on stdout (rank 0).  Multi-GPU runs (torchrun) are replicas:
every rank runs its own copy of the step (weak scaling), no collective on the
data path; time is the max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
    python bench.py --workload qkv_n1|prefill|sweep|quantize|qkv_fused|qkv_norm|gate_up_fused|add_rmsnorm ...
                                                          (secondary workloads)
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "W4A16 g128 GEMV HBM GB/s & GEMM TFLOPS on 1 B200, % of roofline"
GROUP = 128
LLAMA7B_LAYER = [("qkv", 12288, 4096), ("o", 4096, 4096), ("gate_up", 22016, 4096),
                 ("down", 4096, 11008)]
N_LAYERS = 32
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one decode
# launch of the decode kernel on the fused QKV shape at N = 1, from an ncu
# capture of this repository's kernel; it holds only while the kernel source
# is the one captured (sha256 prefix of csrc/w4a16_gemv.cu), and the bench
# reports null otherwise.
DECODE_TRAFFIC = {"src_sha256_prefix": "a308e7b7e1ad5ecb", "qkv_dram_bytes": 26184704, "qkv_alg_bytes": 26181632}
NOMINAL_DENSE_FP16_TFLOPS = 2250.0   # B200 dense fp16/bf16 tensor rate, NVIDIA's figure


def alg_bytes(M, K, N):
    """Algorithmic bytes of one call: int4 weights, 2.5 B/group metadata, X, Y."""
    return M * K // 2 + (M * K // GROUP) * 5 // 2 + 2 * K * N + 2 * M * N


def alg_flops(M, K, N):
    return 2 * M * N * K


def decode_traffic_per_launch(alg_bytes_per_launch):
    """ncu DRAM bytes per decode launch, scaled from the QKV capture by the
    algorithmic bytes (every shape streams its weights once), or None when
    the kernel source changed since the capture."""
    import hashlib

    src = os.path.join(ROOT, "gemm_w4a16_b200", "csrc", "w4a16_gemv.cu")
    try:
        h = hashlib.sha256(open(src, "rb").read()).hexdigest()
    except OSError:
        return None
    pre = DECODE_TRAFFIC["src_sha256_prefix"]
    if not pre or not h.startswith(pre):
        return None
    return DECODE_TRAFFIC["qkv_dram_bytes"] / DECODE_TRAFFIC["qkv_alg_bytes"] * alg_bytes_per_launch


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------ distributed --

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def dist_init(backend):
    import datetime

    import torch.distributed as dist

    if not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(value: float, dist=None, device=None) -> float:
    """Max of a float over all ranks (identity without a process group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, dist=None, device=None) -> float:
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    import torch

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ----------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi clock/throttle samples while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        rows = []
        for ts, line in self.lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                rows.append((ts, float(parts[0]), float(parts[1]), parts[3:]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        inside = [r for r in rows if t0 is None or (t0 <= r[0] <= t1)] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in inside:
            for name, v in zip(names, r[3][1:]):
                if v.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside),
                "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside)}


# ---------------------------------------------------------- decode step ----

def build_decode_step(device, seed=0, n_layers=N_LAYERS):
    """128 distinct packed weight sets plus per-call X and Y (flat buffers)."""
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    calls = []
    x_total = sum(K for _, _, K in LLAMA7B_LAYER) * n_layers
    y_total = sum(M for _, M, _ in LLAMA7B_LAYER) * n_layers
    x_flat = torch.empty(x_total, dtype=torch.float16, device=device)
    y_flat = torch.empty(y_total, dtype=torch.float16, device=device)
    xo = yo = 0
    for layer in range(n_layers):
        for name, M, K in LLAMA7B_LAYER:
            q, z, s = synth.make_weights_torch(M, K, GROUP, gen, device)
            w = w4a16.pack(q, s, z)
            del q, z, s
            x = x_flat[xo:xo + K].view(1, K)
            x.copy_(synth.make_activations_torch(1, K, gen, device))
            y = y_flat[yo:yo + M].view(1, M)
            xo += K
            yo += M
            calls.append((name, w, x, y))
    torch.cuda.synchronize(device)
    return calls, x_flat, y_flat


def run_calls(calls, path=0):
    from gemm_w4a16_b200 import w4a16

    for _, w, x, y in calls:
        if path:
            w4a16.gemm_ex(w, x, Y=y, path=path)
        else:
            w4a16.gemm(w, x, Y=y)


def capture_e2e(calls, ws, flags, x_flat, y_flat, x_host, y_host, device, sizes=None):
    """One CUDA graph of the decode step with its host traffic pipelined
    against the kernels: the calls in consecutive groups of `sizes` calls
    (default: the first layer, 15 layers, 15 layers, the last layer, so that
    only one layer's X waits before the first kernel and one layer's Y
    after the last), every group's X copied in from pinned host memory on
    an H2D stream (all groups queued at once, each group's calls waiting for
    its own copy) and every group's Y copied out on a D2H stream as soon as
    the group's calls are done, overlapping the next group's kernels; both
    streams join the replay stream before the graph ends."""
    import torch

    if sizes is None:
        per_layer = len(LLAMA7B_LAYER)
        mid = len(calls) // per_layer - 2
        if mid < 2:
            sizes = [len(calls)]
        else:
            sizes = [per_layer, per_layer * (mid // 2), per_layer * (mid - mid // 2), per_layer]
    assert sum(sizes) == len(calls)
    groups = []
    xo = yo = 0
    c0 = 0
    for size in sizes:
        cs = calls[c0:c0 + size]
        c0 += size
        xk = sum(w.K for _, w, _, _ in cs)
        ym = sum(w.M for _, w, _, _ in cs)
        groups.append((xo, xo + xk, yo, yo + ym, cs))
        xo += xk
        yo += ym
    assert xo == x_flat.numel() and yo == y_flat.numel()
    h2d = torch.cuda.Stream(device=device)
    d2h = torch.cuda.Stream(device=device)

    def step():
        s = torch.cuda.current_stream(device)
        h2d.wait_stream(s)
        d2h.wait_stream(s)
        ready = []
        with torch.cuda.stream(h2d):
            for x0, x1, _, _, _ in groups:
                x_flat[x0:x1].copy_(x_host[x0:x1], non_blocking=True)
                e = torch.cuda.Event()
                e.record(h2d)
                ready.append(e)
        for (x0, x1, y0, y1, cs), e in zip(groups, ready):
            s.wait_event(e)
            run_calls_ws(cs, ws, flags)
            done = torch.cuda.Event()
            done.record(s)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                y_host[y0:y1].copy_(y_flat[y0:y1], non_blocking=True)
        s.wait_stream(h2d)
        s.wait_stream(d2h)

    return capture(step, device)


def run_calls_ws(calls, ws, flags=0, path=0):
    """Each call through w4a16_gemm_ws on one shared workspace."""
    from gemm_w4a16_b200 import w4a16

    for _, w, x, y in calls:
        w4a16.gemm_ws(w, x, Y=y, path=path, workspace=ws, flags=flags)


def capture(fn, device):
    import torch

    s = torch.cuda.Stream(device=device)
    s.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(s):
        fn()            # warm the launch path once outside capture
    torch.cuda.current_stream(device).wait_stream(s)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize(device)
    return g


def time_steps(g, steps, warmup, device, pre=None, post=None):
    """Replays of graph g: W untimed, then exactly `steps` timed with a CUDA
    event recorded on the replay stream before the first and after every
    replay.  Returns (total ms of the bracketed region, per-replay ms)."""
    import torch

    stream = torch.cuda.current_stream(device)
    for _ in range(warmup):
        if pre:
            pre()
        g.replay()
        if post:
            post()
    torch.cuda.synchronize(device)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    ev[0].record(stream)
    for i in range(steps):
        if pre:
            pre()
        g.replay()
        if post:
            post()
        ev[i + 1].record(stream)
    torch.cuda.synchronize(device)
    per = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    return ev[0].elapsed_time(ev[steps]), per


def settle(g, device, ms=25.0):
    """Replay g for about `ms` milliseconds before a measurement, so that a
    leg that follows a power-hungry one starts at its steady clocks."""
    import torch

    t_end = time.time() + ms * 1e-3
    while time.time() < t_end:
        for _ in range(4):
            g.replay()
        torch.cuda.synchronize(device)


def time_graph(g, steps, warmup, device, pre=None, post=None):
    """Mean ms per replay of graph g over `steps` timed replays."""
    total, _ = time_steps(g, steps, warmup, device, pre, post)
    return total / steps


def pct(values, scale=1.0):
    """median, p10 and p90 of a list (times scale)."""
    import numpy as np

    v = np.asarray(values, dtype=np.float64) * scale
    return {"median": float(np.median(v)), "p10": float(np.percentile(v, 10)),
            "p90": float(np.percentile(v, 90)), "n": int(v.size)}


# ------------------------------------------------------- CPU (oracle) leg --

def _oracle_layer(rows=None, seed=0):
    """Canonical host arrays of one synthetic layer (optionally its first rows)."""
    import numpy as np

    from gemm_w4a16_b200 import synth

    rng = np.random.default_rng(seed)
    layer = []
    for name, M, K in LLAMA7B_LAYER:
        m = M if rows is None else min(rows, M)
        q, z, s = synth.draw_weights(rng, m, K, GROUP)
        x, _ = synth.draw_activations(rng, 1, K)
        layer.append((m, K, q, z, s, x))
    return layer


def _oracle_pass(layer):
    import oracle

    nbytes = 0
    for M, K, q, z, s, x in layer:
        oracle.gemm(q, z, s, x, GROUP)
        nbytes += alg_bytes(M, K, 1)
    return nbytes


def oracle_decode_sample(target_s=12.0, max_layers=N_LAYERS, seed=0, threads=None, rows=None):
    """Time the CPU oracle, as it stands, over synthetic layers of the decode
    step (whole layers, or their first `rows` output rows) until about
    target_s seconds of work, on `threads` host threads (default: all);
    returns GB/s of algorithmic bytes."""
    import oracle

    oracle.set_threads(threads or os.cpu_count() or 1)
    layer = _oracle_layer(rows=rows, seed=seed)
    nbytes = 0
    layers = 0
    t0 = time.perf_counter()
    while layers < max_layers:
        nbytes += _oracle_pass(layer)
        layers += 1
        if time.perf_counter() - t0 >= target_s:
            break
    dt = time.perf_counter() - t0
    what = "full layer(s)" if rows is None else f"layer(s) of the first {rows} rows"
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": oracle.get_threads(),
            "kind": "oracle",
            "sample": f"{layers} {what} of the 4 LLaMA-7B projections at N=1 "
                      f"({layers * 4} oracle products, {nbytes / 1e6:.0f} MB algorithmic, "
                      f"{dt:.1f} s)"}


REF_ROWS = 128   # rows of each projection per reference-arm step


def main_reference(args):
    """The reference arm: the CPU oracle, as it stands, on the host cores.
    One step = the first REF_ROWS output rows of each of the four projections
    of one layer at N = 1 (a bounded sample of the decode step)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle

    oracle.set_threads(os.cpu_count() or 1)
    layer = _oracle_layer(rows=REF_ROWS)
    for _ in range(args.warmup):
        _oracle_pass(layer)
    t0 = time.perf_counter()
    nbytes = 0
    for _ in range(args.steps):
        nbytes += _oracle_pass(layer)
    dt = time.perf_counter() - t0
    value = nbytes / dt / 1e9
    sample = (f"per step: first {REF_ROWS} rows of each of the 4 LLaMA-7B projections "
              f"at N=1 ({nbytes // max(args.steps, 1)} algorithmic bytes)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / max(args.steps, 1), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "llama7b_decode_step_n1", "group": GROUP,
                       "step": sample},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": oracle.get_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------- our path ----

def main_ours(args):
    import torch

    from gemm_w4a16_b200 import build as lib_build
    from gemm_w4a16_b200 import w4a16

    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}), flush=True)
        return 1
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = dist_init("nccl") if world > 1 else None
    if rank == 0:
        lib_build.build(debug=False)
    if dist is not None:
        dist.barrier()
    w4a16.lib()
    peaks, peaks_src = load_peaks()

    if args.workload == "sweep":
        return sweep(args, device)
    if args.workload == "qkv_n1":
        return single_shape(args, device, 12288, 4096, 1)
    if args.workload == "prefill":
        return single_shape(args, device, 12288, 4096, 4096)
    if args.workload == "shape":
        return single_shape(args, device, args.M, args.K, args.N, args.path)
    if args.workload == "quantize":
        return quantize_workload(args, device, peaks)
    if args.workload == "qkv_norm":
        return qkv_norm_workload(args, device, peaks)
    if args.workload == "qkv_fused":
        return qkv_fused_workload(args, device, peaks)
    if args.workload == "gate_up_fused":
        return gate_up_fused_workload(args, device, peaks)
    if args.workload == "add_rmsnorm":
        return add_rmsnorm_workload(args, device, peaks)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)

    calls, x_flat, y_flat = build_decode_step(device, seed=1000 + rank)
    step_bytes = sum(alg_bytes(w.M, w.K, 1) for _, w, _, _ in calls)
    ws = w4a16.Workspace(device, max(w4a16.workspace_size(w.M, w.K, 1) for _, w, _, _ in calls))
    flags = w4a16.FLAG_EARLY_WEIGHTS
    launches_per_step = len(calls)      # one kernel launch per projection at N = 1
    g = capture(lambda: run_calls_ws(calls, ws, flags), device)

    # Device-resident timing (the headline value).
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    t_wall0 = time.time()
    total_ms, per_step = time_steps(g, args.steps, args.warmup, device)
    t_wall1 = time.time()
    ms = total_ms / args.steps
    ms_max = max_over_ranks(ms, dist, device)
    total_bytes = sum_over_ranks(step_bytes * args.steps, dist, device)
    value = total_bytes / (ms_max * args.steps * 1e-3) / 1e9
    clocks = sampler.summary(t_wall0, t_wall1)

    per_shape = per_shape_measure(calls, ws, flags, device, peaks, sampler)

    # End to end: every step copies every call's X in from pinned host
    # memory and every Y back out, inside the event-timed region: pipelined
    # per layer group against the kernels in one graph, and also (reported
    # beside it) serialised around the step's graph.
    x_host = torch.empty(x_flat.shape, dtype=x_flat.dtype, pin_memory=True)
    y_host = torch.empty(y_flat.shape, dtype=y_flat.dtype, pin_memory=True)
    x_host.copy_(x_flat)
    e2e_steps = max(args.steps // 2, 1)
    ms_e2e_serial = time_graph(g, e2e_steps, args.warmup, device,
                               pre=lambda: x_flat.copy_(x_host, non_blocking=True),
                               post=lambda: y_host.copy_(y_flat, non_blocking=True))
    g_e2e = capture_e2e(calls, ws, flags, x_flat, y_flat, x_host, y_host, device)
    ms_e2e = time_graph(g_e2e, e2e_steps, args.warmup, device)
    del g_e2e
    ms_e2e_max = max_over_ranks(ms_e2e, dist, device)
    ms_e2e_serial_max = max_over_ranks(ms_e2e_serial, dist, device)
    e2e_value = sum_over_ranks(step_bytes, dist, device) / (ms_e2e_max * 1e-3) / 1e9
    e2e_serial_value = sum_over_ranks(step_bytes, dist, device) / (ms_e2e_serial_max * 1e-3) / 1e9
    del g, calls, x_flat, y_flat
    torch.cuda.empty_cache()

    extra = {}
    if not args.no_extra:
        # The compute-bound prefill leg last: its power draw slows the first
        # memory-bound points measured after it (QKV N = 1: 9.2 to 11.4
        # against 8.7 us) for longer than a short settling replay.
        extra["n_sweep"] = n_sweep_measure(device, peaks, sampler)
        extra["llama3"] = llama3_measure(device, peaks, sampler)
        extra["fused"] = fused_measure(device, peaks, sampler)
        extra["prefill"] = prefill_measure(device, peaks, sampler)

    res = None
    if rank == 0 and world == 1 and not args.no_cpu:
        res = oracle_decode_sample(target_s=args.cpu_seconds)
        res["single_thread"] = oracle_decode_sample(target_s=args.cpu_seconds, threads=1, rows=512)
    sampler.stop()

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    achieved = step_bytes / (ms * 1e-3) / 1e9
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "ms_per_step_pct": pct(per_step),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "accumulate": "f32", "data": "synthetic",
        "config": {"workload": "llama7b_decode_step_n1",
                   "description": "32 layers x {qkv 12288x4096, o 4096x4096, gate_up 22016x4096, "
                                  "down 4096x11008}, N=1, group 128, 128 distinct weight sets",
                   "bytes_per_step": step_bytes, "global_batch": 1, "seq_len": 1,
                   "l2": "inputs 3.37 GB per step > 126 MB L2 (no flush needed)",
                   "launch": "cuda_graph, programmatic dependent launch (early weights)",
                   "api": "w4a16_gemm_ws (auto path: decode kernel gemv_kernel, early weights)",
                   "parallelism": f"replicas{world}"},
        "roofline": {"bound": "hbm", "kernel": "gemv_kernel", "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks_src,
                     "traffic": decode_traffic_per_launch(step_bytes / launches_per_step),
                     "traffic_note": "DRAM bytes per launch, scaled from the QKV ncu capture"},
        "per_shape": per_shape,
        "e2e": {"value": e2e_value, "unit": "GB/s",
                "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 2), "ms_per_step": ms_e2e_max,
                "api": "w4a16_gemm_ws (128 calls captured in a CUDA graph) + pinned H2D/D2H by torch copy_, "
                       "per layer group (1, 15, 15, 1 layers) on copy streams overlapping the kernels",
                "serialised": {"value": e2e_serial_value,
                               "ms_per_step": ms_e2e_serial_max,
                               "api": "all X in, the step's graph, all Y out, on one stream"}},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    line.update(extra)
    if res:
        line["cpu_baseline"] = res
    print(json.dumps(line), flush=True)
    return 0


def per_shape_measure(calls, ws, flags, device, peaks, sampler, reps=60):
    """Each projection type alone: its 32 distinct weight sets in one graph
    (so every launch reads its weights from HBM); per-call microseconds as
    median / p10 / p90 over the replays."""
    from gemm_w4a16_b200 import w4a16  # noqa: F401

    out = {}
    for name, M, K in LLAMA7B_LAYER:
        sub = [c for c in calls if c[0] == name]
        gs = capture(lambda sub=sub: run_calls_ws(sub, ws, flags), device)
        t0 = time.time()
        _, per = time_steps(gs, reps, 5, device)
        t1 = time.time()
        us = pct(per, 1e3 / len(sub))
        b = alg_bytes(M, K, 1)
        out[name] = {"M": M, "K": K, "N": 1, "us": us["median"], "us_pct": us,
                     "GBps": b / (us["median"] * 1e-6) / 1e9,
                     "frac_hbm": b / (us["median"] * 1e-6) / 1e9 / peaks["hbm_gbs"],
                     "clocks": sampler.summary(t0, t1)}
        del gs
    return out


def make_device_problem(device, M, K, N, seed, outlier_frac=0.0):
    import numpy as np
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    q, z, s = synth.make_weights_torch(M, K, GROUP, gen, device)
    w = w4a16.pack(q, s, z)
    x = synth.make_activations_torch(N, K, gen, device)
    if outlier_frac:
        rng = np.random.default_rng(seed)
        idx = torch.from_numpy(rng.choice(K, int(round(outlier_frac * K)), replace=False)).to(device)
        x[:, idx] = (x[:, idx].float() * 20).half()
    return w, x


def prefill_measure(device, peaks, sampler, reps=50, copies=3):
    """The two prefill GEMMs of the benchmark configuration (1 % outlier
    channels in X), TFLOP/s.  `copies` distinct (W, X, Y) sets per graph
    (> 250 MB, beyond L2) so no call finds its inputs cached; per-call
    microseconds as median / p10 / p90 over the replays, against the measured
    bf16 peak (fp16 runs at the same rate) and NVIDIA's dense fp16 figure."""
    import torch

    from gemm_w4a16_b200 import w4a16

    out = {}
    for name, M, K, N in (("qkv_n4096", 12288, 4096, 4096), ("down_n2048", 4096, 11008, 2048)):
        sets = []
        for c in range(copies):
            w, x = make_device_problem(device, M, K, N, seed=7 + c, outlier_frac=0.01)
            sets.append((w, x, torch.empty((N, M), dtype=torch.float16, device=device)))
        g = capture(lambda: [w4a16.gemm(w, x, Y=y) for w, x, y in sets], device)
        t0 = time.time()
        _, per = time_steps(g, reps, 5, device)
        t1 = time.time()
        us = pct(per, 1e3 / copies)
        tf = alg_flops(M, K, N) / (us["median"] * 1e-6) / 1e12
        out[name] = {"M": M, "K": K, "N": N, "us": us["median"], "us_pct": us, "TFLOPS": tf,
                     "path": w4a16.select_path(M, K, N),
                     "frac_tensor": tf / peaks["bf16_tflops"], "peak": peaks["bf16_tflops"],
                     "peak_kind": "measured bf16 burst (cuBLAS; fp16 same rate)",
                     "frac_nominal_dense_fp16": tf / NOMINAL_DENSE_FP16_TFLOPS,
                     "clocks": sampler.summary(t0, t1)}
        del g, sets
        torch.cuda.empty_cache()
    return out


SWEEP_N = (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096)


def n_sweep_measure(device, peaks, sampler, copies=16, reps=20):
    """N sweep on the fused QKV shape (M = 12288, K = 4096), every kernel that
    takes the N (decode kernel up to 64 tokens, 8 per launch; split
    tensor-core decode up to 64; tensor-core tiles always), 16 rotated weight copies (420 MB,
    beyond L2).  Rows: [N, path, median us, roofline fraction, chosen]."""
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    M, K = 12288, 4096
    ws_copies = [make_device_problem(device, M, K, 1, seed=100 + i)[0] for i in range(copies)]
    rows = []
    t0 = time.time()
    for N in SWEEP_N:
        gen = torch.Generator(device=device)
        gen.manual_seed(N)
        x = synth.make_activations_torch(N, K, gen, device)
        y = torch.empty((N, M), dtype=torch.float16, device=device)
        wsp = w4a16.Workspace(device, w4a16.workspace_size(M, K, min(N, w4a16.GEMV_TC_MAX_TOKENS)))
        chosen = w4a16.select_path_ws(M, K, N)
        paths = [w4a16.PATH_TC]
        if N <= 64:
            paths.insert(0, w4a16.PATH_GEMV)
        if N <= w4a16.GEMV_TC_MAX_TOKENS:
            paths.append(w4a16.PATH_GEMV_TC)
        for path in paths:
            flags = w4a16.FLAG_EARLY_WEIGHTS if path != w4a16.PATH_TC else 0
            g = capture(lambda path=path, flags=flags: [w4a16.gemm_ws(w, x, Y=y, path=path, workspace=wsp,
                                                                     flags=flags) for w in ws_copies], device)
            settle(g, device)
            _, per = time_steps(g, reps, 10, device)
            us = pct(per, 1e3 / copies)["median"]
            gbs = alg_bytes(M, K, N) / (us * 1e-6) / 1e9
            tfs = alg_flops(M, K, N) / (us * 1e-6) / 1e12
            rows.append([N, {1: "gemv", 2: "tc", 3: "gemv_tc"}[path], round(us, 2),
                         round(max(gbs / peaks["hbm_gbs"], tfs / peaks["bf16_tflops"]), 3),
                         path == chosen])
            del g
    t1 = time.time()
    del ws_copies
    torch.cuda.empty_cache()
    return {"M": M, "K": K, "columns": ["N", "path", "us", "roof_frac", "auto_choice"], "rows": rows,
            "clocks": sampler.summary(t0, t1)}


def fused_measure(device, peaks, sampler, reps=20):
    """The fused forms and the secondary kernels, compactly: per-call
    microseconds (median over `reps` graph replays, each graph several
    rotated copies, beyond L2) with the clock summary of each window.
      qkv_norm_n1     add_rmsnorm + gemm_qkv_ws chained vs add_rmsnorm_gemm_qkv
                      (LLaMA-7B QKV, N = 1, early weights);
      qkv_epilogue    plain product vs the QKV split + bias form, N = 1 and 4096;
      gate_up         plain product vs SiLU(gate)*up form vs plain + torch, N = 1
                      and 4096;
      add_rmsnorm     16384 x 4096 (HBM bytes 8 per channel);
      quantize_qkv    the group quantiser on the 12288 x 4096 weight."""
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    out = {}
    fl = w4a16.FLAG_EARLY_WEIGHTS

    def timed(fns, per_graph):
        res = {}
        for name, fn in fns.items():
            g = capture(fn, device)
            t0 = time.time()
            settle(g, device)
            _, per = time_steps(g, reps, 10, device)
            res[name] = {"us": pct(per, 1e3 / per_graph)["median"], "clocks": sampler.summary(t0, time.time())}
            del g
        return res

    # Residual add + RMS norm folded into the QKV projection, N = 1.
    M, K, splits = 12288, 4096, (4096, 4096, 4096)
    gen = torch.Generator(device=device)
    gen.manual_seed(31)
    gamma = (1.0 + 0.1 * torch.randn(K, device=device, generator=gen)).half()
    sets = []
    for c in range(8):
        w, _ = make_device_problem(device, M, K, 1, seed=60 + c)
        h = torch.randn((1, K), device=device, generator=gen).half()
        d = torch.randn((1, K), device=device, generator=gen).half()
        sets.append((w, h, d, torch.empty_like(h), torch.empty_like(h),
                     tuple(torch.empty((1, m), dtype=torch.float16, device=device) for m in splits)))
    ws = w4a16.Workspace(device, w4a16.workspace_size(M, K, 1))
    out["qkv_norm_n1"] = timed({
        "chain": lambda: [(w4a16.add_rmsnorm(h, gamma, d=d, r_out=r, X=X),
                           w4a16.gemm_qkv_ws(w, X, splits, out=o, workspace=ws, flags=fl))
                          for w, h, d, r, X, o in sets],
        "fused": lambda: [w4a16.add_rmsnorm_gemm_qkv(h, gamma, w, splits, d=d, r_out=r, out=o, flags=fl)
                          for w, h, d, r, X, o in sets]}, len(sets))
    del sets

    # QKV split + bias epilogue against the plain product.
    res = {}
    for N, copies in ((1, 8), (4096, 2)):
        probs = [make_device_problem(device, M, K, N, seed=70 + c) for c in range(copies)]
        bias = torch.randn(M, device=device, generator=gen).half()
        ys = [torch.empty((N, M), dtype=torch.float16, device=device) for _ in probs]
        os_ = [tuple(torch.empty((N, m), dtype=torch.float16, device=device) for m in splits) for _ in probs]
        ws.ensure(w4a16.workspace_size(M, K, N))
        res[f"n{N}"] = timed({
            "plain": lambda: [w4a16.gemm_ws(w, x, Y=y, workspace=ws, flags=fl) for (w, x), y in zip(probs, ys)],
            "fused_split_bias": lambda: [w4a16.gemm_qkv_ws(w, x, splits, bias=bias, out=o, workspace=ws, flags=fl)
                                         for (w, x), o in zip(probs, os_)]}, copies)
        del probs, ys, os_
        torch.cuda.empty_cache()
    out["qkv_epilogue"] = res

    # SiLU(gate) * up epilogue.
    Mi = 11008
    res = {}
    for N, copies in ((1, 8), (4096, 2)):
        sets = []
        for _ in range(copies):
            q, z, sc = synth.make_weights_torch(2 * Mi, K, GROUP, gen, device)
            sets.append((w4a16.pack_gate_up(q, sc, z), w4a16.pack(q, sc, z),
                         synth.make_activations_torch(N, K, gen, device),
                         torch.empty((N, Mi), dtype=torch.float16, device=device),
                         torch.empty((N, 2 * Mi), dtype=torch.float16, device=device)))
            del q, z, sc
        ws.ensure(w4a16.workspace_size(2 * Mi, K, N))
        res[f"n{N}"] = timed({
            "plain": lambda: [w4a16.gemm_ws(wp, x, Y=y, workspace=ws, flags=fl) for _, wp, x, _, y in sets],
            "fused": lambda: [w4a16.gemm_gate_up_ws(wg, x, H=h, workspace=ws, flags=fl)
                              for wg, _, x, h, _ in sets],
            "plain_then_torch": lambda: [(w4a16.gemm_ws(wp, x, Y=y, workspace=ws, flags=fl),
                                          torch.mul(torch.nn.functional.silu(y[:, :Mi]), y[:, Mi:], out=h))
                                         for _, wp, x, h, y in sets]}, copies)
        del sets
        torch.cuda.empty_cache()
    out["gate_up"] = res

    # Residual add + RMS norm at prefill width, and the group quantiser.
    Nn = 16384
    h = torch.randn((Nn, K), device=device, generator=gen).half()
    d = torch.randn((Nn, K), device=device, generator=gen).half()
    r, X = torch.empty_like(h), torch.empty_like(h)
    t = timed({"add_rmsnorm": lambda: w4a16.add_rmsnorm(h, gamma, d=d, r_out=r, X=X)}, 1)["add_rmsnorm"]
    gbs = (8 * Nn * K + 2 * K) / (t["us"] * 1e-6) / 1e9
    out["add_rmsnorm_n16384"] = dict(t, GBps=gbs, frac_hbm=gbs / peaks["hbm_gbs"])
    del h, d, r, X
    wts = [torch.randn((M, K), device=device, dtype=torch.float32).mul_(0.05).half() for _ in range(4)]
    qs = [(torch.empty((M, K), dtype=torch.uint8, device=device),
           torch.empty((M, K // GROUP), dtype=torch.float16, device=device),
           torch.empty((M, K // GROUP), dtype=torch.uint8, device=device)) for _ in wts]
    lib = w4a16.lib()

    def quantize_all():
        stream = torch.cuda.current_stream(device).cuda_stream   # the capture stream inside capture
        for w, (q, s, z) in zip(wts, qs):
            if lib.w4a16_quantize(w.data_ptr(), M, K, GROUP, q.data_ptr(), s.data_ptr(), z.data_ptr(), stream):
                raise RuntimeError("w4a16_quantize failed")

    t = timed({"quantize": quantize_all}, len(wts))["quantize"]
    gbs = (3 * M * K + 3 * M * (K // GROUP)) / (t["us"] * 1e-6) / 1e9
    out["quantize_qkv"] = dict(t, GBps=gbs, frac_hbm=gbs / peaks["hbm_gbs"])
    del wts, qs
    torch.cuda.empty_cache()
    return out


LLAMA3_SHAPES = [("qkv", 6144, 4096), ("o", 4096, 4096), ("gate_up", 28672, 4096), ("down", 4096, 14336),
                 ("lm_head", 128256, 4096)]


def llama3_measure(device, peaks, sampler, reps=20):
    """LLaMA-3-8B batched decode, N in {1, 16, 64}, the automatic path of the
    workspace entry point (early weights); rotated copies totalling at least
    400 MB per shape (beyond L2).  Rows: [shape, N, path, median us, GB/s,
    roofline fraction]."""
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    rows = []
    t0 = time.time()
    first = True
    for name, M, K in LLAMA3_SHAPES:
        copies = max(2, min(16, -(-400_000_000 // alg_bytes(M, K, 1))))
        wts = [make_device_problem(device, M, K, 1, seed=300 + i)[0] for i in range(copies)]
        for N in (1, 16, 64):
            gen = torch.Generator(device=device)
            gen.manual_seed(N)
            x = synth.make_activations_torch(N, K, gen, device)
            y = torch.empty((N, M), dtype=torch.float16, device=device)
            wsp = w4a16.Workspace(device, w4a16.workspace_size(M, K, N))
            g = capture(lambda: [w4a16.gemm_ws(w, x, Y=y, workspace=wsp, flags=w4a16.FLAG_EARLY_WEIGHTS)
                                 for w in wts], device)
            settle(g, device, 250.0 if first else 25.0)   # after the N sweep's compute-bound end
            first = False
            _, per = time_steps(g, reps, 10, device)
            us = pct(per, 1e3 / copies)["median"]
            gbs = alg_bytes(M, K, N) / (us * 1e-6) / 1e9
            tfs = alg_flops(M, K, N) / (us * 1e-6) / 1e12
            rows.append([name, N, {1: "gemv", 2: "tc", 3: "gemv_tc"}[w4a16.select_path_ws(M, K, N)],
                         round(us, 2), round(gbs, 1),
                         round(max(gbs / peaks["hbm_gbs"], tfs / peaks["bf16_tflops"]), 3)])
            del g
        del wts
        torch.cuda.empty_cache()
    t1 = time.time()
    return {"columns": ["shape", "N", "path", "us", "GBps", "roof_frac"], "rows": rows,
            "clocks": sampler.summary(t0, t1)}


def qkv_norm_workload(args, device, peaks):
    """Residual add + RMS norm + fused QKV projection of LLaMA-7B at N = 1
    (h, d [1, 4096]; weight 12288 x 4096 as (4096, 4096, 4096); 8 rotated
    weight copies, beyond L2), two arms, each a CUDA graph:
      chain  w4a16_add_rmsnorm (X and r to memory), then w4a16_gemm_qkv_ws
             with early weights (its weight stream overlaps the norm kernel);
      fused  w4a16_add_rmsnorm_gemm_qkv with early weights (X never stored).
    Microseconds per (norm + projection) pair, three passes of alternating
    order, median clock per pass."""
    import torch

    from gemm_w4a16_b200 import w4a16

    M, K, N, splits = 12288, 4096, 1, (4096, 4096, 4096)
    gen = torch.Generator(device=device)
    gen.manual_seed(31)
    gamma = (1.0 + 0.1 * torch.randn(K, device=device, generator=gen)).half()
    sets = []
    for c in range(8):
        w, _ = make_device_problem(device, M, K, N, seed=60 + c)
        h = torch.randn((N, K), device=device, generator=gen).half()
        d = torch.randn((N, K), device=device, generator=gen).half()
        outs = tuple(torch.empty((N, m), dtype=torch.float16, device=device) for m in splits)
        sets.append((w, h, d, torch.empty_like(h), torch.empty_like(h), outs))
    ws = w4a16.Workspace(device, w4a16.workspace_size(M, K, N))
    fl = w4a16.FLAG_EARLY_WEIGHTS

    def chain():
        for w, h, d, r, X, outs in sets:
            w4a16.add_rmsnorm(h, gamma, eps=1e-6, d=d, r_out=r, X=X)
            w4a16.gemm_qkv_ws(w, X, splits, out=outs, workspace=ws, flags=fl)

    def fused():
        for w, h, d, r, X, outs in sets:
            w4a16.add_rmsnorm_gemm_qkv(h, gamma, w, splits, eps=1e-6, d=d, r_out=r, out=outs, flags=fl)

    arms = {"chain": chain, "fused": fused}
    graphs = {name: capture(fn, device) for name, fn in arms.items()}
    sampler = ClockSampler(torch.cuda.current_device())
    sampler.start()
    time.sleep(0.2)
    runs = {name: [] for name in arms}
    for order in (list(arms), list(arms)[::-1], list(arms)):
        for name in order:
            t0 = time.time()
            us = time_graph(graphs[name], args.steps, args.warmup, device) * 1e3 / len(sets)
            runs[name].append((us, sampler.summary(t0, time.time())))
    sampler.stop()
    for name in arms:
        us = [u for u, _ in runs[name]]
        print(json.dumps({"workload": f"add_rmsnorm + qkv {name} M={M} K={K} N={N}",
                          "us": sum(us) / len(us), "us_each": us,
                          "sm_mhz_each": [c["sm_mhz"] for _, c in runs[name]],
                          "reasons": sorted({r for _, c in runs[name] for r in c["reasons"]})}), flush=True)
    return 0


def qkv_fused_workload(args, device, peaks):
    """Fused QKV projection of LLaMA-7B (3 x 4096 rows, K = 4096) at N = 1
    (8 rotated weight copies, beyond L2) and N = 4096, four arms:
      plain           w4a16_gemm into one [N][M] buffer (no split, no bias);
      fused_split     w4a16_gemm_qkv writing Q, K, V separately, no bias;
      fused_split_bias  the same with an fp16 bias;
      unfused         w4a16_gemm, then a torch add per projection for the
                      split and the bias (what a caller writes without the
                      fused form; timing comparator only).
    Each arm is a CUDA graph timed in three passes, the order of the arms
    alternating (forward, reverse, forward), with the median SM clock of each
    timing window sampled; reported are the mean time, each pass's time and
    clock, and the mean of time x clock (cycles), which a clock drift under the
    power cap does not move."""
    import torch

    from gemm_w4a16_b200 import w4a16

    M, K, splits = 12288, 4096, (4096, 4096, 4096)
    bounds = [(0, 4096), (4096, 8192), (8192, 12288)]
    sampler = ClockSampler(device.index or 0)
    sampler.start()
    try:
        for N, copies_n in ((1, 8), (4096, 1)):
            problems = [make_device_problem(device, M, K, N, seed=50 + c) for c in range(copies_n)]
            bias = torch.randn(M, device=device).half()
            ys = [torch.empty((N, M), dtype=torch.float16, device=device) for _ in problems]
            outs = [tuple(torch.empty((N, m), dtype=torch.float16, device=device) for m in splits)
                    for _ in problems]

            def plain():
                for (w, x), y in zip(problems, ys):
                    w4a16.gemm(w, x, Y=y)

            def fused_split():
                for (w, x), o in zip(problems, outs):
                    w4a16.gemm_qkv(w, x, splits, out=o)

            def fused():
                for (w, x), o in zip(problems, outs):
                    w4a16.gemm_qkv(w, x, splits, bias=bias, out=o)

            def unfused():
                for (w, x), y, o in zip(problems, ys, outs):
                    w4a16.gemm(w, x, Y=y)
                    for (c0, c1), oi in zip(bounds, o):
                        torch.add(y[:, c0:c1], bias[c0:c1], out=oi)

            arms = {"plain": plain, "fused_split": fused_split, "fused_split_bias": fused,
                    "unfused_gemm_then_torch_split_bias": unfused}
            graphs = {name: capture(fn, device) for name, fn in arms.items()}
            names = list(arms)
            runs = {name: [] for name in arms}
            for order in (names, names[::-1], names):
                for name in order:
                    t0 = time.time()
                    us = time_graph(graphs[name], args.steps, args.warmup, device) * 1e3 / copies_n
                    t1 = time.time()
                    runs[name].append((us, sampler.summary(t0, t1)))
            for name in arms:
                us = [u for u, _ in runs[name]]
                mhz = [c["sm_mhz"] for _, c in runs[name]]
                reasons = sorted({r for _, c in runs[name] for r in c["reasons"]})
                mean = sum(us) / len(us)
                kcyc = (sum(u * f for u, f in zip(us, mhz)) / len(us) / 1e3) if None not in mhz else None
                print(json.dumps({"workload": f"qkv {name} M={M} K={K} N={N}", "us": mean,
                                  "us_each": us, "sm_mhz_each": mhz, "kcycles": kcyc, "reasons": reasons,
                                  "GBps": alg_bytes(M, K, N) / (mean * 1e-6) / 1e9,
                                  "TFLOPS": alg_flops(M, K, N) / (mean * 1e-6) / 1e12}), flush=True)
            del graphs, problems, ys, outs
    finally:
        sampler.stop()
    return 0


def gate_up_fused_workload(args, device, peaks):
    """Fused gate/up projection of LLaMA-7B (Mi = 11008, K = 4096) at N = 1
    (8 rotated weight copies, 375 MB, beyond L2) and N = 4096 (2 copies),
    three arms, each a CUDA graph through the workspace entry points:
      fused     w4a16_gemm_gate_up_ws on the gate/up packing (H [N][Mi]);
      plain     w4a16_gemm_ws on the same weight packed in row order (Y [N][2 Mi]);
      unfused   the plain product, then torch silu(Y[:, :Mi]) * Y[:, Mi:]
                (what a caller writes without the fused form; timing only).
    Per-call microseconds, median / p10 / p90 over the replays, with the SM
    clock of each window."""
    import torch

    from gemm_w4a16_b200 import synth, w4a16

    Mi, K = 11008, 4096
    M = 2 * Mi
    sampler = ClockSampler(device.index or 0)
    sampler.start()
    try:
        for N, copies_n in ((1, 8), (4096, 2)):
            gen = torch.Generator(device=device)
            gen.manual_seed(61)
            sets = []
            for _ in range(copies_n):
                q, z, sc = synth.make_weights_torch(M, K, GROUP, gen, device)
                sets.append((w4a16.pack_gate_up(q, sc, z), w4a16.pack(q, sc, z),
                             synth.make_activations_torch(N, K, gen, device),
                             torch.empty((N, Mi), dtype=torch.float16, device=device),
                             torch.empty((N, M), dtype=torch.float16, device=device),
                             torch.empty((N, Mi), dtype=torch.float16, device=device)))
                del q, z, sc
            ws = w4a16.Workspace(device, w4a16.workspace_size(M, K, N))
            flags = w4a16.FLAG_EARLY_WEIGHTS

            def fused():
                for wg, _, x, h, _, _ in sets:
                    w4a16.gemm_gate_up_ws(wg, x, H=h, workspace=ws, flags=flags)

            def plain():
                for _, wp, x, _, y, _ in sets:
                    w4a16.gemm_ws(wp, x, Y=y, workspace=ws, flags=flags)

            def unfused():
                for _, wp, x, _, y, h2 in sets:
                    w4a16.gemm_ws(wp, x, Y=y, workspace=ws, flags=flags)
                    torch.mul(torch.nn.functional.silu(y[:, :Mi]), y[:, Mi:], out=h2)

            for name, fn in (("fused", fused), ("plain", plain), ("unfused_plain_then_torch", unfused)):
                g = capture(fn, device)
                t0 = time.time()
                _, per = time_steps(g, args.steps, args.warmup, device)
                t1 = time.time()
                us = pct(per, 1e3 / copies_n)
                print(json.dumps({"workload": f"gate_up {name} Mi={Mi} K={K} N={N}", "us": us["median"],
                                  "us_pct": us, "path": w4a16.select_path_ws(M, K, N),
                                  "GBps": alg_bytes(M, K, N) / (us["median"] * 1e-6) / 1e9,
                                  "TFLOPS": alg_flops(M, K, N) / (us["median"] * 1e-6) / 1e12,
                                  "clocks": sampler.summary(t0, t1)}), flush=True)
                del g
            del sets
            torch.cuda.empty_cache()
    finally:
        sampler.stop()
    return 0


def quantize_workload(args, device, peaks):
    """Group quantiser fp16 W -> (q, s, z) on the four LLaMA-7B projection
    shapes, 8 rotated weight copies per shape (beyond L2); HBM bytes per call:
    2 read + 1 written per weight, plus 3 bytes of scale and zero per group."""
    import torch

    from gemm_w4a16_b200 import w4a16

    for name, M, K in LLAMA7B_LAYER:
        copies = [torch.randn((M, K), device=device, dtype=torch.float32).mul_(0.05).half()
                  for _ in range(8)]
        outs = [(torch.empty((M, K), dtype=torch.uint8, device=device),
                 torch.empty((M, K // GROUP), dtype=torch.float16, device=device),
                 torch.empty((M, K // GROUP), dtype=torch.uint8, device=device)) for _ in copies]
        lib = w4a16.lib()
        stream = torch.cuda.current_stream().cuda_stream

        def one_pass():
            for w, (q, s, z) in zip(copies, outs):
                st = lib.w4a16_quantize(w.data_ptr(), M, K, GROUP, q.data_ptr(), s.data_ptr(), z.data_ptr(),
                                        stream)
                if st != 0:
                    raise RuntimeError(f"w4a16_quantize failed ({st})")

        for _ in range(args.warmup):
            one_pass()
        torch.cuda.synchronize(device)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            one_pass()
        e1.record()
        torch.cuda.synchronize(device)
        us = e0.elapsed_time(e1) * 1e3 / (args.steps * len(copies))
        nbytes = 3 * M * K + 3 * M * (K // GROUP)
        gbps = nbytes / (us * 1e-6) / 1e9
        print(json.dumps({"workload": f"quantize {name} M={M} K={K}", "us": us, "GBps": gbps,
                          "frac_hbm": gbps / peaks["hbm_gbs"]}), flush=True)
        del copies, outs
    return 0


def add_rmsnorm_workload(args, device, peaks):
    """Residual add + RMS normalisation at LLaMA-7B width (K = 4096): N = 1
    (one decode token; 64 rotated row buffers per graph) and N = 16384 (four
    4096-token prefill batches; 512 MB of h, d, r and X per call, beyond L2).
    HBM bytes per call: h and d read, r and X written, 2 bytes each per
    channel, plus gamma once.  Each size one CUDA graph of w4a16_add_rmsnorm
    calls."""
    import torch

    from gemm_w4a16_b200 import w4a16

    K = 4096
    gen = torch.Generator(device=device)
    gen.manual_seed(7)
    gamma = (1.0 + 0.1 * torch.randn(K, device=device, generator=gen)).half()
    for N, copies_n in ((1, 64), (16384, 1)):
        sets = []
        for _ in range(copies_n):
            h = torch.randn((N, K), device=device, generator=gen).half()
            d = torch.randn((N, K), device=device, generator=gen).half()
            sets.append((h, d, torch.empty_like(h), torch.empty_like(h)))

        def fn():
            for h, d, r, X in sets:
                w4a16.add_rmsnorm(h, gamma, eps=1e-6, d=d, r_out=r, X=X)

        g = capture(fn, device)
        us = time_graph(g, args.steps, args.warmup, device) * 1e3 / copies_n
        nbytes = 8 * N * K + 2 * K
        gbps = nbytes / (us * 1e-6) / 1e9
        print(json.dumps({"workload": f"add_rmsnorm N={N} K={K}", "us": us, "GBps": gbps,
                          "frac_hbm": gbps / peaks["hbm_gbs"], "launches_per_graph": copies_n}), flush=True)
        del g, sets
    return 0


def single_shape(args, device, M, K, N, path=0):
    """One shape, plain launches through w4a16_gemm_ws (any path, with a
    workspace; used for ncu captures and quick timing)."""
    import torch

    from gemm_w4a16_b200 import w4a16

    w, x = make_device_problem(device, M, K, N, seed=3)
    y = torch.empty((N, M), dtype=torch.float16, device=device)
    ws = w4a16.Workspace(device, w4a16.workspace_size(M, K, N))
    for _ in range(args.warmup):
        w4a16.gemm_ws(w, x, Y=y, path=path, workspace=ws)
    torch.cuda.synchronize(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.steps):
        w4a16.gemm_ws(w, x, Y=y, path=path, workspace=ws)
    e1.record()
    torch.cuda.synchronize(device)
    ms = e0.elapsed_time(e1) / args.steps
    b, f = alg_bytes(M, K, N), alg_flops(M, K, N)
    print(json.dumps({"workload": f"M={M} K={K} N={N}", "us": ms * 1e3,
                      "GBps": b / (ms * 1e-3) / 1e9, "TFLOPS": f / (ms * 1e-3) / 1e12,
                      "path": path or w4a16.select_path_ws(M, K, N),
                      "note": "plain launches; weights may sit in L2 across iterations"}))
    return 0


def sweep(args, device):
    """N sweep on the fused QKV shape, both kernels, 16 weight copies rotated
    (16 x 26 MB > L2) so that weights come from HBM."""
    import torch

    from gemm_w4a16_b200 import w4a16

    peaks, _ = load_peaks()
    M, K = 12288, 4096
    copies = [make_device_problem(device, M, K, 1, seed=100 + i)[0] for i in range(16)]
    for N in (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048, 4096):
        from gemm_w4a16_b200 import synth
        gen = torch.Generator(device=device)
        gen.manual_seed(N)
        x = synth.make_activations_torch(N, K, gen, device)
        y = torch.empty((N, M), dtype=torch.float16, device=device)
        for path in (w4a16.PATH_GEMV, w4a16.PATH_TC):
            if path == w4a16.PATH_GEMV and N > 256:
                continue
            try:
                g = capture(lambda path=path: [w4a16.gemm_ex(w, x, Y=y, path=path) for w in copies],
                            device)
            except w4a16.W4A16Error as e:
                print(json.dumps({"N": N, "path": path, "error": str(e)}), flush=True)
                continue
            ms = time_graph(g, 5, 2, device) / len(copies)
            b, f = alg_bytes(M, K, N), alg_flops(M, K, N)
            gbs, tfs = b / (ms * 1e-3) / 1e9, f / (ms * 1e-3) / 1e12
            print(json.dumps({"N": N, "path": "gemv" if path == 1 else "tc", "us": ms * 1e3,
                              "GBps": gbs, "TFLOPS": tfs,
                              "roof_frac": max(gbs / peaks["hbm_gbs"], tfs / peaks["bf16_tflops"]),
                              "auto": w4a16.select_path(M, K, N)}), flush=True)
            del g
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["decode", "qkv_n1", "prefill", "sweep", "shape", "quantize",
                                           "qkv_fused", "gate_up_fused", "add_rmsnorm", "qkv_norm"],
                    default="decode")
    ap.add_argument("--M", type=int, default=12288)
    ap.add_argument("--K", type=int, default=4096)
    ap.add_argument("--N", type=int, default=1)
    ap.add_argument("--path", type=int, default=0,
                    help="0 auto, 1 decode kernel, 2 tensor-core tiles, 3 split tensor-core decode")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the prefill, N-sweep and LLaMA-3 measurements")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return main_reference(args)
    return main_ours(args)


if __name__ == "__main__":
    sys.exit(main())
