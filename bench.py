#!/usr/bin/env python
"""Benchmark of the weight-only low-bit GEMM library on B200.

Default workload: one denoise step of the FLUX.2-Klein-4B transformer's low-bit linear chain at
a 1024x1024 image (4096 image + 512 text tokens): 5 double-stream blocks (image and text QKV,
out, MLP-up, MLP-down) and 20 single-stream blocks (fused QKV+MLP-in, fused out), ternary
2-bit weights with fp16 scales per group of 128, d = 3072. One step = one lowbit_gemm_batch
call over the 80 linears, with inputs resident in HBM (3.7 GB of activations and 0.75 GB of
packed weights, far larger than L2, so no flush is needed between steps).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl lowbit|reference]

Prints one JSON line (rank 0). Under torchrun each rank runs its own replica (weak scaling);
the timed region is bracketed by a barrier and a device synchronize and the max over ranks is
reported. `--impl reference` times the CPU oracle (fp64, host cores) on a bounded sample of
the same workload.
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

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "low-bit GEMM TFLOP/s (% of B200 bf16 TC peak) at 1024² Klein shapes; HBM GB/s"
UNIT = "TFLOP/s"
DEFAULT_WORKLOAD = "klein_step_chain_1024sq_ternary_g128"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# The sources each kernel is built from (besides the headers every kernel includes): a capture
# stays valid while these are unchanged.
KERNEL_SOURCES = {"lowbit_gemm_kernel": ("gemm_sm100.cu", "tcgen05_ptx.cuh"),
                  "lowbit_smallm_kernel": ("smallm_kernel.cuh", "smallm_host.cu", "smallm_b1.cu", "smallm_b2.cu",
                                           "smallm_b4.cu")}
SHARED_SOURCES = ("sm100_ptx.cuh", "lowbit_internal.h")


def kernel_source_hash(kernel=None):
    """sha256 over the sources a kernel is built from (all CUDA sources and the ABI header when
    `kernel` is None): identifies the code a capture measured."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_only_w2_b200", "csrc")
    inc = os.path.join(ROOT, "include")
    if kernel is None:
        files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh", ".h")))
        files += sorted(os.path.join(inc, f) for f in os.listdir(inc) if f.endswith(".h"))
    else:
        files = [os.path.join(csrc, f) for f in (*KERNEL_SOURCES[kernel], *SHARED_SOURCES)]
        files += [os.path.join(inc, "lowbit.h")]
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(key):
    """DRAM bytes per launch from the committed ncu summary for this workload, or None if there is
    none or the captured kernel's sources have changed since."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            entry = json.load(f).get(key)
    except Exception:
        return None
    if not entry or entry.get("source_sha256") != kernel_source_hash(entry.get("kernel")):
        return None
    return entry.get("dram_bytes_per_launch")


def rotation_copies(step_bytes_: int, weight_bytes_: int, l2_bytes: int) -> int:
    """Distinct weight copies a workload rotates through: 1 if its bytes reach twice L2, else at
    least 20 and enough that the copies' weights exceed 2.2x L2 (at most 256)."""
    if step_bytes_ >= 2 * l2_bytes:
        return 1
    return min(256, max(20, -(-int(2.2 * l2_bytes) // max(1, weight_bytes_))))


def is_hbm_bound(flops: float, nbytes: float, peaks: dict) -> bool:
    """Below the ridge point (peak flop/s over peak byte/s) a workload is bound by HBM."""
    ridge = peaks.get("bf16_tflops", 1590.0) * 1e12 / (peaks.get("hbm_gbs", 6650.0) * 1e9)
    return flops / nbytes < ridge


SHAPE_SAMPLES, SHAPE_REPLAYS = 21, 4   # per-launch timing: median of 21 samples of 4 graph replays


def measure_shapes(items, copies, lb, torch, device, stream, cap_stream, samples=SHAPE_SAMPLES,
                   replays=SHAPE_REPLAYS):
    """Per-launch durations of each distinct shape of `items` (ms): {(M, K, N): (call, GEMM kernel,
    X conversion, reps)}.

    For each distinct shape, graph A holds `reps` back-to-back lowbit_gemm calls (rotating weight
    copies where there are several, so weights stream from HBM as in the timed steps) and graph B
    one lowbit_gemm_batch of the same `reps` linears sharing one X, which the library converts
    once. A sample replays a graph `replays` times between two events on the launching stream; the
    per-launch time is the median over `samples` samples of sample time / (replays * reps). For
    more than 16 tokens a call is the X conversion pass plus the GEMM kernel: the conversion's time
    is (A - B) / (reps - 1) per launch and the GEMM kernel's is the call's minus that. At most 16
    tokens a call is the small-M GEMM kernel alone."""
    def time_graph(gph, per_sample, warm=2):
        for _ in range(warm):
            gph.replay()
        torch.cuda.synchronize(device)
        ts = []
        for _ in range(samples):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(replays):
                gph.replay()
            e1.record(stream)
            torch.cuda.synchronize(device)
            ts.append(e0.elapsed_time(e1) / (replays * per_sample))
        return statistics.median(ts)

    def capture(fn):
        gph = torch.cuda.CUDAGraph()
        cap_stream.wait_stream(stream)
        with torch.cuda.stream(cap_stream):
            with torch.cuda.graph(gph, stream=cap_stream):
                fn()
        stream.wait_stream(cap_stream)
        return gph

    shape_times = {}
    seen = {}
    for it in items:
        seen.setdefault((it["spec"].M, it["spec"].K, it["spec"].N), it)
    for key, it in seen.items():
        reps = max(10, copies)
        sp = it["spec"]

        def calls():
            for i in range(reps):
                w_p, w_s, w_z = it["reps"][i % copies]
                lb.gemm(it["x"], w_p, w_s, w_z, sp.bits, sp.group_size, out=it["y"])

        g_a = capture(calls)
        t_call = time_graph(g_a, reps)
        del g_a
        t_conv = 0.0
        if sp.M > 16:
            shared = [lb.make_desc(it["x"], *it["reps"][i % copies], it["y"], sp.bits, sp.group_size)
                      for i in range(reps)]
            g_b = capture(lambda: lb.gemm_batch(shared, device))
            t_shared = time_graph(g_b, reps)
            del g_b
            t_conv = max(0.0, (t_call - t_shared) * reps / (reps - 1))
        shape_times[key] = (t_call, t_call - t_conv, t_conv, reps)
    return shape_times


CONFIGS = ("tiny_ternary_g64", "qkv_512sq_ternary_g128", "mlp_1024sq_binary_g128", "te_m512_uint4_g64",
           "te_m16_uint4_g64", "klein_linears_m1_ternary_g128")
# Whole-step workloads measured beside them: the transformer step with separate Q/K/V and
# add-Q/K/V projections (100 linears) and the text encoder's 4-layer MLP chain at 512 and 16 tokens.
STEP_CONFIGS = ("klein_step_linears100_1024sq_ternary_g128", "te_mlp4_m512_uint4_g64", "te_mlp4_m16_uint4_g64")


def capture_steps(lb, torch, desc_sets, device, stream, cap_stream):
    """One CUDA graph per weight copy, each holding one lowbit_gemm_batch over the step's linears
    (replaying a graph measures the GPU, not the host's per-call submission cost)."""
    lb.gemm_batch(desc_sets[0], device)   # allocates the shared workspace before capture
    torch.cuda.synchronize(device)
    graphs = []
    cap_stream.wait_stream(stream)
    with torch.cuda.stream(cap_stream):
        for descs in desc_sets:
            gph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(gph, stream=cap_stream):
                lb.gemm_batch(descs, device)
            graphs.append(gph)
    stream.wait_stream(cap_stream)
    torch.cuda.synchronize(device)
    return graphs


def measure_step_config(name, lb, torch, device, stream, cap_stream, peaks, l2_bytes, steps=10, samples=5):
    """Step time of a whole workload run as one lowbit_gemm_batch per step (graph-replayed, weight
    copies rotated below twice L2): the median over `samples` samples of `steps` steps each."""
    specs = synth.WORKLOADS[name]
    flops, nbytes = step_flops(specs), step_bytes(specs)
    copies = rotation_copies(nbytes, weight_bytes(specs), l2_bytes)
    items, desc_sets = setup(specs, device, lb, torch, pinned=False, copies=copies)   # items own the buffers
    graphs = capture_steps(lb, torch, desc_sets, device, stream, cap_stream)
    n = max(steps, copies)
    for i in range(max(3, copies)):
        graphs[i % copies].replay()
    torch.cuda.synchronize(device)
    ts = []
    for _ in range(samples):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(n):
            graphs[i % copies].replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ts.append(e0.elapsed_time(e1) / n)
    ms = statistics.median(ts)
    hbm = is_hbm_bound(flops, nbytes, peaks)
    out = {"linears_per_step": len(specs), "ms_per_step": ms, "tflops": flops / (ms * 1e-3) / 1e12,
           "gbs": nbytes / (ms * 1e-3) / 1e9, "bound": "hbm" if hbm else "tensor",
           "weight_copies_rotated": copies, "steps_per_sample": n}
    if hbm:
        out["frac_of_hbm"] = out["gbs"] / peaks.get("hbm_gbs")
    else:
        out["frac_of_burst"] = out["tflops"] / peaks.get("bf16_tflops")
    del graphs, desc_sets, items
    return out


def measure_configs(lb, torch, device, stream, cap_stream, peaks, l2_bytes):
    """Per-launch results of the reference configurations (see CONFIGS), each linear timed as in
    measure_shapes with fewer replays per sample: per shape the call, GEMM kernel and conversion times, the
    throughput of the GEMM kernel and its fraction of the burst bf16 peak (tensor-bound) or of the
    HBM bandwidth (HBM-bound)."""
    out = {}
    for name in CONFIGS:
        specs = synth.WORKLOADS[name]
        copies = rotation_copies(step_bytes(specs), weight_bytes(specs), l2_bytes)
        items, _ = setup(specs, device, lb, torch, pinned=False, copies=copies)
        times = measure_shapes(items, copies, lb, torch, device, stream, cap_stream, samples=21, replays=2)
        hbm = is_hbm_bound(step_flops(specs), step_bytes(specs), peaks)
        shapes = []
        for sp in specs:
            t_call, t_gemm, t_conv, _ = times[(sp.M, sp.K, sp.N)]
            e = {"MKN": [sp.M, sp.K, sp.N], "call_us": t_call * 1e3, "gemm_us": t_gemm * 1e3,
                 "x_conversion_us": t_conv * 1e3, "gemm_tflops": sp.flops / (t_gemm * 1e-3) / 1e12,
                 "call_gbs": sp.algorithmic_bytes() / (t_call * 1e-3) / 1e9}
            if hbm:
                e["frac_of_hbm"] = e["call_gbs"] / peaks.get("hbm_gbs")
            else:
                e["gemm_frac_of_burst"] = e["gemm_tflops"] / peaks.get("bf16_tflops")
            shapes.append(e)
        out[name] = {"bound": "hbm" if hbm else "tensor", "weight_copies_rotated": copies, "linears": shapes}
        del items
        torch.cuda.synchronize(device)
        torch.cuda.empty_cache()
    for name in STEP_CONFIGS:
        out[name] = {"step": measure_step_config(name, lb, torch, device, stream, cap_stream, peaks, l2_bytes)}
        torch.cuda.synchronize(device)
        torch.cuda.empty_cache()
    if lb.device_status() != 0:
        raise RuntimeError("kernel timeout reported while measuring the reference configurations")
    return out


def max_over_ranks(v: float, world: int, device=None) -> float:
    """The maximum of v over all ranks of the default process group (v itself when alone)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(world: int, flops_per_step: float, ms_per_step: float) -> float:
    """Whole-job TFLOP/s: every rank runs the step (replicas), timed by the slowest rank."""
    return world * flops_per_step / (ms_per_step * 1e-3) / 1e12


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------------------------------------
# clocks sampled during the timed region
# --------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.idx = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.idx)], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# --------------------------------------------------------------------------------------------
# workload setup
# --------------------------------------------------------------------------------------------
def setup(specs, device, lb, torch, pinned=True, copies=1):
    """Device inputs / outputs for every linear (weights packed on the GPU by the library),
    plus pinned host copies of the activations and host buffers for the outputs.

    copies > 1 gives each linear that many distinct device copies of its packed weights, scales
    and zeros (same values), used in rotation so that a workload smaller than L2 still streams
    its weights from HBM every step. Returns (items, descriptor lists, one per copy)."""
    items = []
    for spec in specs:
        prob = synth.make_problem(spec)
        codes = torch.from_numpy(prob.codes).to(device)
        packed = lb.pack(codes, spec.bits)
        del codes
        x_host = torch.from_numpy(prob.x_bf16.view(np.int16)).view(torch.bfloat16)
        if pinned:
            x_host = x_host.pin_memory()
        x = x_host.to(device)
        s = torch.from_numpy(prob.scales).to(device)
        z = torch.from_numpy(prob.zeros).to(device) if prob.zeros is not None else None
        y = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=device)
        y_host = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, pin_memory=pinned)
        reps = [(packed, s, z)] + [(packed.clone(), s.clone(), z.clone() if z is not None else None)
                                   for _ in range(copies - 1)]
        items.append(dict(spec=spec, x=x, packed=packed, s=s, z=z, y=y, x_host=x_host, y_host=y_host, reps=reps))
    desc_sets = [[lb.make_desc(it["x"], it["reps"][c][0], it["reps"][c][1], it["reps"][c][2], it["y"],
                               it["spec"].bits, it["spec"].group_size) for it in items] for c in range(copies)]
    return items, desc_sets


def weight_bytes(specs):
    """Packed codes + scales (+ zeros) of the workload: what streams from HBM every step."""
    return sum(s.algorithmic_bytes() - s.M * s.K * 2 - s.M * s.N * 2 for s in specs)


def step_flops(specs):
    return sum(s.flops for s in specs)


def step_bytes(specs):
    return sum(s.algorithmic_bytes() for s in specs)


# --------------------------------------------------------------------------------------------
# CPU oracle timing (bounded sample)
# --------------------------------------------------------------------------------------------
def oracle_sample(specs, rows_per_shape: int):
    """Distinct shapes of the workload, each with its first `rows_per_shape` activation rows."""
    seen = {}
    for s in specs:
        seen.setdefault((s.M, s.K, s.N, s.bits, s.group_size), s)
    out = []
    for s in seen.values():
        prob = synth.make_problem(s)
        m = min(rows_per_shape, s.M)
        import oracle
        packed, _ = oracle.pack(prob.codes, s.bits)
        out.append((s, np.ascontiguousarray(prob.x_bf16[:m]), packed, prob.scales, prob.zeros, m))
    return out


def time_oracle(sample, threads=0):
    import oracle
    t0 = time.perf_counter()
    flops = 0
    for s, x, packed, sc, z, m in sample:
        oracle.gemm(x, packed, sc, z, s.N, s.bits, s.group_size, threads=threads)
        flops += 2 * m * s.K * s.N
    dt = time.perf_counter() - t0
    return flops, dt


def cpu_baseline(specs, rows_per_shape=32):
    import oracle
    sample = oracle_sample(specs, rows_per_shape)
    flops, dt = time_oracle(sample)
    nshapes = len(sample)
    # the tiny configuration (64 x 256 x 512, ternary g64) whole, on one thread
    tiny = oracle_sample(synth.WORKLOADS["tiny_ternary_g64"], 64)
    tf, t1 = time_oracle(tiny, threads=1)
    return {"value": flops / dt / 1e12, "unit": UNIT, "cores": oracle.default().threads(0), "kind": "oracle",
            "sample": f"{nshapes} distinct shapes of the workload, first {rows_per_shape} activation rows each "
                      f"(full K and N, weights decoded inside the timed call); {flops / 1e9:.1f} GFLOP in {dt:.1f} s",
            "host_cpus": os.cpu_count(),
            "single_thread_tiny": {"seconds": t1, "tflops": tf / t1 / 1e12,
                                   "what": "the whole 64 x 256 x 512 ternary g64 GEMM on one host thread"}}


# --------------------------------------------------------------------------------------------
# arms
# --------------------------------------------------------------------------------------------
def run_reference(args, specs, workload):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    rows = args.ref_rows
    sample = oracle_sample(specs, rows)
    for _ in range(args.warmup):
        time_oracle(sample)
    times = []
    flops = 0
    for _ in range(args.steps):
        f, dt = time_oracle(sample)
        flops = f
        times.append(dt)
    t = sum(times)
    value = flops * args.steps / t / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload, "sample_rows_per_shape": rows},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.default().threads(0), "kind": "oracle",
                             "sample": f"{len(sample)} distinct shapes, first {rows} activation rows each, "
                                       f"{flops / 1e9:.1f} GFLOP per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_lowbit(args, specs, workload):
    import torch
    import torch.distributed as dist
    import bit_weight_only_w2_b200 as lb

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=torch.device("cuda", local_rank))
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    lb.load()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(specs, args.ref_rows)   # before any timed GPU work; uses host cores only

    flops = step_flops(specs)
    nbytes = step_bytes(specs)
    l2_bytes = torch.cuda.get_device_properties(device).L2_cache_size
    # A workload that fits in L2 rotates distinct copies of its weights (at least 20, and enough
    # to exceed twice L2) so that every step reads them from HBM, with no flush between steps.
    copies = rotation_copies(nbytes, weight_bytes(specs), l2_bytes)
    items, desc_sets = setup(specs, device, lb, torch, pinned=not args.no_e2e, copies=copies)
    descs = desc_sets[0]
    stream = torch.cuda.current_stream(device)
    peaks, peak_src = load_peaks()
    # bound of the workload: below the ridge point (peak flop/s per peak byte/s) it is HBM-bound
    hbm_bound = is_hbm_bound(flops, nbytes, peaks)
    # kernels per step: one per linear of at most 16 tokens, two above (X conversion + GEMM; every
    # linear here has its own X)
    launches_per_step = sum(1 if s.M <= 16 else 2 for s in specs)

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(v):
        return max_over_ranks(v, world, device)

    # Each step is one lowbit_gemm_batch over the workload's linears, captured once per weight
    # copy as a CUDA graph and replayed (the end-to-end number below calls the API directly).
    cap_stream = torch.cuda.Stream(device)
    graphs = capture_steps(lb, torch, desc_sets[:copies], device, stream, cap_stream)
    step_idx = [0]

    def one_step():
        graphs[step_idx[0] % copies].replay()
        step_idx[0] += 1

    for _ in range(max(args.warmup, copies if copies > 1 else 0)):
        one_step()
    torch.cuda.synchronize(device)
    if lb.device_status() != 0:
        raise RuntimeError("kernel timeout reported during warm-up")

    clocks = ClockSampler(device.index if device.index is not None else 0)
    clocks.start()
    barrier()
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        one_step()
    b.record(stream)
    torch.cuda.synchronize(device)
    ms_total = a.elapsed_time(b)
    barrier()
    clk = clocks.stop()
    ms_total = ranks_max(ms_total)
    ms_step = ms_total / args.steps
    value = job_value(world, flops, ms_step)
    if lb.device_status() != 0:
        raise RuntimeError("kernel timeout reported during the timed steps")

    shape_times = measure_shapes(items, copies, lb, torch, device, stream, cap_stream)
    per = [(s, *shape_times[(s.M, s.K, s.N)][:3]) for s in specs]     # (spec, call, gemm, conversion) ms
    launch_ms = sum(c for _, c, _, _ in per) / len(per)
    gemm_ms = sum(g for _, _, g, _ in per) / len(per)
    conv_ms = sum(v for _, _, _, v in per) / len(per)
    launch_flops = sum(sp.flops for sp, _, _, _ in per) / len(per)
    launch_bytes = sum(sp.algorithmic_bytes() for sp, _, _, _ in per) / len(per)
    per_graph = SHAPE_SAMPLES * SHAPE_REPLAYS
    launches_timed = sum((2 if k[0] > 16 else 1) * per_graph * r for k, (_, _, _, r) in shape_times.items())
    # Per-launch figures of the other reference configurations, measured the same way after the
    # headline's timed region (so that one run of the default workload corroborates them).
    others = None
    if world == 1 and not args.no_configs and workload == DEFAULT_WORKLOAD:
        others = measure_configs(lb, torch, device, stream, cap_stream, peaks, l2_bytes)

    # End to end through the public API, as a user would pipeline it: each step copies every
    # linear's activations in (pinned host -> device, copy stream), runs lowbit_gemm per linear
    # as soon as its input has landed, and copies each output back (device -> pinned host,
    # second copy stream) as soon as it is written. Cross-step hazards are ordered with events:
    # an input is overwritten only after the previous step's GEMM read it, an output only after
    # the previous step's copy-out read it.
    e2e = None
    if not args.no_e2e:
        h2d = sum(it["x"].numel() * 2 for it in items)
        d2h = sum(it["y"].numel() * 2 for it in items)
        s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
        n_it = len(items)
        x_ready = [torch.cuda.Event() for _ in range(n_it)]
        y_ready = [torch.cuda.Event() for _ in range(n_it)]
        x_free = [torch.cuda.Event() for _ in range(n_it)]
        y_free = [torch.cuda.Event() for _ in range(n_it)]
        started = [False]

        def e2e_step():
            with torch.cuda.stream(s_in):
                for i, it in enumerate(items):
                    if started[0]:
                        s_in.wait_event(x_free[i])
                    it["x"].copy_(it["x_host"], non_blocking=True)
                    x_ready[i].record(s_in)
            for i, it in enumerate(items):
                stream.wait_event(x_ready[i])
                if started[0]:
                    stream.wait_event(y_free[i])
                lb.gemm(it["x"], it["packed"], it["s"], it["z"], it["spec"].bits, it["spec"].group_size,
                        out=it["y"])
                y_ready[i].record(stream)
                x_free[i].record(stream)
            with torch.cuda.stream(s_out):
                for i, it in enumerate(items):
                    s_out.wait_event(y_ready[i])
                    it["y_host"].copy_(it["y"], non_blocking=True)
                    y_free[i].record(s_out)
            started[0] = True

        pipelined = h2d + d2h >= (64 << 20)

        def e2e_step_batched():
            # small transfers: one batched call between the copies costs less host time
            for it in items:
                it["x"].copy_(it["x_host"], non_blocking=True)
            lb.gemm_batch(descs, device)
            for it in items:
                it["y_host"].copy_(it["y"], non_blocking=True)

        run_e2e = e2e_step if pipelined else e2e_step_batched
        run_e2e()
        torch.cuda.synchronize(device)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e2e_steps = max(1, min(args.steps, 5))
        a.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for _ in range(e2e_steps):
            run_e2e()
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)
        b.record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = ranks_max(a.elapsed_time(b)) / e2e_steps
        e2e = {"value": world * flops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
               "mode": ("copies on two streams overlapping lowbit_gemm per linear" if pipelined
                        else "copy in, one lowbit_gemm_batch, copy out")}

    traffic = measured_traffic(workload)
    burst = peaks.get("bf16_tflops")
    if hbm_bound:
        peak_bw = peaks.get("hbm_gbs")
        achieved = launch_bytes / (launch_ms * 1e-3) / 1e9
        roofline = {"bound": "hbm", "achieved": achieved, "peak": peak_bw, "unit": "GB/s",
                    "frac": achieved / peak_bw, "traffic": traffic,
                    "peak_source": f"{peak_src} HBM copy bandwidth",
                    "kernel": ("lowbit_smallm_kernel" if all(sp.M <= 16 for sp in specs)
                               else "lowbit_gemm_kernel (+ X conversion), one lowbit_gemm call"),
                    "us_per_launch": launch_ms * 1e3, "launches_timed": launches_timed,
                    "algorithmic_mb_per_launch": launch_bytes / 1e6,
                    "algorithmic_gflop_per_launch": launch_flops / 1e9,
                    "tflops_per_launch": launch_flops / (launch_ms * 1e-3) / 1e12,
                    "weight_copies_rotated": copies}
    else:
        # Each per-launch figure comes from short back-to-back replays of one shape (a few ms),
        # a kernel timed on its own: the burst peak applies.
        achieved = launch_flops / (gemm_ms * 1e-3) / 1e12
        call = launch_flops / (launch_ms * 1e-3) / 1e12
        roofline = {"bound": "tensor", "achieved": achieved, "peak": burst, "unit": "TFLOP/s",
                    "frac": achieved / burst, "traffic": traffic,
                    "peak_source": f"{peak_src} burst bf16 dense (kernels timed in short back-to-back replays)",
                    "kernel": "lowbit_gemm_kernel (GEMM kernel alone: the X conversion's share is taken out)",
                    "us_per_launch": gemm_ms * 1e3, "launches_timed": launches_timed,
                    "algorithmic_gflop_per_launch": launch_flops / 1e9,
                    "algorithmic_mb_per_launch": launch_bytes / 1e6,
                    "call": {"what": "one lowbit_gemm call = X conversion pass + GEMM kernel",
                             "achieved": call, "frac": call / burst, "us_per_launch": launch_ms * 1e3,
                             "x_conversion_us_per_launch": conv_ms * 1e3},
                    "step_frac_of_burst_peak": (flops / (ms_step * 1e-3) / 1e12) / burst}
        if copies > 1:
            roofline["weight_copies_rotated"] = copies

    if rank == 0:
        spec0 = specs[0]
        cfg = {"workload": workload, "linears_per_step": len(specs), "bits": spec0.bits,
               "group_size": spec0.group_size, "gflop_per_step": flops / 1e9,
               "algorithmic_mb_per_step": nbytes / 1e6,
               "shapes_MKN": sorted({(s.M, s.K, s.N) for s in specs}),
               "l2": (f"{copies} rotating copies of the weights ({copies * weight_bytes(specs) / 1e6:.0f} MB, "
                      f"over 2x L2; no flush)") if copies > 1 else "inputs larger than L2 (no flush)",
               "parallelism": "replicas" if world > 1 else "single GPU"}
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
                "hbm_gbs": world * nbytes / (ms_step * 1e-3) / 1e9,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": launches_per_step * args.steps, "clocks": clk}
        if others is not None:
            line["configs"] = others
        if len(specs) >= 40:   # a denoise step's chain: the pages count 4 steps per image
            line["config"]["ms_per_4_steps"] = 4 * ms_step
        print(json.dumps(line), flush=True)
        if args.per_shape:
            for (m, kk, n), (t_call, t_gemm, t_conv, reps) in sorted(shape_times.items()):
                f = 2 * m * kk * n
                sp = next(x for x in specs if (x.M, x.K, x.N) == (m, kk, n))
                print(f"# shape M={m} K={kk} N={n}: call {t_call * 1e3:.2f} us ({f / t_call / 1e9:.1f} TFLOP/s, "
                      f"{sp.algorithmic_bytes() / t_call / 1e6:.0f} GB/s); GEMM kernel {t_gemm * 1e3:.2f} us "
                      f"({f / t_gemm / 1e9:.1f} TFLOP/s); X conversion {t_conv * 1e3:.2f} us; {reps} per graph",
                      file=sys.stderr)
    del graphs, items, descs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def relaunch_under_torchrun(gpus: int, argv) -> int:
    """Run this script as `gpus` ranks of one node (torchrun, rendezvous on 127.0.0.1) and return
    their exit status: `--gpus N` outside torchrun never times one GPU under an N-GPU label."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def check_world(gpus: int, world: int) -> None:
    """The ranks that run must be the GPUs the line will report."""
    if world != gpus:
        raise SystemExit(f"bench.py: --gpus {gpus} but {world} ranks were launched")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="lowbit", choices=["lowbit", "reference"])
    ap.add_argument("--ref-rows", type=int, default=32, help="activation rows per shape in the CPU oracle sample")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--per-shape", action="store_true", help="print per-shape launch times to stderr")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-launch results of the other reference configurations (default workload)")
    ap.add_argument("--only-linear", default="", help="comma-separated indices of the workload's linears to run "
                                                      "(profiling one shape); default all")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    if "WORLD_SIZE" not in os.environ and args.gpus > 1:
        if args.impl == "lowbit":
            import torch
            if torch.cuda.device_count() < args.gpus:
                raise SystemExit(f"bench.py: --gpus {args.gpus} but {torch.cuda.device_count()} GPUs are visible")
        return relaunch_under_torchrun(args.gpus, sys.argv[1:])
    check_world(args.gpus, int(os.environ.get("WORLD_SIZE", "1")))
    specs = synth.WORKLOADS[args.workload]
    if args.only_linear:
        specs = [specs[int(i)] for i in args.only_linear.split(",")]
        args.workload = f"{args.workload}[{args.only_linear}]"
    if args.impl == "reference":
        return run_reference(args, specs, args.workload)
    return run_lowbit(args, specs, args.workload)


if __name__ == "__main__":
    sys.exit(main())
