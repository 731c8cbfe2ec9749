#!/usr/bin/env python
"""Benchmark of the MX hot path on B200: the cast (GB/s against HBM) and the
block-scaled GEMM (TFLOP/s against the tensor cores).

Default workload (one "step"): the cast bandwidth sweep -- one bf16
8192 x 8192 tensor (N(0,1), 0.01% outliers x 1e3) cast along rows to all six
element formats (E4M3, E5M2, E2M3, E3M2, E2M1, INT8), RNE, MMA scale layout.
Inputs rotate over three device copies (3 x 128 MiB > the 126 MB L2) so no cast
reads its input from L2.  `value` = algorithmic bytes of all casts / device
time (GB/s).  The same line carries a "gemm" object: the Llama-3-8B-shaped
MXFP4 GEMMs (M=8192: 4096->6144, 4096->14336, 14336->4096, bf16 out) timed the
same way on operands cast in advance.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mx|reference]

Multi-GPU: one process per GPU (torchrun); each rank runs the same per-GPU
workload on its own data (weak scaling, no data-path collective); the time is
the max over ranks.  `--impl reference` times the CPU oracle on a bounded
sample of the same workload (rank 0 only).
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

METRIC = "MX cast GB/s vs HBM peak; MX GEMM TFLOP/s vs block-scaled tensor peak"
FMTS = ["e4m3", "e5m2", "e2m3", "e3m2", "e2m1", "int8"]
BITS = {"e4m3": 8, "e5m2": 8, "e2m3": 6, "e3m2": 6, "e2m1": 4, "int8": 8}
ROWS = COLS = 8192
N_ROTATE = 3
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic per launch (dram__bytes_read.sum + dram__bytes_write.sum) of
# the roofline kernels, from one ncu capture of this benchmark's own launches
# (summaries under profiles/).  Each entry holds the kernel
# sources, the sha256 of their contents at capture time and bytes per launch
# by workload.  A figure is reported only while the sources still hash to that
# value; after any change to them it reads null until captured again.
_CSRC = os.path.join(ROOT, "microscaling_block_scaled_mx_b200", "csrc")
MEASURED_TRAFFIC = {
    # the third of three consecutive casts of one format captured with
    # --cache-control none, so each launch also carries the write-back of its
    # predecessor's output still in L2 (steady state: reads + writes of one cast)
    "cast_rows": (("mx_cast.cu", "mx_device.cuh", "mx_encode.cuh"),
                  "8b734928cc1e08710e6c1619c3ea512a525f233816c157ec451316e7aef9c23a",
                  {"e4m3_bf16_8192x8192": 134282752 + 70009600, "e5m2_bf16_8192x8192": 134250496 + 66572800,
                   "e2m3_bf16_8192x8192": 134224640 + 53562112, "e3m2_bf16_8192x8192": 134220544 + 52639744,
                   "e2m1_bf16_8192x8192": 134220288 + 36188160, "int8_bf16_8192x8192": 134219776 + 68327680}),
    # the GEMMs: default cache control (L2 flushed before the launch), so reads
    # show re-reads and writes count only what left L2 during the launch; "x4":
    # operands with x4 scales
    "gemm": (("mx_gemm.cu", "mx_encode.cuh"),
             "6857d04b731b1d6b91f472390b0595c1f8be37ebd11ed4d86eb7c5ae9c88039c",
             {"e2m1_x4_8192x6144x4096": 37304320 + 56930816, "e2m1_x4_8192x14336x4096": 59648768 + 188995584,
              "e2m1_x4_8192x4096x14336": 140673536 + 52436736, "e4m3_8192x3072x768": 8976384 + 1790208,
              "e4m3_8192x768x3072": 28427264 + 0, "e2m1_x4_4096x14336x16384": 456610048 + 210655232}),
}


# Warp instructions per value of the column (Hadamard + SR) cast kernels, from
# ncu's smsp__inst_executed.sum on one launch divided by the launch's values;
# the same source-hash rule as MEASURED_TRAFFIC.  They give the instruction-
# issue roofline of those casts: at most 4 warp instructions per clock per SM.
MEASURED_INSTR = {
    "cast_cols_had_sr": (("mx_cast.cu", "mx_device.cuh", "mx_encode.cuh"),
                         "8b734928cc1e08710e6c1619c3ea512a525f233816c157ec451316e7aef9c23a",
                         {"e2m1_bf16_x4_16384x4096": 27130504 / (16384 * 4096),
                          "e2m1_bf16_x4_16384x14336": 94438024 / (16384 * 14336)}),
    "cast_dual_had_sr": (("mx_cast.cu", "mx_device.cuh", "mx_encode.cuh"),
                         "8b734928cc1e08710e6c1619c3ea512a525f233816c157ec451316e7aef9c23a",
                         {"e2m1_bf16_16384x4096": 40931272 / (16384 * 4096),
                          "e2m1_bf16_16384x14336": 142829512 / (16384 * 14336)}),
}


def measured_instr(kernel: str, workload: str):
    names, sha, table = MEASURED_INSTR[kernel]
    if sha is None or workload not in table or sources_sha256(names) != sha:
        return None
    return table[workload]


def issue_bound_us(instr_per_value: float, values: int, sms: int, sm_mhz: float) -> float:
    """Time at the instruction-issue roofline: every SM issues at most one warp
    instruction per clock on each of its four schedulers."""
    return instr_per_value * values / (sms * 4 * sm_mhz * 1e6) * 1e6


def sources_sha256(names) -> str:
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(_CSRC, n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(kernel: str, workload: str):
    names, sha, table = MEASURED_TRAFFIC[kernel]
    if sha is None or workload not in table or sources_sha256(names) != sha:
        return None
    return table[workload]


def cast_alg_bytes(fmt: str, rows: int = ROWS, cols: int = COLS, in_bytes: int = 2) -> int:
    """Bytes a cast must move: read the input once, write codes and E8M0 scales once."""
    n = rows * cols
    return n * in_bytes + n * BITS[fmt] // 8 + n // 32


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.samples = []
        if self.proc is None:
            return False
        time.sleep(0.2)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                self.samples.append({"sm": float(parts[1]), "max": float(parts[2]), "power": float(parts[3]),
                                     "hw_slowdown": parts[5], "hw_thermal": parts[6], "sw_thermal": parts[7],
                                     "sw_power_cap": parts[8]})
            except ValueError:
                continue
        return False

    def summary(self):
        s = getattr(self, "samples", [])
        if not s:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        busy = [x for x in s if x["power"] > 200] or s
        reasons = set()
        for x in busy:
            for k in ("hw_slowdown", "hw_thermal", "sw_thermal", "sw_power_cap"):
                if x[k].lower() == "active":
                    reasons.add({"hw_thermal": "hw_thermal_slowdown", "sw_thermal": "sw_thermal_slowdown"}.get(k, k))
        return {"sm_mhz": statistics.median(x["sm"] for x in busy), "sm_max_mhz": max(x["max"] for x in s),
                "samples": len(busy), "reasons": sorted(reasons)}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample
# ---------------------------------------------------------------------------

def oracle_cast_sample(rows: int, x=None):
    """Time the oracle casting `rows` rows of the sweep input to all six formats."""
    import oracle
    from microscaling_block_scaled_mx_b200 import inputs as I
    if x is None:
        x = I.cast_sweep_input(rows, COLS)
    oracle.build()
    t0 = time.perf_counter()
    for f in FMTS:
        oracle.quantize(x, 1, oracle.FORMATS[f], scale_layout=oracle.MMA)
    dt = time.perf_counter() - t0
    nbytes = sum(cast_alg_bytes(f, rows, COLS) for f in FMTS)
    return nbytes / dt / 1e9, dt, nbytes


def cpu_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from microscaling_block_scaled_mx_b200 import inputs as I
    # each step casts a bounded sample of rows, sized so that all steps take
    # about a minute of oracle time (between 32 and 512 rows per step)
    _, dt64, _ = oracle_cast_sample(64)        # also warms the library
    rows = int(60.0 / (args.steps * dt64 / 64)) // 32 * 32
    rows = max(32, min(512, rows))
    x = I.cast_sweep_input(rows, COLS)
    vals = []
    for _ in range(args.warmup):
        oracle_cast_sample(rows, x)
    t_total = 0.0
    nbytes = 0
    for _ in range(args.steps):
        v, dt, nb = oracle_cast_sample(rows, x)
        vals.append(v)
        t_total += dt
        nbytes += nb
    value = nbytes / t_total / 1e9
    sample = f"{rows} x {COLS} rows of the sweep input, six formats per step"
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t_total / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "cast_sweep_bf16_8192x8192_6fmt", "global_batch": args.gpus,
                       "parallelism": f"replicas{args.gpus}", "sampled_rows": rows},
            "cpu_baseline": {"value": round(value, 3), "unit": "GB/s", "cores": cpu_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 3), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# product arm
# ---------------------------------------------------------------------------

def run_mx(args):
    import torch
    import torch.distributed as dist
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200 import mx

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    from microscaling_block_scaled_mx_b200 import dist as mxdist
    barrier = mxdist.barrier

    def max_over_ranks(x: float) -> float:
        return mxdist.max_over_ranks(x, dev)

    peaks, peak_kind = load_peaks()
    stream = torch.cuda.current_stream()
    if args.only:
        # profiling: the named phases alone, on their own workloads (not a bench line)
        phases = {"gemm": lambda: run_gemm_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks,
                                                 world),
                  "gemm_fp8": lambda: run_gemm_phase(args, dev, stream, peaks, peak_kind, barrier,
                                                     max_over_ranks, world, fmt="e4m3"),
                  "wgrad": lambda: run_wgrad_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks,
                                                   world),
                  "dual": lambda: run_dual_phase(args, dev, stream, peaks, barrier, max_over_ranks, world),
                  "nvfp4": lambda: run_nvfp4_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks,
                                                   world)}
        names = args.only.split(",")
        if "cast" in names and len(names) > 1:
            raise SystemExit("--only cast runs alone")
        res = {name: phases[name]() for name in names if name != "cast"}
        if "cast" not in names:
            if rank == 0:
                print(json.dumps({"profiling_only": args.only, **res}), flush=True)
            if world > 1:
                dist.destroy_process_group()
            return 0
        args.no_gemm = args.no_wgrad = args.no_dual = args.no_nvfp4 = True
        args.no_e2e = args.no_cpu_baseline = True

    # ---- inputs (host generation, then resident in HBM) ----
    bits = I.cast_sweep_input(ROWS, COLS, seed_stream=rank)
    host = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)
    xs = [host.to(dev) for _ in range(N_ROTATE)]
    outs = {}
    for f in FMTS:
        outs[f] = [(torch.empty((ROWS, mx.codes_row_bytes(f, COLS)), dtype=torch.uint8, device=dev),
                    torch.empty(mx.scales_bytes("mma", ROWS, COLS), dtype=torch.uint8, device=dev))
                   for _ in range(N_ROTATE)]
    stream = torch.cuda.current_stream()

    def step(i):
        for j, f in enumerate(FMTS):
            r = (i * len(FMTS) + j) % N_ROTATE
            c, s = outs[f][r]
            mx.quantize(xs[r], 1, f, codes=c, scales=s, scale_layout="mma")

    def timed_region(body, n):
        """Milliseconds of n calls of body(i), events only at the two ends (an
        event between launches costs device time and lets the host fall behind)."""
        barrier()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(n):
            body(i)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(t0.elapsed_time(t1))

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()

    # timed region: K steps, barrier + synchronize on both sides
    with ClockSampler(local) as clocks:
        ms_total = timed_region(step, args.steps)
    launches = len(FMTS) * args.steps
    alg_bytes_step = sum(cast_alg_bytes(f) for f in FMTS)
    value = world * alg_bytes_step * args.steps / (ms_total * 1e-3) / 1e9

    # per format: a timed region of that cast alone (same input rotation)
    per_fmt = {}
    n_fmt = max(3 * N_ROTATE, min(args.steps, 300))
    for f in FMTS:
        def one(i, f=f):
            r = i % N_ROTATE
            c, s = outs[f][r]
            mx.quantize(xs[r], 1, f, codes=c, scales=s, scale_layout="mma")
        one(0)
        us = 1e3 * timed_region(one, n_fmt) / n_fmt
        launches += n_fmt
        per_fmt[f] = {"us": round(us, 2), "gbs": round(cast_alg_bytes(f) / (us * 1e-6) / 1e9, 1)}
    # the roofline kernel's average launch duration in the timed region above
    achieved = alg_bytes_step * args.steps / (ms_total * 1e-3) / 1e9
    hbm_peak = float(peaks["hbm_gbs"])
    traffic = None
    t_fmt = {f: measured_traffic("cast_rows", f"{f}_bf16_{ROWS}x{COLS}") for f in FMTS}
    if all(v is not None for v in t_fmt.values()):
        traffic = round(statistics.mean(t_fmt.values()))
        for f in FMTS:
            per_fmt[f]["traffic"] = t_fmt[f]
            per_fmt[f]["alg_bytes"] = cast_alg_bytes(f)
    roofline = {"bound": "hbm", "kernel": "cast_rows_kernel (six format instantiations)",
                "achieved": round(achieved, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(achieved / hbm_peak, 4), "peak_kind": f"{peak_kind} copy bandwidth (burst)",
                "traffic": traffic, "alg_bytes_per_launch": round(alg_bytes_step / len(FMTS)),
                "per_format": per_fmt}

    # ---- end to end through the C ABI with host buffers ----
    # The tensor streams through in row chunks on three streams: the host->device
    # copy of chunk i+1 and the device->host copy of chunk i-1 overlap the six
    # casts of chunk i (the two copy directions use separate engines).  Each
    # chunk's outputs (codes and plain-layout scales of all six formats) sit
    # contiguously in one device buffer, so they return to pinned host memory
    # in one copy per chunk.
    pinned = host.pin_memory()
    E2E_CHUNKS = 8
    rows_c = ROWS // E2E_CHUNKS
    seg = []                                   # (format, codes offset, scales offset) inside a chunk
    off = 0
    for f in FMTS:
        cb = rows_c * mx.codes_row_bytes(f, COLS)
        sb = mx.scales_bytes("plain", rows_c, COLS)
        seg.append((f, off, off + cb, sb))
        off += cb + sb
        off = (off + 255) // 256 * 256         # keep every slice 256-byte aligned
    chunk_bytes = off
    dev_chunks = [torch.empty(chunk_bytes, dtype=torch.uint8, device=dev) for _ in range(E2E_CHUNKS)]
    host_chunks = torch.empty((E2E_CHUNKS, chunk_bytes), dtype=torch.uint8).pin_memory()
    d2h = E2E_CHUNKS * chunk_bytes
    h2d = pinned.numel() * 2
    s_in, s_cast, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_step():
        s_in.wait_stream(stream)      # each step starts after the previous one ended
        for i in range(E2E_CHUNKS):
            r0, r1 = i * rows_c, (i + 1) * rows_c
            with torch.cuda.stream(s_in):
                xs[0][r0:r1].copy_(pinned[r0:r1], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(s_in)
            with torch.cuda.stream(s_cast):
                s_cast.wait_event(ev)
                buf = dev_chunks[i]
                for (f, co, so, sb) in seg:
                    c = buf[co:so].view(rows_c, -1)
                    mx.quantize(xs[0][r0:r1], 1, f, codes=c, scales=buf[so:so + sb], scale_layout="plain",
                                stream=s_cast)
                evc = torch.cuda.Event()
                evc.record(s_cast)
            with torch.cuda.stream(s_out):
                s_out.wait_event(evc)
                host_chunks[i].copy_(dev_chunks[i], non_blocking=True)
        stream.wait_stream(s_out)

    e2e_steps = min(args.steps, 50)
    e2e_val = None
    if not args.no_e2e:
        for _ in range(args.warmup):
            e2e_step()
        torch.cuda.synchronize()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1))
        e2e_val = world * alg_bytes_step * e2e_steps / (e2e_ms * 1e-3) / 1e9

    gemm = run_gemm_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks, world)
    if gemm is not None:
        launches_gemm = gemm.pop("_launches")
    else:
        launches_gemm = 0
    gemm8 = run_gemm_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks, world, fmt="e4m3")
    if gemm8 is not None:
        launches_gemm += gemm8.pop("_launches")
    wgrad = None if args.no_wgrad else run_wgrad_phase(args, dev, stream, peaks, peak_kind, barrier,
                                                        max_over_ranks, world)
    dual = None if args.no_dual else run_dual_phase(args, dev, stream, peaks, barrier, max_over_ranks, world)
    if dual is not None:
        launches_gemm += dual.pop("_launches")
    nvfp4 = None if args.no_nvfp4 else run_nvfp4_phase(args, dev, stream, peaks, peak_kind, barrier,
                                                        max_over_ranks, world)
    if nvfp4 is not None:
        launches_gemm += nvfp4.pop("_launches")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, dt, nb = oracle_cast_sample(2048)
        cpu = {"value": round(v, 3), "unit": "GB/s", "cores": cpu_threads(), "kind": "oracle",
               "sample": f"2048 x {COLS} rows of the sweep input cast to all six formats ({dt:.1f} s wall)"}

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_total / args.steps, 4),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic",
                "config": {"workload": "cast_sweep_bf16_8192x8192_6fmt", "global_batch": world,
                           "seq_len": None, "parallelism": f"replicas{world}",
                           "formats": FMTS, "block_axis": "rows", "rounding": "rne",
                           "l2": f"inputs rotate over {N_ROTATE} device buffers of 128 MiB (> L2)"},
                "roofline": roofline,
                "cpu_baseline": cpu,
                "e2e": None if e2e_val is None else
                       {"value": round(e2e_val, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                        "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                        "path": "pinned host bf16 -> H2D -> mx_quantize (6 formats) -> D2H codes+scales, "
                                "8 row chunks pipelined over 3 streams, one D2H copy per chunk"},
                "gpu_launches": launches + launches_gemm,
                "clocks": clocks.summary()}
        if gemm is not None:
            line["gemm"] = gemm
        if gemm8 is not None:
            line["gemm_fp8"] = gemm8
        if wgrad is not None:
            line["wgrad"] = wgrad
        if dual is not None:
            line["dual_cast"] = dual
        if nvfp4 is not None:
            line["nvfp4"] = nvfp4
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_gemm_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks, world, fmt="e2m1"):
    """Block-scaled GEMMs on operands cast in advance: the Llama-3-8B-shaped
    MXFP4 set (fmt e2m1) or the GPT-2-small-shaped MXFP8 set (fmt e4m3); None
    if the GEMM is not available in this build."""
    import torch
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200 import mx
    if args.no_gemm:
        return None
    shapes = I.LLAMA3_GEMMS if fmt == "e2m1" else I.GPT2_GEMMS
    cfg_index = 3 if fmt == "e2m1" else 2
    # MXFP4 operands carry x4 scales (the pair kernel's cheaper scale copies);
    # the short-K MXFP8 shapes keep the MMA layout and the one-SM kernel
    sl = "mma_x4" if fmt == "e2m1" else "mma"
    ops = []
    for idx, (M, N, K) in enumerate(shapes):
        if fmt == "e2m1" and str(idx) not in args.gemm_shapes.split(","):
            continue
        xb, wb = I.linear_operands(M, K, N, cfg_index, stream=idx)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(dev)
        ac, as_ = mx.quantize(x, 1, fmt, scale_layout=sl)
        bc, bs = mx.quantize(w, 1, fmt, scale_layout=sl)
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ops.append((M, N, K, ac, as_, bc, bs, c))
        del x, w
    try:
        M, N, K, ac, as_, bc, bs, c = ops[0]
        mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)
    except mx.MxError as e:
        if e.status == -4:
            return None
        raise
    flops_step = sum(2.0 * M * N * K for (M, N, K, *_r) in ops)
    for _ in range(args.warmup):
        for (M, N, K, ac, as_, bc, bs, c) in ops:
            mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)
    torch.cuda.synchronize()

    def timed_region(body, n):
        barrier()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(n):
            body(i)
        t1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(t0.elapsed_time(t1))

    def step(i):
        for (M, N, K, ac, as_, bc, bs, c) in ops:
            mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)

    with ClockSampler(dev.index or 0) as clk:
        ms = timed_region(step, args.steps)
    clocks = clk.summary()
    launches = len(ops) * args.steps
    value = world * flops_step * args.steps / (ms * 1e-3) / 1e12
    per_shape = {}
    n_shape = max(3, min(args.steps, 200))
    for (M, N, K, ac, as_, bc, bs, c) in ops:
        def one(i, M=M, N=N, K=K, ac=ac, as_=as_, bc=bc, bs=bs, c=c):
            mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)
        us = 1e3 * timed_region(one, n_shape) / n_shape
        launches += n_shape
        per_shape[f"{M}x{N}x{K}"] = {"us": round(us, 1), "tflops": round(2.0 * M * N * K / (us * 1e-6) / 1e12, 1)}
    traffic = None
    t_shape = {k: measured_traffic("gemm", f"{fmt}_{'x4_' if sl == 'mma_x4' else ''}{k}") for k in per_shape}
    if all(v is not None for v in t_shape.values()):
        traffic = round(statistics.mean(t_shape.values()))
        for k in per_shape:
            per_shape[k]["traffic"] = t_shape[k]
    # all launches of the timed region are this kernel: its average launch duration
    achieved = flops_step * args.steps / (ms * 1e-3) / 1e12
    # the same GEMMs with C quantized in the epilogue (to the operand format, along
    # N: the next layer's A operand) against the GEMM followed by a row cast of C
    fused = {}
    q_steps = max(3, min(args.steps, 20))
    for (M, N, K, ac, as_, bc, bs, c) in ([] if args.no_fused else ops):
        qc = torch.empty((M, mx.codes_row_bytes(fmt, N)), dtype=torch.uint8, device=dev)
        qs = torch.empty(mx.scales_bytes("mma", M, N), dtype=torch.uint8, device=dev)
        res = {}
        for label in ("gemm_then_cast", "fused"):
            def once(label=label, M=M, N=N, K=K, ac=ac, as_=as_, bc=bc, bs=bs, c=c, qc=qc, qs=qs):
                if label == "fused":
                    mx.gemm_quantize(ac, as_, bc, bs, M, N, K, fa=fmt, out_fmt=fmt, out=(qc, qs),
                                     operand_layout=sl)
                else:
                    mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)
                    mx.quantize(c, 1, fmt, codes=qc, scales=qs)
            for _ in range(args.warmup):
                once()
            torch.cuda.synchronize()
            barrier()
            q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            q0.record(stream)
            for _ in range(q_steps):
                once()
            q1.record(stream)
            torch.cuda.synchronize()
            barrier()
            res[label] = max_over_ranks(1e3 * q0.elapsed_time(q1) / q_steps)
            launches += q_steps * (1 if label == "fused" else 2)
        fused[f"{M}x{N}x{K}"] = {"gemm_then_cast_us": round(res["gemm_then_cast"], 1),
                                 "fused_us": round(res["fused"], 1),
                                 "speedup": round(res["gemm_then_cast"] / res["fused"], 3)}
    ratio = 4.0 if fmt == "e2m1" else 2.0             # nominal fp4 : fp8 : bf16 = 9 : 4.5 : 2.25
    # A GEMM loop of a quarter second or more runs into the board's power cap
    # and settles at the sustained clock: the sustained cuBLAS figure is its
    # denominator then, the burst one for a shorter loop.
    sustained = ms >= 250.0
    peak = ratio * float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
    if fmt == "e2m1":
        workload = ("llama3_8b_mxfp4_gemms_m8192 (4096->6144, 4096->14336, 14336->4096), bf16 out, "
                    "x4 operand scales")
        kernel = "mx_gemm_pair_kernel (cta_group::2, kind::mxf4, x4 scales)"
    else:
        workload = "gpt2_small_mxfp8_gemms_m8192 (768->3072, 3072->768), bf16 out"
        kernel = ("mx_gemm_panel_kernel (768->3072: resident B panel) and mx_gemm_kernel (3072->768); "
                  "cta_group::1, kind::mxf8f6f4")
    # Llama-3 "quantized along K, and again along M": the first shape's
    # activation X (8192 x 4096) and output C (8192 x 6144, bf16) cast with
    # blocks along M (tokens, transposed out), and the weight-gradient-shaped
    # product C^T X contracting over the 8192 tokens
    along_m = None
    if fmt == "e2m1" and ops and not args.no_fused:
        M, N, K, ac, as_, bc, bs, c = ops[0]
        xb, _ = I.linear_operands(M, K, N, cfg_index, stream=0)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        mx.gemm(ac, as_, bc, bs, M, N, K, fa=fmt, out=c, scale_layout=sl)
        xc, xs = mx.quantize(x, 0, fmt, scale_layout=sl)         # K x M codes: x^T along tokens
        cc, cs = mx.quantize(c, 0, fmt, scale_layout=sl)         # N x M codes: C^T along tokens
        ct = torch.empty((N, K), dtype=torch.float32, device=dev)
        steps_m = max(3, min(args.steps, 20))
        timings = {}
        for label, fn in (("cast_x_along_m", lambda: mx.quantize(x, 0, fmt, codes=xc, scales=xs, scale_layout=sl)),
                          ("cast_c_along_m", lambda: mx.quantize(c, 0, fmt, codes=cc, scales=cs, scale_layout=sl)),
                          ("gemm_ct_x", lambda: mx.gemm(cc, cs, xc, xs, N, K, M, fa=fmt, out=ct, scale_layout=sl))):
            for _ in range(args.warmup):
                fn()
            timings[label] = 1e3 * timed_region(lambda i, fn=fn: fn(), steps_m) / steps_m
            launches += steps_m
        along_m = {"workload": f"X {M}x{K} and C {M}x{N} bf16 cast along M to E2M1 (RNE, x4 scales); "
                               f"C^T X = {N}x{K}x{M}, fp32 out"}
        for label, n in (("cast_x_along_m", M * K), ("cast_c_along_m", M * N)):
            alg = n * 2 + n // 2 + n // 32
            along_m[label] = {"us": round(timings[label], 1), "gbs": round(alg / (timings[label] * 1e-6) / 1e9, 1)}
        along_m["gemm_ct_x"] = {"us": round(timings["gemm_ct_x"], 1),
                                "tflops": round(2.0 * N * K * M / (timings["gemm_ct_x"] * 1e-6) / 1e12, 1)}
        del x, xc, xs, cc, cs, ct
    return {"metric": "MX GEMM TFLOP/s", "value": round(value, 1), "unit": "TFLOP/s",
            "workload": workload, "ms_per_step": round(ms / args.steps, 4),
            "roofline": {"bound": "tensor", "kernel": kernel,
                         "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4),
                         "peak_kind": f"{peak_kind} bf16 {'sustained' if sustained else 'burst'} x {ratio:g} "
                                      f"(nominal ratio for the operand type; timed loop {ms:.0f} ms)",
                         "clocks": clocks, "traffic": traffic, "per_shape": per_shape},
            "quantizing_epilogue": fused,
            "along_m": along_m,
            "_launches": launches}


def run_wgrad_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks, world):
    """Weight-gradient step: dY 16384x4096 and X 16384x14336 (bf16, Student-t)
    cast along tokens with the fixed-sign Hadamard and stochastic rounding to
    E2M1, then dW = dY^T X / 32 in fp32.  Times the two casts and the GEMM."""
    import torch
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200 import mx
    dyb, xb = I.wgrad_operands()
    T, Do = dyb.shape
    Di = xb.shape[1]
    dy = torch.from_numpy(dyb.view(np.int16)).view(torch.bfloat16).to(dev)
    x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
    del dyb, xb
    ac = torch.empty((Do, T // 2), dtype=torch.uint8, device=dev)
    as_ = torch.empty(mx.scales_bytes("mma_x4", Do, T), dtype=torch.uint8, device=dev)
    bc = torch.empty((Di, T // 2), dtype=torch.uint8, device=dev)
    bs = torch.empty(mx.scales_bytes("mma_x4", Di, T), dtype=torch.uint8, device=dev)
    dw = torch.empty((Do, Di), dtype=torch.float32, device=dev)
    # x4 scales for the dW GEMM (the pair kernel's cheaper scale copies)
    ops = {"cast_dY": lambda: mx.quantize(dy, 0, "e2m1", rnd="sr", seed=42, hadamard=True, codes=ac, scales=as_,
                                          scale_layout="mma_x4"),
           "cast_X": lambda: mx.quantize(x, 0, "e2m1", rnd="sr", seed=43, hadamard=True, codes=bc, scales=bs,
                                         scale_layout="mma_x4"),
           "gemm_dW": lambda: mx.gemm(ac, as_, bc, bs, Do, Di, T, fa="e2m1", alpha=1.0 / 32, out=dw,
                                      scale_layout="mma_x4")}

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(e0.elapsed_time(e1))

    steps = max(3, min(args.steps, 20))
    for _ in range(args.warmup):
        for fn in ops.values():
            fn()
    torch.cuda.synchronize()
    ms = timed(lambda: [fn() for fn in ops.values()], steps)      # the whole step
    with ClockSampler(dev.index or 0) as clk:
        us = {k: 1e3 * timed(fn, steps) / steps for k, fn in ops.items()}
    sm_mhz = clk.summary()["sm_mhz"] or 1965.0
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    cast_bytes = {"cast_dY": T * Do * 2 + T * Do // 2 + T * Do // 32,
                  "cast_X": T * Di * 2 + T * Di // 2 + T * Di // 32}
    flops = 2.0 * Do * Di * T
    fp4_peak = 4.0 * float(peaks["bf16_tflops"])
    hbm = float(peaks["hbm_gbs"])
    out = {"workload": "wgrad_mxfp4 dY 16384x4096, X 16384x14336 (Student-t), Hadamard+SR along tokens, "
                       "x4 scales, dW fp32", "steps": steps, "ms_per_step": round(ms / steps, 4)}
    values = {"cast_dY": T * Do, "cast_X": T * Di}
    shape = {"cast_dY": f"{T}x{Do}", "cast_X": f"{T}x{Di}"}
    for k in ("cast_dY", "cast_X"):
        gbs = cast_bytes[k] / (us[k] * 1e-6) / 1e9
        hbm_us = cast_bytes[k] / (hbm * 1e9) * 1e6
        out[k] = {"us": round(us[k], 1), "gbs": round(gbs, 1), "frac_hbm": round(gbs / hbm, 4)}
        ipv = measured_instr("cast_cols_had_sr", f"e2m1_bf16_x4_{shape[k]}")
        if ipv is not None:
            alu_us = issue_bound_us(ipv, values[k], sms, sm_mhz)
            out[k]["alu"] = {"warp_instr_per_value": round(ipv, 4), "bound_us": round(alu_us, 1), "sm_mhz": sm_mhz,
                             "frac": round(alu_us / us[k], 4)}
            # the roofline is the slower of the two bounds
            out[k]["roofline"] = {"bound": "alu" if alu_us > hbm_us else "hbm",
                                  "frac": round(max(alu_us, hbm_us) / us[k], 4)}
    tf = flops / (us["gemm_dW"] * 1e-6) / 1e12
    out["gemm_dW"] = {"us": round(us["gemm_dW"], 1), "tflops": round(tf, 1), "frac": round(tf / fp4_peak, 4),
                      "peak": round(fp4_peak, 1), "traffic": measured_traffic("gemm", f"e2m1_x4_{Do}x{Di}x{T}")}
    return out


def run_dual_phase(args, dev, stream, peaks, barrier, max_over_ranks, world):
    """Dual cast of the weight-gradient operands (dY 16384x4096, X 16384x14336,
    bf16): E2M1 codes along rows (RNE, for the forward and data-gradient GEMMs)
    and along tokens (Hadamard + SR, for the weight-gradient GEMM) from one
    read, timed against the two single-axis casts that produce the same bytes."""
    import torch
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200 import mx
    dyb, xb = I.wgrad_operands()
    rng = np.random.default_rng(1004)
    act = I.to_bf16_bits(rng.standard_normal((8192, 4096)).astype(np.float32))
    # (name, tensor, format, column rounding, Hadamard on the column output)
    cases = [("dY", dyb, "e2m1", "sr", True), ("X", xb, "e2m1", "sr", True),
             ("act_e4m3", act, "e4m3", "rne", False)]
    ops = []
    for name, bits, f, rc, had in cases:
        t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
        out = mx.quantize_dual(t, f, rnd_rows="rne", rnd_cols=rc, seed_cols=42, hadamard=had)
        ops.append((name, t, f, rc, had, out))
    del dyb, xb, act
    launches = 0

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(1e3 * e0.elapsed_time(e1) / n)

    steps = max(3, min(args.steps, 20))
    hbm = float(peaks["hbm_gbs"])
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    out = {"workload": "dual cast: dY 16384x4096 and X 16384x14336 bf16 to E2M1 (rows RNE, tokens Hadamard+SR); "
                       "Llama-3 activation 8192x4096 bf16 to E4M3 (RNE both axes)", "steps": steps}
    for name, t, f, rc, had, o in ops:
        def dual(t=t, f=f, rc=rc, had=had, o=o):
            mx.quantize_dual(t, f, rnd_rows="rne", rnd_cols=rc, seed_cols=42, hadamard=had, out=o)

        def two(t=t, f=f, rc=rc, had=had, o=o):
            mx.quantize(t, 1, f, codes=o[0], scales=o[1])
            mx.quantize(t, 0, f, rnd=rc, seed=42, hadamard=had, codes=o[2], scales=o[3])
        for _ in range(args.warmup):
            dual()
            two()
        with ClockSampler(dev.index or 0) as clk:
            d, s2 = timed(dual, steps), timed(two, steps)
        sm_mhz = clk.summary()["sm_mhz"] or 1965.0
        launches += 3 * steps
        n = t.numel()
        bits = mx.FMT_BITS[mx.FMT[f]]
        alg = n * 2 + 2 * (n * bits // 8 + n // 32)        # one read, two sets of codes and scales
        out[name] = {"dual_us": round(d, 1), "two_casts_us": round(s2, 1), "speedup": round(s2 / d, 3),
                     "dual_gbs": round(alg / (d * 1e-6) / 1e9, 1),
                     "frac_hbm": round(alg / (d * 1e-6) / 1e9 / hbm, 4)}
        ipv = measured_instr("cast_dual_had_sr", f"{f}_bf16_{t.shape[0]}x{t.shape[1]}") if had else None
        if ipv is not None:
            alu_us = issue_bound_us(ipv, n, sms, sm_mhz)
            hbm_us = alg / (hbm * 1e9) * 1e6
            out[name]["alu"] = {"warp_instr_per_value": round(ipv, 4), "bound_us": round(alu_us, 1),
                                "sm_mhz": sm_mhz, "frac": round(alu_us / d, 4)}
            out[name]["roofline"] = {"bound": "alu" if alu_us > hbm_us else "hbm",
                                     "frac": round(max(alu_us, hbm_us) / d, 4)}
    out["_launches"] = launches
    return out


def run_nvfp4_phase(args, dev, stream, peaks, peak_kind, barrier, max_over_ranks, world):
    """NVFP4 (16-element E2M1 blocks, E4M3 block scales, one fp32 encode scale
    per domain): the cast of a Llama-3-8B activation 8192 x 4096 bf16 with a
    global domain and with CTA-local domains of 128 rows, and the three
    Llama-3-8B GEMM shapes on NVFP4 operands (activations CTA-local, weights
    global), bf16 out."""
    import torch
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200 import mx
    local_rows = 128
    steps = max(3, min(args.steps, 50))
    hbm = float(peaks["hbm_gbs"])
    fp4_peak = 4.0 * float(peaks["bf16_tflops"])
    launches = 0

    def timed(fn, n):
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        return max_over_ranks(1e3 * e0.elapsed_time(e1) / n)

    out = {"workload": "nvfp4: cast of a Llama-3-8B activation 8192x4096 bf16 (global, and CTA-local "
                       f"domains of {local_rows} rows), MMA scale layout; Llama-3-8B GEMMs M=8192 on NVFP4 "
                       "operands (activations CTA-local, weights global, x4 scales), bf16 out", "steps": steps}
    # cast: inputs rotate over three device copies (> L2)
    xb, _ = I.linear_operands(8192, 4096, 128, 3, stream=0)
    xs = [torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev) for _ in range(N_ROTATE)]
    rows, cols = xs[0].shape
    cast = {}
    for label, dom in (("global", 0), ("cta_local", local_rows)):
        bufs = [mx.quantize_nvfp4(x, dom) for x in xs]
        it = [0]

        def one(dom=dom, bufs=bufs, it=it):
            r = it[0] % N_ROTATE
            it[0] += 1
            mx.quantize_nvfp4(xs[r], dom, out=bufs[r])
        for _ in range(args.warmup):
            one()
        us = timed(one, steps)
        launches += steps * 3
        n = rows * cols
        alg = n * 2 + n // 2 + n // 16 + 4 * mx.lib().mx_nvfp4_domains(rows, dom)
        cast[label] = {"us": round(us, 1), "gbs": round(alg / (us * 1e-6) / 1e9, 1),
                       "frac_hbm": round(alg / (us * 1e-6) / 1e9 / hbm, 4),
                       "kernels": "nv_amax + nv_quant + nv_final"}
    out["cast"] = cast
    del xs
    gemm = {}
    total_flops = total_us = 0.0
    for idx, (M, N, K) in enumerate(I.LLAMA3_GEMMS):
        xb, wb = I.linear_operands(M, K, N, 3, stream=idx)
        x = torch.from_numpy(xb.view(np.int16)).view(torch.bfloat16).to(dev)
        w = torch.from_numpy(wb.view(np.int16)).view(torch.bfloat16).to(dev)
        a = mx.quantize_nvfp4(x, local_rows, scale_layout="mma_x4")
        b = mx.quantize_nvfp4(w, 0, scale_layout="mma_x4")
        c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        del x, w

        def g(a=a, b=b, c=c, M=M, N=N, K=K):
            mx.gemm_nvfp4(a, b, M, N, K, local_rows, 0, out=c, scale_layout="mma_x4")
        for _ in range(args.warmup):
            g()
        us = timed(g, steps)
        launches += steps
        fl = 2.0 * M * N * K
        total_flops += fl
        total_us += us
        tf = fl / (us * 1e-6) / 1e12
        gemm[f"{M}x{N}x{K}"] = {"us": round(us, 1), "tflops": round(tf, 1), "frac": round(tf / fp4_peak, 4)}
    out["gemm"] = {"kernel": "mx_gemm_pair_kernel (cta_group::2, kind::mxf4nvf4, scale_vec::4X, x4 scales)",
                   "per_shape": gemm, "tflops": round(total_flops / (total_us * 1e-6) / 1e12, 1),
                   "peak": round(fp4_peak, 1),
                   "peak_kind": f"{peak_kind} bf16 burst x 4 (nominal ratio for FP4 operands)"}
    out["_launches"] = launches
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mx", "reference"], default="mx")
    ap.add_argument("--no-gemm", action="store_true", help="skip the GEMM phase")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end phase")
    ap.add_argument("--only", default="", help="profiling: comma-separated phases to run alone "
                    "(cast, gemm, gemm_fp8, wgrad, dual, nvfp4)")
    ap.add_argument("--no-wgrad", action="store_true", help="skip the weight-gradient phase")
    ap.add_argument("--no-dual", action="store_true", help="skip the dual-cast phase")
    ap.add_argument("--no-nvfp4", action="store_true", help="skip the NVFP4 phase")
    ap.add_argument("--no-fused", action="store_true", help="skip the quantizing-epilogue comparison")
    ap.add_argument("--fmts", default=",".join(FMTS), help="comma-separated cast formats (profiling)")
    ap.add_argument("--gemm-shapes", default="0,1,2", help="indices of the Llama-3 GEMM shapes to time")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)      # at least three untimed warm-up steps
    FMTS[:] = [f for f in args.fmts.split(",") if f]
    if args.impl == "reference":
        return run_reference(args)
    return run_mx(args)


if __name__ == "__main__":
    sys.exit(main())
