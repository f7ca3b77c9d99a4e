#!/usr/bin/env python3
"""Benchmark: fused decode-GEMV over losslessly compressed BF16 weights on B200.

Default workload: the Llama-3.1-8B-shaped stack (32 layers of q, k, v, o, gate,
up, down plus the lm_head, 7.5 G weights), the largest configuration that fits
one GPU.  One step = one token: every GEMV of the stack, captured as one CUDA
graph, with x and y resident in HBM and every layer larger than L2.  As the NWC
page runs its models, the projections that read the same input are fused
(q, k, v into one matrix, gate and up into another: 4 calls per layer);
--no-fuse runs all 7.  With a
single-matrix workload (--workload attn_4096_outliers, ...) one step is one
nwc_gemv call, rotating over enough compressed copies that the weights never
sit in L2 (126 MB).  Exactly --steps steps are timed; when they take less than
half a second the timed region is repeated and the median is reported.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--batch B]
    python bench.py --impl reference ...   # the CPU oracle on the host cores

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun, one rank per GPU) are
independent replicas: every rank runs the same per-GPU work, with no collective
on the data path (weak scaling); time is the max over ranks.
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

METRIC = ("fused decode-GEMV µs/call, effective GB/s & % of B200 HBM peak; "
          "compression ratio")
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024
KERNEL_SOURCE = os.path.join(ROOT, "lossless_bf16_weight_nwc_b200", "csrc", "kernels.cu")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 50 tokens for a stack; 20000 calls for a matrix)")
    ap.add_argument("--warmup", type=int, default=None,
                    help="untimed warm-up steps (default 5 tokens; 200 calls), at least 3")
    ap.add_argument("--impl", default="nwc", choices=["nwc", "reference"])
    ap.add_argument("--workload", default="llama31_8b_stack")
    ap.add_argument("--min-region-s", type=float, default=0.5,
                    help="repeat the timed region until this much time is covered")
    ap.add_argument("--batch", type=int, default=1)
    ap.add_argument("--graph-calls", type=int, default=0,
                    help="calls per captured graph (0 = one pass over the rotating copies)")
    ap.add_argument("--no-cublas", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=2000)
    ap.add_argument("--e2e-mode", default="host-y", choices=["copy", "host-y"],
                    help="how y reaches the host in the end-to-end leg")
    ap.add_argument("--streams", type=int, default=1, choices=[1, 2],
                    help="bit streams per lane and tile of the compressed matrices")
    ap.add_argument("--code", default="prefix", choices=["prefix", "rank", "escape"],
                    help="exponent code: the length-limited prefix code (NWB1), the ranked "
                         "unary code (NWR1, 7 ranks) or the prefix code of the 16 most "
                         "frequent exponents with verbatim runs for the rest (NWE1)")
    ap.add_argument("--lmax", type=int, default=0,
                    help="code length limit of the compressed matrices (0: the library's "
                         "automatic choice, 7 unless a matrix has more than 128 exponents; "
                         "8..12 take the 16 KiB table of 12-bit peeks)")
    ap.add_argument("--tc-min-batch", type=int, default=None,
                    help="smallest batch that takes the tensor-core kernel (default: the "
                         "library's, 17; 0 = never)")
    ap.add_argument("--report", action="store_true",
                    help="the five configurations as a markdown table (not the headline line)")
    ap.add_argument("--report-json", default=None, help="with --report: every line, to this file")
    ap.add_argument("--fuse", dest="fuse", action="store_true", default=True,
                    help="stacks: q, k, v and gate, up each run as one stacked matrix (the "
                         "default)")
    ap.add_argument("--no-fuse", dest="fuse", action="store_false",
                    help="stacks: every projection its own matrix and call")
    ap.add_argument("--shard", action="store_true",
                    help="one matrix split by output rows over the ranks (ShardedMatrix): "
                         "each rank decodes its rows, then one NCCL all-gather of y per "
                         "step (strong scaling); default: independent replicas")
    return ap.parse_args()


def measured_peaks() -> tuple[dict, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return {"hbm_gbs": FALLBACK_HBM_GBS}, "fallback"


def kernel_source_hash() -> str:
    """Hash of the kernel source's code: '//' comments, trailing blanks and
    empty lines are dropped, so that a comment edit keeps a capture valid while
    any change to the code itself does not."""
    lines = []
    with open(KERNEL_SOURCE, encoding="utf-8") as f:
        for line in f:
            code = line.split("//", 1)[0].rstrip()
            if code:
                lines.append(code)
    return hashlib.sha256("\n".join(lines).encode()).hexdigest()[:16]


def format_suffix(args) -> str:
    """Key suffix of a non-default compressed format in the traffic summary."""
    return ("" if args.code == "prefix" else f"_{args.code}") + \
        ("" if args.streams == 1 else f"_s{args.streams}") + \
        ("" if not getattr(args, "lmax", 0) else f"_l{args.lmax}")


def profile_traffic(workload: str, batch: int) -> float | None:
    """Per-launch DRAM bytes of the GEMV kernel from a committed ncu summary,
    if that summary was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        data = json.load(f)
    entry = data.get(f"{workload}/b{batch}")
    if not entry or entry.get("kernel_sha") != kernel_source_hash():
        return None
    return float(entry["dram_bytes_per_launch"])


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = f"/tmp/nwc_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self) -> dict:
        if not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        sm, smax, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    smax = float(parts[2])
                    power.append(float(parts[3]))
                except ValueError:
                    continue
                for name, val in zip(names, parts[5:9]):
                    if val.lower() == "active":
                        reasons.add(name)
        os.unlink(self.path)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax,
                "power_w_max": max(power) if power else None, "samples": len(sm),
                "reasons": sorted(reasons)}


def dist_setup(n_gpus: int):
    import torch
    rank, world = 0, 1
    if n_gpus > 1 or "RANK" in os.environ:
        import datetime

        import torch.distributed as dist
        rank = int(os.environ.get("RANK", 0))
        world = int(os.environ.get("WORLD_SIZE", 1))
        local = int(os.environ.get("LOCAL_RANK", rank))
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's time: every rank contributes, all get the maximum."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_region(run_steps, steps: int, stream, world: int, min_s: float):
    """Times `steps` steps (run_steps(stream) enqueues them), each region
    bracketed by a barrier and a device synchronize, the max over ranks; when a
    region is shorter than min_s it is repeated (the same count on every rank)
    and the median is returned.  Returns (ms for the steps, repeats, all ms)."""
    import torch

    def once() -> float:
        barrier(world)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            t0.record(stream)
            run_steps(stream)
            t1.record(stream)
        stream.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        return max_over_ranks(t0.elapsed_time(t1), world)

    first = once()
    repeats = 1 if first >= 1e3 * min_s else min(50, int(np.ceil(1e3 * min_s / max(first, 1e-3))))
    times = [first] + [once() for _ in range(repeats - 1)]
    return statistics.median(times), repeats, times


def replica_value(weight_bytes: float, world: int, ms_per_step: float) -> float:
    """Whole-job effective GB/s: every rank runs the same per-GPU work (weak
    scaling, independent replicas), so the job moves world x weight_bytes per
    step in the slowest rank's time."""
    return world * weight_bytes / (ms_per_step * 1e-3) / 1e9


def _oracle_sample(workload: str, batch: int, rows: int):
    """A bounded sample of the workload for the oracle: the first `rows` rows of
    its first matrix, encoded by the oracle, and the batch of activations."""
    import oracle
    from lossless_bf16_weight_nwc_b200 import synth
    wl = synth.workload(workload)
    spec = wl.matrices[0]
    rows = min(rows, spec.rows)
    w = synth.matrix(spec, wl.seed, 0, rows)
    x = synth.activations(wl.seed, batch, spec.cols)
    return oracle, oracle.encode(w), x, rows, spec.cols


def cpu_baseline(workload: str, batch: int, budget_s: float = 12.0) -> dict:
    """The oracle as it stands (decode + FP64 GEMV), single-threaded, on a
    bounded sample: whole calls on up to 4096 rows of the workload's first
    matrix until the budget is spent, in the bench metric's unit."""
    orc, blob, x, rows, cols = _oracle_sample(workload, batch, 4096)
    calls, t0 = 0, time.perf_counter()
    while True:
        orc.gemv(orc.decode(blob), x)
        calls += 1
        el = time.perf_counter() - t0
        if el >= budget_s or calls >= 50:
            break
    per_call = el / calls
    return {"value": 2.0 * rows * cols / per_call / 1e9, "unit": "GB/s", "cores": 1,
            "kind": "oracle", "us_per_call": per_call * 1e6,
            "sample": f"{calls} whole oracle calls (decode of the blob + FP64 GEMV, batch {batch}) "
                      f"on {rows}x{cols} rows of '{workload}' matrix 0, single thread"}


def run_reference(args) -> None:
    """The reference arm: the oracle on the host cores, rank 0 only.  Each step
    is one oracle call (decode + FP64 GEMV) on a 256-row sample of the
    workload's first matrix; at most as many of the --steps as fit in about a
    minute are timed, after --warmup untimed calls."""
    rank = int(os.environ.get("RANK", 0))
    if rank != 0:
        return
    orc, blob, x, rows, cols = _oracle_sample(args.workload, args.batch, 256)
    for _ in range(max(args.warmup, 1)):
        orc.gemv(orc.decode(blob), x)
    t0 = time.perf_counter()
    orc.gemv(orc.decode(blob), x)
    est = time.perf_counter() - t0
    steps = max(1, min(args.steps, int(60.0 / max(est, 1e-6))))
    t0 = time.perf_counter()
    for _ in range(steps):
        orc.gemv(orc.decode(blob), x)
    el = time.perf_counter() - t0
    step_s = el / steps
    value = 2.0 * rows * cols / step_s / 1e9
    sample = (f"{steps} oracle calls (decode + FP64 GEMV, batch {args.batch}) on {rows}x{cols} "
              f"rows of '{args.workload}' matrix 0, single thread, after {max(args.warmup, 1)} "
              f"warm-up calls")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": max(args.warmup, 1),
        "ms_per_step": step_s * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": args.workload, "batch": args.batch,
                   "matrix": f"{rows}x{cols} (sample)"},
        "cpu_baseline": {"kind": "oracle", "cores": 1, "sample": sample, "value": value,
                         "unit": "GB/s"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


STACKS = ("qwen3_4b_stack", "llama31_8b_stack")
CODES = {"prefix": 0, "rank": 1, "escape": 2}    # nwc_opts.code


def run_stack(args) -> None:
    """Per-token sequence of a layer stack: every GEMV of every layer, then the
    lm_head, captured as one CUDA graph; a step is one token.  Layer weights:
    layer 0 of the workload, generated once, compressed once and held as two
    device copies that alternate between layers (a layer is larger than L2, so
    every read is cold); the lm_head is its first rows repeated (synth).  With
    --fuse, the projections that read the same input (q, k, v; gate, up) are
    one matrix each, their rows stacked, compressed under one code table and
    multiplied in one call (the cuBLAS leg uses the same stacked shapes)."""
    import torch

    from lossless_bf16_weight_nwc_b200 import _lib, synth
    rank, world = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl, layer0_parts, head, n_layers = synth.stack_parts(args.workload)
    units = (synth.fused_layer(layer0_parts) if args.fuse
             else [(m.name.rsplit(".", 1)[-1], [m]) for m in layer0_parts])
    layer0 = [synth.MatrixSpec(f"layers.0.{g}", sum(p.rows for p in ps), ps[0].cols, ps[0].kind,
                               ps[0].std, ps[0].tensor) for g, ps in units]
    parts_of = {sp.name: ps for sp, (_, ps) in zip(layer0, units)}
    batch = args.batch
    steps = args.steps if args.steps is not None else 50
    specs = layer0 + [head]
    host_w = {}
    comp = {}
    for sp in specs:
        host_w[sp.name] = (synth.head_matrix(sp, wl.seed) if sp is head
                           else synth.stacked_matrix(parts_of[sp.name], wl.seed))
        comp[sp.name] = _lib.CompressedMatrix.compress(host_w[sp.name], device=dev,
                                                       streams=args.streams,
                                                       code=CODES[args.code], lmax=args.lmax)
    sets = [{sp.name: comp[sp.name] for sp in layer0}]
    second = {}
    for sp in layer0:
        m0 = comp[sp.name]
        m = _lib.CompressedMatrix(m0.image.clone(), None, sp.rows, sp.cols, m0.blob_bytes)
        m.handle = _lib.nwc_handle_from_device(m.image, m.image.numel())
        second[sp.name] = m
    sets.append(second)
    if args.tc_min_batch is not None:
        for m in list(comp.values()) + list(second.values()):
            _lib.nwc_gemv_set_tc_min_batch(m.handle, args.tc_min_batch)
    xs = {k: torch.from_numpy(synth.activations(wl.seed, batch, k).view(np.int16))
          .view(torch.bfloat16).to(dev) for k in {sp.cols for sp in specs}}
    ys = {n: torch.empty((batch, n), dtype=torch.float32, device=dev) for n in {sp.rows for sp in specs}}
    stream = torch.cuda.Stream(device=dev)
    seq = [(sets[l % 2][sp.name], sp) for l in range(n_layers) for sp in layer0] + [(comp[head.name], head)]
    paths = [_lib.nwc_gemv_path(m.handle, xs[sp.cols], batch) for m, sp in seq]
    launches = sum(n for n, _ in paths)
    kernel = "gemv_tc_kernel" if all(tc for _, tc in paths) else \
        "gemv_kernel" if not any(tc for _, tc in paths) else "gemv_kernel+gemv_tc_kernel"

    def token(y_head=None):
        for m, sp in seq:
            yt = y_head if (sp is head and y_head is not None) else ys[sp.rows]
            _lib.nwc_gemv(m.handle, xs[sp.cols], yt, batch, stream.cuda_stream)

    with torch.cuda.stream(stream):
        for _ in range(3):
            token()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        token()
    warm = max(args.warmup if args.warmup is not None else 5, 3)
    with torch.cuda.stream(stream):
        for _ in range(warm):
            g.replay()
    stream.synchronize()

    def run_steps(st):
        for _ in range(steps):
            g.replay()

    with ClockSampler(dev.index) as clocks:
        region_ms, repeats, region_all = timed_region(run_steps, steps, stream, world,
                                                      args.min_region_s)
    ms_per_token = region_ms / steps

    # Parity spot check: the lm_head, the layer's first and last matrices
    # (q or the stacked qkv; down), sampled rows.
    parity_ok = True
    if rank == 0:
        import oracle
        for sp in (head, layer0[0], layer0[-1]):
            xh = synth.activations(wl.seed, batch, sp.cols)
            comp[sp.name].gemv(torch.from_numpy(xh.view(np.int16)).view(torch.bfloat16).to(dev),
                               y=ys[sp.rows])
            idx = np.unique(np.linspace(0, sp.rows - 1, 256).astype(np.int64))
            ref = oracle.gemv(host_w[sp.name][idx], xh)
            got = ys[sp.rows].double().cpu().numpy()[:, idx]
            wf = synth.bf16_bits_to_float(host_w[sp.name][idx]).astype(np.float64)
            xf = synth.bf16_bits_to_float(xh).astype(np.float64)
            bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
            parity_ok = parity_ok and bool((np.abs(got - ref) <= bound).all())

    weight_bytes = sum(2.0 * sp.rows * sp.cols for _, sp in seq)
    comp_bytes = sum(float(m.compressed_bytes) for m, _ in seq)
    image_bytes = sum(float(m.device_bytes) for m, _ in seq)
    x_bytes = sum(2.0 * batch * sp.cols for _, sp in seq)
    y_bytes = sum(4.0 * batch * sp.rows for _, sp in seq)
    peaks, peak_src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    alg = comp_bytes + x_bytes + y_bytes
    achieved = alg / (ms_per_token * 1e-3) / 1e9

    # End to end: the hidden-state x copied in from pinned memory and the logits
    # stored by the lm_head kernel into pinned host memory, every token.
    e2e = None
    if args.e2e_steps > 0:
        xh_pin = torch.from_numpy(synth.activations(wl.seed, batch, layer0[0].cols).view(np.int16)) \
            .view(torch.bfloat16).pin_memory()
        logits = torch.empty((batch, head.rows), dtype=torch.float32).pin_memory()
        ge = torch.cuda.CUDAGraph()
        with torch.cuda.graph(ge, stream=stream):
            xs[layer0[0].cols].copy_(xh_pin, non_blocking=True)
            token(y_head=logits)
        n_e2e = min(args.e2e_steps, steps)
        with torch.cuda.stream(stream):
            ge.replay()
        stream.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(n_e2e):
                ge.replay()
            e1.record(stream)
        stream.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / n_e2e
        e2e = {"value": world * weight_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "us_per_token": e2e_ms * 1e3,
               "h2d_bytes_per_step": int(2 * batch * layer0[0].cols),
               "d2h_bytes_per_step": int(4 * batch * head.rows),
               "transfers": "hidden state by a captured copy from pinned memory; logits stored "
                            "by the lm_head kernel into pinned host memory"}
        del ge

    cublas = None
    if not args.no_cublas:
        wts = {sp.name: torch.from_numpy(host_w[sp.name].view(np.int16)).view(torch.bfloat16).to(dev)
               for sp in specs}
        wts2 = {sp.name: wts[sp.name].clone() for sp in layer0}
        xb = {k: v for k, v in xs.items()}
        yb = {n: torch.empty((batch, n), dtype=torch.bfloat16, device=dev) for n in ys}
        dense = [((wts if l % 2 == 0 else wts2)[sp.name], sp) for l in range(n_layers) for sp in layer0]
        dense.append((wts[head.name], head))
        with torch.cuda.stream(stream):
            for wt, sp in dense:
                torch.matmul(xb[sp.cols], wt.t(), out=yb[sp.rows])
        stream.synchronize()
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb, stream=stream):
            for wt, sp in dense:
                torch.matmul(xb[sp.cols], wt.t(), out=yb[sp.rows])
        reps = max(3, min(steps, 50))
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gb.replay()
            c0.record(stream)
            for _ in range(reps):
                gb.replay()
            c1.record(stream)
        stream.synchronize()
        cb_ms = c0.elapsed_time(c1) / reps
        cublas = {"us_per_token": cb_ms * 1e3, "effective_gbs": weight_bytes / (cb_ms * 1e-3) / 1e9,
                  "speedup_nwc_vs_cublas": cb_ms / ms_per_token}
        del gb, wts, wts2

    line = {
        "metric": METRIC, "value": replica_value(weight_bytes, world, ms_per_token), "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": warm, "ms_per_step": ms_per_token,
        "timed_regions": {"repeats": repeats, "statistic": "median over repeats of the max "
                          "over ranks", "ms_each": [round(t, 4) for t in region_all]},
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "batch": batch, "step": f"one token: {len(seq)} GEMVs "
                   f"({n_layers} layers x {len(layer0)} + lm_head), one CUDA graph",
                   "layer": [f"{g} {sp.rows}x{sp.cols}" for (g, _), sp in zip(units, layer0)],
                   "fused": bool(args.fuse), "streams_per_lane": args.streams,
                   "code": args.code, "lmax": args.lmax,
                   "weights": "layer 0 generated, two device copies alternating over the layers; "
                              f"lm_head = its first {synth.HEAD_BLOCK_ROWS} rows repeated",
                   "l2": "inputs larger than L2: every layer is larger than L2",
                   "launch": "CUDA graph replay", "parallelism": f"replicas x{world}"},
        "us_per_token": ms_per_token * 1e3,
        "tokens_per_s": 1e3 / ms_per_token,
        "compression_ratio": weight_bytes / comp_bytes,
        "compressed_bytes_per_token": comp_bytes,
        "device_image_bytes_per_token": image_bytes,
        "footprint_ratio": weight_bytes / image_bytes,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm,
                     "traffic": profile_traffic(
                         args.workload + ("_fused" if args.fuse else "") + format_suffix(args),
                         batch),
                     "traffic_basis": "DRAM bytes per GEMV launch, averaged over a token's "
                                      "launches (committed ncu summary, current kernel source "
                                      "only; else null)",
                     "algorithmic_bytes_per_launch": alg / launches,
                     "peak_source": f"{peak_src} hbm_gbs (copy)", "kernel": kernel,
                     "basis": "algorithmic bytes of the token's GEMVs / graph time per token",
                     "tokens_per_s_ceiling_at_peak": hbm * 1e9 / alg},
        "clocks": clocks.summary(),
        "e2e": e2e,
        "gpu_launches": steps * launches,
        "kernel_path": kernel,
        "parity_spot_check": parity_ok,
        "cublas_bf16": cublas,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, batch)
        line["cpu_baseline"].pop("us_per_call", None)
    del g
    return line if rank == 0 else None


def run_matrix(args):
    """One matrix of the workload: a step is one nwc_gemv call, rotating over
    enough compressed copies that the weights never sit in L2."""
    import torch

    from lossless_bf16_weight_nwc_b200 import _lib, synth
    rank, world = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.workload(args.workload)
    spec = wl.matrices[0]
    batch = args.batch
    w = synth.matrix(spec, wl.seed)
    x_host = synth.activations(wl.seed, batch, spec.cols)
    first = _lib.CompressedMatrix.compress(w, device=dev, streams=args.streams,
                                           code=CODES[args.code], lmax=args.lmax)
    image_bytes = first.compressed_bytes   # blob, table and schedules (no scratch)
    copies = max(2, int(np.ceil(2.2 * L2_BYTES / image_bytes)))
    copies = min(copies, args.steps) if args.steps >= 2 else copies
    mats = [first] + [_lib.CompressedMatrix(first.image.clone(), None, spec.rows, spec.cols,
                                            first.blob_bytes) for _ in range(copies - 1)]
    for m in mats[1:]:
        m.handle = _lib.nwc_handle_from_device(m.image, m.image.numel())
    if args.tc_min_batch is not None:
        for m in mats:
            _lib.nwc_gemv_set_tc_min_batch(m.handle, args.tc_min_batch)
    x = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).to(dev)
    y = torch.empty((batch, spec.rows), dtype=torch.float32, device=dev)
    launches_per_call, on_tc = _lib.nwc_gemv_path(first.handle, x, batch)
    kernel = "gemv_tc_kernel" if on_tc else "gemv_kernel"
    stream = torch.cuda.Stream(device=dev)

    def call(m, s):
        _lib.nwc_gemv(m.handle, x, y, batch, s.cuda_stream)

    # Warm-up (also configures kernel attributes before capture).
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            call(mats[i % copies], stream)
    stream.synchronize()

    # Exactly args.steps calls: full replays of a graph of `calls_per_graph`
    # calls, then one graph of the remainder.
    steps = args.steps
    calls_per_graph = min(args.graph_calls or copies, steps)
    replays, rest = divmod(steps, calls_per_graph)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(calls_per_graph):
            call(mats[i % copies], stream)
    g_rest = None
    if rest:
        g_rest = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_rest, stream=stream):
            for i in range(rest):
                call(mats[i % copies], stream)
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
    stream.synchronize()

    def run_steps(st):
        for _ in range(replays):
            g.replay()
        if g_rest is not None:
            g_rest.replay()

    with ClockSampler(dev.index) as clocks:
        elapsed_ms, repeats, region_all = timed_region(run_steps, steps, stream, world,
                                                       args.min_region_s)
    clock = clocks.summary()

    # The timed region holds GEMV launches only, so their average duration there
    # is the region's event time over its launches (consecutive launches overlap
    # their prologue with the previous tail).  For comparison, the duration of
    # one launch on its own: event pairs around direct launches on the stream,
    # queued behind a GPU sleep so that the intervals hold the kernels, not host
    # submission gaps.
    kernel_ms = elapsed_ms / (steps * launches_per_call)
    durs = []
    n_timed = min(256, 8 * copies)
    for _ in range(4):
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_timed)]
        with torch.cuda.stream(stream):
            torch.cuda._sleep(100_000_000)
            for i in range(n_timed):
                ev[i][0].record(stream)
                call(mats[i % copies], stream)
                ev[i][1].record(stream)
        stream.synchronize()
        durs += [a.elapsed_time(b) for a, b in ev]
    isolated_ms = statistics.mean(durs) / launches_per_call
    ms_per_step = elapsed_ms / steps

    # Parity spot check of the timed configuration.
    y_ref = None
    if rank == 0:
        import oracle
        rows_chk = np.arange(0, spec.rows, max(1, spec.rows // 256))
        y_ref = oracle.gemv(w, x_host)[:, rows_chk]
        call(mats[0], torch.cuda.current_stream())
        y_gpu = y.double().cpu().numpy()[:, rows_chk]
        wf = synth.bf16_bits_to_float(w[rows_chk]).astype(np.float64)
        xf = synth.bf16_bits_to_float(x_host).astype(np.float64)
        bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
        parity_ok = bool((np.abs(y_gpu - y_ref) <= bound).all())
    else:
        parity_ok = True

    weight_bytes = 2.0 * spec.rows * spec.cols
    x_bytes, y_bytes = 2.0 * batch * spec.cols, 4.0 * batch * spec.rows
    alg_bytes = image_bytes + x_bytes + y_bytes
    peaks, peak_src = measured_peaks()
    hbm = float(peaks["hbm_gbs"])
    eff_gbs = replica_value(weight_bytes, world, ms_per_step)
    achieved = alg_bytes / (kernel_ms * 1e-3) / 1e9
    traffic = profile_traffic(args.workload + format_suffix(args), batch)

    # End to end through the public API with host buffers: pinned x in, y out.
    e2e = None
    if args.e2e_steps > 0:
        xh = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).pin_memory()
        yh = torch.empty((batch, spec.rows), dtype=torch.float32).pin_memory()
        xd = torch.empty_like(x)
        torch.cuda.synchronize()
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        # "copy": x and y move with cudaMemcpyAsync around the call; "host-y": the
        # kernel stores y straight into the pinned (device-mapped) host buffer.
        host_y = args.e2e_mode == "host-y"
        with torch.cuda.stream(stream):
            e0.record(stream)
            for i in range(args.e2e_steps):
                xd.copy_(xh, non_blocking=True)
                _lib.nwc_gemv(mats[i % copies].handle, xd, yh if host_y else y, batch,
                              stream.cuda_stream)
                if not host_y:
                    yh.copy_(y, non_blocking=True)
            e1.record(stream)
        stream.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world) / args.e2e_steps
        e2e = {"value": world * weight_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
               "us_per_call": e2e_ms * 1e3, "h2d_bytes_per_step": int(x_bytes),
               "d2h_bytes_per_step": int(y_bytes),
               "transfers": ("x by cudaMemcpyAsync; y stored by the kernel into pinned host "
                             "memory" if host_y else "x and y by cudaMemcpyAsync")}

    # Uncompressed BF16 cuBLAS GEMV on the same shape and L2 policy, for context.
    cublas = None
    if not args.no_cublas:
        wt = torch.from_numpy(w.view(np.int16)).view(torch.bfloat16).to(dev)
        n_w = max(2, int(np.ceil(2.2 * L2_BYTES / (weight_bytes))))
        wts = [wt] + [wt.clone() for _ in range(n_w - 1)]
        yb = torch.empty((batch, spec.rows), dtype=torch.bfloat16, device=dev)
        with torch.cuda.stream(stream):
            for i in range(20):
                torch.matmul(x, wts[i % n_w].t(), out=yb)
        stream.synchronize()
        gb = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gb, stream=stream):
            for i in range(n_w):
                torch.matmul(x, wts[i % n_w].t(), out=yb)
        reps = max(1, 2000 // n_w)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            gb.replay()
            c0.record(stream)
            for _ in range(reps):
                gb.replay()
            c1.record(stream)
        stream.synchronize()
        cb_ms = c0.elapsed_time(c1) / (reps * n_w)
        cublas = {"us_per_call": cb_ms * 1e3,
                  "effective_gbs": weight_bytes / (cb_ms * 1e-3) / 1e9,
                  "speedup_nwc_vs_cublas": cb_ms / ms_per_step}
        del wts

    line = {
        "metric": METRIC,
        "value": eff_gbs,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": steps,
        "warmup": max(args.warmup, 3),
        "ms_per_step": ms_per_step,
        "timed_regions": {"repeats": repeats, "statistic": "median over repeats of the max "
                          "over ranks", "ms_each": [round(t, 4) for t in region_all]},
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "matrix": f"{spec.rows}x{spec.cols}",
                   "batch": batch, "values": spec.kind, "streams_per_lane": args.streams,
                   "code": args.code, "lmax": args.lmax,
                   "l2": f"inputs larger than L2: {copies} rotating compressed copies "
                         f"({copies * image_bytes / 2**20:.0f} MiB)",
                   "launch": "CUDA graph replay", "parallelism": f"replicas x{world}"},
        "us_per_call": ms_per_step * 1e3,
        "compression_ratio": weight_bytes / image_bytes,
        "compressed_bytes": image_bytes,
        "footprint_ratio": weight_bytes / first.device_bytes,
        "pct_hbm_peak_compressed": 100.0 * (image_bytes / (kernel_ms * 1e-3) / 1e9) / hbm,
        "pct_of_8tbs_compressed": 100.0 * (image_bytes / (kernel_ms * 1e-3) / 1e9) / 8000.0,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": traffic,
                     "peak_source": f"{peak_src} hbm_gbs (copy)",
                     "kernel": kernel, "kernel_us": kernel_ms * 1e3,
                     "basis": "algorithmic bytes per launch / timed-region event time per launch",
                     "isolated_launch_us": isolated_ms * 1e3,
                     "algorithmic_bytes_per_launch": alg_bytes},
        "clocks": clock,
        "e2e": e2e,
        "gpu_launches": steps * launches_per_call,
        "kernel_path": kernel,
        "parity_spot_check": parity_ok,
        "cublas_bf16": cublas,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload, batch)
        line["cpu_baseline"].pop("us_per_call", None)
    # Release graphs before the process group.
    del g, g_rest
    return line if rank == 0 else None


def main():
    args = parse_args()
    if args.steps is None and args.workload not in STACKS:
        args.steps = 20000
    if args.warmup is None and args.workload not in STACKS:
        args.warmup = 200
    if args.impl == "reference":
        if args.steps is None:
            args.steps = 50
        if args.warmup is None:
            args.warmup = 3
        run_reference(args)
        return
    if args.report:
        run_report(args)
        return
    if args.shard:
        if args.workload in STACKS:
            raise SystemExit("--shard takes a single-matrix workload")
        line = run_matrix_sharded(args)
    else:
        line = run_stack(args) if args.workload in STACKS else run_matrix(args)
    if line is not None:
        print(json.dumps(line))
    if int(os.environ.get("WORLD_SIZE", 1)) > 1:
        import torch.distributed as dist
        if dist.is_initialized():
            dist.destroy_process_group()


def run_matrix_sharded(args):
    """One matrix of the workload split by output rows over the job's ranks
    (whole 8-row tile blocks, one code table per shard): a step is one GEMV of
    each rank's rows plus one NCCL all-gather that leaves the whole y on every
    rank.  Each rank rotates over enough device copies of its shard that the
    weights never sit in L2.  Steps are launched eagerly (the gather is a
    collective) and timed with CUDA events between barriers; the time is the
    slowest rank's, and value counts the whole matrix once (strong scaling)."""
    import torch

    from lossless_bf16_weight_nwc_b200 import _lib, synth
    from lossless_bf16_weight_nwc_b200.sharded import ShardedMatrix
    rank, world = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    wl = synth.workload(args.workload)
    spec = wl.matrices[0]
    batch = args.batch
    w = synth.matrix(spec, wl.seed)
    x_host = synth.activations(wl.seed, batch, spec.cols)
    sm = ShardedMatrix.compress(w, group=None, device=dev, streams=args.streams,
                                code=CODES[args.code], lmax=args.lmax)
    local = sm.local
    image_bytes = local.compressed_bytes if local is not None else 0
    copies = max(2, int(np.ceil(2.2 * L2_BYTES / max(image_bytes, 1)))) if local else 1
    mats = [local]
    if local is not None:
        for _ in range(copies - 1):
            m = _lib.CompressedMatrix(local.image.clone(), None, local.rows, local.cols,
                                      local.blob_bytes)
            m.handle = _lib.nwc_handle_from_device(m.image, m.image.numel())
            mats.append(m)
        if args.tc_min_batch is not None:
            for m in mats:
                _lib.nwc_gemv_set_tc_min_batch(m.handle, args.tc_min_batch)
    x = torch.from_numpy(x_host.view(np.int16)).view(torch.bfloat16).to(dev)
    y_local = torch.empty((batch, local.rows if local else 0), dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        m = mats[i % len(mats)]
        if m is None:
            return sm.gemv(x)
        return sm.gemv(x, local_gemv=lambda xx: (
            _lib.nwc_gemv(m.handle, xx, y_local, batch, stream.cuda_stream), y_local)[1])

    for i in range(max(args.warmup, 3)):
        step(i)
    torch.cuda.synchronize()
    steps = args.steps
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        barrier(world)
        torch.cuda.synchronize()
        e0.record(stream)
        for i in range(steps):
            y = step(i)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
    ms = max_over_ranks(e0.elapsed_time(e1), world) / steps
    parity_ok = True
    if rank == 0:
        import oracle
        rows_chk = np.arange(0, spec.rows, max(1, spec.rows // 256))
        y_ref = oracle.gemv(w[rows_chk], x_host)
        y_gpu = y.double().cpu().numpy()[:, rows_chk]
        wf = synth.bf16_bits_to_float(w[rows_chk]).astype(np.float64)
        xf = synth.bf16_bits_to_float(x_host).astype(np.float64)
        bound = 1e-2 * np.outer(np.linalg.norm(xf, axis=1), np.linalg.norm(wf, axis=1)) * 2.0 ** -8
        parity_ok = bool((np.abs(y_gpu - y_ref) <= bound).all())
    weight_bytes = 2.0 * spec.rows * spec.cols
    peaks, peak_src = measured_peaks()
    line = {
        "metric": METRIC, "value": weight_bytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": max(args.warmup, 3), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": args.workload, "matrix": f"{spec.rows}x{spec.cols}",
                   "batch": batch, "parallelism": f"rows x{world} (ShardedMatrix) + all-gather of y",
                   "rows_per_rank": [e - s for s, e in sm.ranges],
                   "l2": f"inputs larger than L2: {copies} rotating copies of each shard",
                   "launch": "eager (GEMV + NCCL all-gather per step)"},
        "us_per_call": ms * 1e3,
        "roofline": {"bound": "hbm", "achieved": image_bytes / (ms * 1e-3) / 1e9,
                     "peak": float(peaks["hbm_gbs"]), "unit": "GB/s",
                     "frac": image_bytes / (ms * 1e-3) / 1e9 / float(peaks["hbm_gbs"]),
                     "traffic": None, "peak_source": f"{peak_src} hbm_gbs (copy)",
                     "basis": "rank 0's compressed shard bytes / time per step (GEMV + gather)"},
        "clocks": clocks.summary(),
        "e2e": None,
        "gpu_launches": steps,
        "kernel_path": "gemv_tc_kernel" if local is not None and _lib.nwc_gemv_path(
            local.handle, x, batch)[1] else "gemv_kernel",
        "parity_spot_check": parity_ok,
    }
    for m in mats[1:]:
        m.close()
    sm.close()
    return line if rank == 0 else None


def run_report(args) -> None:
    """The five benchmark configurations in one run, as a markdown table
    (and every configuration's JSON line in --report-json when given): per
    call or per token, effective and compressed GB/s, fraction of the HBM
    peak, compression ratio, the uncompressed cuBLAS time and the kernel
    path."""
    rows = [("single_1024", 1, None), ("attn_4096_outliers", 1, None),
            ("attn_4096_outliers", 4, None), ("attn_4096_outliers", 16, None),
            ("attn_4096_outliers", 64, None), ("mlp_pair_t5", 1, None), ("mlp_pair_t5", 2, None),
            ("mlp_pair_t5", 8, None), ("mlp_pair_t5", 64, None),
            ("qwen3_4b_stack", 1, False), ("qwen3_4b_stack", 1, True),
            ("llama31_8b_stack", 1, False), ("llama31_8b_stack", 1, True),
            ("llama31_8b_stack", 16, True), ("llama31_8b_stack", 64, True)]
    lines = []
    for workload, batch, fuse in rows:
        a = argparse.Namespace(**vars(args))
        a.workload, a.batch, a.report = workload, batch, False
        if fuse is not None:
            a.fuse = fuse
        a.no_cpu_baseline = True
        a.e2e_steps = 0
        stack = workload in STACKS
        a.steps = args.steps if args.steps is not None else (10 if stack else 4000)
        a.warmup = 3 if stack else 50
        line = run_stack(a) if stack else run_matrix(a)
        lines.append(line)
        print(f"{workload} b{batch}: {line['ms_per_step'] * 1e3:.2f} us", file=sys.stderr, flush=True)
    gather = gather_report()
    print("| workload | batch | µs per step | effective GB/s | compressed GB/s | fraction of HBM "
          "peak | ratio | cuBLAS BF16 µs | kernel |")
    print("|---|---|---|---|---|---|---|---|---|")
    for (workload, batch, fuse), line in zip(rows, lines):
        if fuse is not None:
            workload = f"{workload} ({'fused' if fuse else 'unfused'})"
        rf = line["roofline"]
        comp = line.get("compressed_bytes") or line.get("compressed_bytes_per_token")
        us = line["ms_per_step"] * 1e3
        cb = line.get("cublas_bf16") or {}
        cb_us = cb.get("us_per_call") or cb.get("us_per_token")
        print(f"| {workload} | {batch} | {us:.2f} | {line['value']:.0f} | "
              f"{comp / (us * 1e-6) / 1e9:.0f} | {rf['frac']:.3f} ({rf['peak_source']}) | "
              f"{line['compression_ratio']:.3f} | {cb_us:.2f} | {line.get('kernel_path')} |")
    print()
    print("| row gather from the 151936 x 2560 lm_head | µs per call (L2 flushed) |")
    print("|---|---|")
    for name, us in gather:
        print(f"| {name} | {us:.2f} |")
    if args.report_json:
        with open(args.report_json, "w") as f:
            for line in lines:
                f.write(json.dumps(line) + "\n")
            f.write(json.dumps({"gather_report": dict(gather)}) + "\n")


def gather_report(calls: int = 64) -> list:
    """Embedding lookup from the compressed Qwen3-4B-shaped lm_head
    (151936 x 2560, tied embedding): n random rows per call (n = 1, 8), against
    one GEMV of the same stack's 4096 x 2560 q projection at batch 1.  Each
    call is timed alone with CUDA events after a 256 MiB write that evicts L2,
    with fresh row ids per call; the gathered rows are checked bit for bit."""
    import torch

    from lossless_bf16_weight_nwc_b200 import _lib, synth
    dev = torch.device("cuda", torch.cuda.current_device())
    wl, layer0, head, _ = synth.stack_parts("qwen3_4b_stack")
    w_head = synth.head_matrix(head, wl.seed)
    m_head = _lib.CompressedMatrix.compress(w_head, device=dev)
    q = layer0[0]
    w_q = synth.matrix(q, wl.seed)
    m_q = _lib.CompressedMatrix.compress(w_q, device=dev)
    x = torch.from_numpy(synth.activations(wl.seed, 1, q.cols).view(np.int16)).view(
        torch.bfloat16).to(dev)
    y = torch.empty((1, q.rows), dtype=torch.float32, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    rng = np.random.default_rng(11)
    out = []

    def timed(fn):
        for _ in range(3):
            fn(0)
        torch.cuda.synchronize()
        durs = []
        for i in range(calls):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            fn(i)
            e1.record()
            torch.cuda.synchronize()
            durs.append(e0.elapsed_time(e1) * 1e3)
        return statistics.median(durs)

    for n in (1, 8):
        ids = [torch.from_numpy(rng.integers(0, head.rows, n).astype(np.int32)).to(dev)
               for _ in range(calls)]
        got = m_head.gather_rows(ids[0])
        assert np.array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16),
                              w_head[ids[0].cpu().numpy()]), "gather parity"
        out.append((f"gather {n} row{'s' if n > 1 else ''}",
                    timed(lambda i: m_head.gather_rows(ids[i]))))
    out.append(("GEMV 4096 x 2560 (q projection), batch 1",
                timed(lambda i: _lib.nwc_gemv(m_q.handle, x, y, 1))))
    st, word = m_head.device_error()
    assert st == 0, ("device error", st, word)
    m_head.close()
    m_q.close()
    return out




if __name__ == "__main__":
    main()
