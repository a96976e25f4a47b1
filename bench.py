#!/usr/bin/env python
"""Benchmark of the masked HLA forward on B200.

Default workload: ratio-normalised second-order HLA, bf16 inputs, fp32 output,
B=4, H=16, T=4096, d=dv=64 (262,144 tokens per step), synthetic seeded inputs.
One step = one full forward (segment summaries, exclusive scan of the summaries, output pass).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  Device timing: CUDA events recorded by the
library on the launching stream around every phase of every timed step; L2 is
flushed (a 512 MiB write) before every step, outside the events.  Multi-GPU
(torchrun): every rank runs its own batch of the same shape (no collective on
the data path: heads are independent), time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import hla_inputs  # noqa: E402

DEFAULT_WORKLOAD = "hla2n_bf16_4x16x4096x64"
METRIC = "HLA-2 masked fwd tokens/sec (B·H·T/s) at d=64 bf16; % of B200 bf16 tensor peak"
UNIT = "tokens/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__)
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(hla_inputs.WORKLOADS))
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--decode-steps", type=int, default=20,
                   help="streaming decode steps timed after the forward (0: skip)")
    p.add_argument("--segment-chunks", type=int, default=0,
                   help="tensor-core path: 128-token chunks per segment (0 = the library's choice)")
    p.add_argument("--backward-steps", type=int, default=10,
                   help="timed steps of the second-order backward at the workload's shape (0: skip)")
    p.add_argument("--workload-steps", type=int, default=10,
                   help="timed steps per workload of the 'workloads' object (0: skip it)")
    args = p.parse_args(argv)
    if args.warmup < 3:
        p.error("--warmup must be >= 3")
    if args.steps < 1:
        p.error("--steps must be >= 1")
    return args


# ---------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def dist_init(world: int, backend: str):
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity for one rank)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_value(tokens_per_rank: int, world: int, max_seconds_per_step: float) -> float:
    """Whole-job throughput: all ranks' tokens over the slowest rank's time."""
    return tokens_per_rank * world / max_seconds_per_step


# ---------------------------------------------------------------------------
# clocks sampled while the GPU works
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(prefix="hla_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        if self.path and os.path.exists(self.path):
            for line in open(self.path):
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        busy = [x for x in sm if smax and x > 0.5 * max(smax)] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# roofline bookkeeping
# ---------------------------------------------------------------------------

def load_peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def output_kernel_model(path: str, w: hla_inputs.Workload):
    """Algorithmic work of the output kernel per token: the products the method needs per
    chunk of c tokens, each 2 flop per multiply-add, divided by c (no discarded halves of
    stacked products, no state walk)."""
    D = w.d
    c = 128 if path in ("tc", "tc-output") else 64
    if w.op in ("ahla", "ahlan", "ahlad"):
        # per token: A = Q K^T, Y = A V, O = A Y (2cD each), Q P0 and Q E0 (2D^2 each)
        flops = 6 * c * D + 4 * D * D
    elif w.op == "hla2u":
        # per token: A* = Q K^T, P Q^T, A K, W V (2cD each); A A*^T (2c^2); Q S0, Q (S0 C0),
        # (A K) C0 (2D^2 each); S0 C0 once per chunk (2D^3 / c)
        flops = 8 * c * D + 2 * c * c + 6 * D * D + 2 * D ** 3 // c
    elif path == "tc-output" and w.op == "hla3":
        # the third-order output kernel on the tensor cores (c = 128): A* = Q K^T, P Q^T, A V,
        # W Y (2cD each), A A^T (2c^2), Q S0, Q P0, Q F0 (2D^2 each), counted once (fp32)
        flops = 8 * c * D + 2 * c * c + 6 * D * D
    elif w.op == "hla2d" and path == "tc":
        # the decayed output walker forms O and carries the state. Per token: A* = Q K^T,
        # Gam P Q^T, H K, W V (2cD each), At A^T and H U^T (2c^2 each), P = Q S0, Z C0, Q G0
        # (2D^2 each); the state: K^T Lam K, Q^T Lam V, K C0, K^T Y (2D^2 each), U^T Lam V (2cD)
        flops = 10 * c * D + 14 * D * D + 4 * c * c
    else:
        # per token: A = Q K^T (2cD), P = Q S0 (2D^2), W = [P|A][Q|A]^T (2c(D+c)), O = [Q|W][R0;V] (2D(D+c))
        flops = 2 * c * D + 2 * D * D + 2 * c * (D + c) + 2 * D * (D + c)
        if w.op in ("hla3", "hla3n", "hla3d"):
            flops += 2 * D * (D + c)      # the third order also forms Y = [Q|A][P0;V] before O = [Q|W][F0;Y]
    return {"bound": "tensor" if path in ("tc", "tc-output") else "alu", "flops_per_token": flops, "chunk": c}


def alu_peak_tflops(sm_mhz: float) -> float:
    """FP32 FFMA peak of a B200: 148 SMs x 128 lanes x 2 flop x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args):
    import torch
    import higher_order_linear_chunked_b200 as hla

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device (this library has no CPU path)")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist_init(world, "nccl")
    base = hla_inputs.workload(args.workload)
    w = base.scaled(seed=base.seed + rank)
    q, k, v, g = hla_inputs.make_inputs(w)
    tokens = w.tokens
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    gd = g.to(dev) if g is not None else None
    out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device=dev)
    op = hla.OP_CODES[w.op]
    if args.segment_chunks:
        hla.set_segment_chunks(args.segment_chunks)
    ws = hla.make_workspace(op, qd, vd, decayed=gd is not None)
    dcode = hla.HLA_BF16 if w.dtype == "bf16" else hla.HLA_F32
    launches_per_step = hla.kernel_launches(op, dcode, gd is not None, w.B, w.H, w.T, w.d, w.dv)
    path = {1: "tc", 2: "tc-output"}.get(hla.uses_tensor_cores(op, dcode, gd is not None, w.B, w.H, w.T, w.d, w.dv), "simt")
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    if args.segment_chunks:
        hla.set_segment_chunks(args.segment_chunks)

    def new_events():
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        for e in evs:
            e.record()
        return evs

    # warm-up
    for _ in range(args.warmup):
        flush.zero_()
        hla.forward(w.op, qd, kd, vd, gamma=gd, eps=w.eps, out=out, workspace=ws)
    torch.cuda.synchronize()
    if hla.read_device_status(ws) != 0:
        raise SystemExit("device status word set during warm-up")
    events = [new_events() for _ in range(args.steps)]
    torch.cuda.synchronize()

    # The timed steps: the plain forward between two events per step (events between the
    # kernels would serialise the output walk's programmatic launch behind the summary walk).
    bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    clocks.start()
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        flush.zero_()                                            # outside the timed events
        bounds[i][0].record()
        hla.forward(w.op, qd, kd, vd, gamma=gd, eps=w.eps, out=out, workspace=ws)
        bounds[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    clocks.stop()
    step_ms = [a.elapsed_time(b) for a, b in bounds]
    # Phase breakdown (the output kernel's time for the roofline): the same forward with events
    # before the summary kernel, after it, after the scan and after the output kernel.
    for i in range(args.steps):
        flush.zero_()
        hla.forward_profiled(w.op, qd, kd, vd, events[i], gamma=gd, eps=w.eps, out=out, workspace=ws)
    torch.cuda.synchronize()
    out_ms = [ev[2].elapsed_time(ev[3]) for ev in events]
    sum_ms = [ev[0].elapsed_time(ev[1]) for ev in events]
    scan_ms = [ev[1].elapsed_time(ev[2]) for ev in events]
    status = hla.read_device_status(ws)
    total_ms = sum(step_ms)
    max_total_ms = max_over_ranks(total_ms, world, dev)
    ms_per_step = max_total_ms / args.steps
    value = weak_scaling_value(tokens, world, ms_per_step / 1e3)

    # end to end through the public API with host buffers (pinned), copies inside the timed
    # region.  The batch is cut into per-batch-index slices, each on its own stream (copy in,
    # forward, copy out), so one slice's copies overlap another slice's compute and the two
    # copy directions overlap each other.
    e2e = None
    if args.e2e_steps > 0:
        qh, kh, vh = (x.pin_memory() for x in (q, k, v))
        oh = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32).pin_memory()
        main = torch.cuda.current_stream(dev)
        G = w.B
        streams = [torch.cuda.Stream(dev) for _ in range(G)]
        gws = [hla.make_workspace(op, qd[b:b + 1], vd[b:b + 1], decayed=gd is not None) for b in range(G)]
        e_ms = []
        for i in range(args.e2e_steps + 2):
            flush.zero_()
            a, b_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(main)
            for b, s in enumerate(streams):
                s.wait_stream(main)
                with torch.cuda.stream(s):
                    sl = slice(b, b + 1)
                    qd[sl].copy_(qh[sl], non_blocking=True)
                    kd[sl].copy_(kh[sl], non_blocking=True)
                    vd[sl].copy_(vh[sl], non_blocking=True)
                    hla.forward(w.op, qd[sl], kd[sl], vd[sl], gamma=gd, eps=w.eps, out=out[sl], workspace=gws[b],
                                stream=s)
                    oh[sl].copy_(out[sl], non_blocking=True)
            for s in streams:
                main.wait_stream(s)
            b_ev.record(main)
            torch.cuda.synchronize()
            if i >= 2:
                e_ms.append(a.elapsed_time(b_ev))
        for b in range(G):
            if hla.read_device_status(gws[b]) != 0:
                raise SystemExit("device status word set during the end-to-end run")
        e2e_ms = max_over_ranks(sum(e_ms) / len(e_ms), world, dev)
        h2d = sum(x.numel() * x.element_size() for x in (q, k, v))
        e2e = {"value": weak_scaling_value(tokens, world, e2e_ms / 1e3), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": oh.numel() * oh.element_size(),
               "ms_per_step": e2e_ms,
               "pipeline": f"{G} batch slices on {G} streams: copy in, forward, copy out per slice"}

    peaks, peak_kind = load_peaks()
    decode = None
    if args.decode_steps > 0:
        decode = decode_measure(w, qd, kd, vd, gd, flush, args.decode_steps, peaks, peak_kind)
    backward = None
    if args.backward_steps > 0 and w.op in ("hla2", "hla2n", "ahla") and gd is None:
        backward = backward_measure(w, qd, kd, vd, flush, args.backward_steps, peaks, q, k, v, rank, peak_kind)
    clk = clocks.summary()
    model = output_kernel_model(path, w)
    out_avg_ms = statistics.mean(out_ms)
    roofline = roofline_of(path, w, out_avg_ms, tokens, peaks, peak_kind)
    roofline["traffic"] = _traffic_from_profiles(path, w)
    roofline["phase_ms"] = {"note": "separate loop with events between the kernels (serialised)",
                            "step": statistics.mean([ev[0].elapsed_time(ev[3]) for ev in events]),
                            "summary": statistics.mean(sum_ms), "scan": statistics.mean(scan_ms),
                            "output": out_avg_ms}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, q, k, v, g)

    # parity of the timed output itself: the fp64 oracle on every head and token (rank 0)
    parity = None
    if rank == 0 and not args.no_cpu_baseline:
        parity = parity_against_oracle(w, out, q, k, v, g)

    # the problem's five workloads at full size: throughput, the output kernel against its roofline,
    # and the full-output parity error against the oracle (rank 0, one GPU)
    workloads = None
    if rank == 0 and world == 1 and args.workload_steps > 0:
        del flush
        workloads = measure_workloads(dev, args, peaks, peak_kind, {w.name: (value, ms_per_step, roofline,
                                                                             parity)})

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
            "config": {"workload": w.name, "op": w.op, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "dv": w.dv,
                       "tokens_per_gpu": tokens, "path": path, "chunk": model["chunk"],
                       "segment_chunks": args.segment_chunks or "auto",
                       "l2": "flushed before every step (512 MiB write, outside the timed events)",
                       "parallelism": f"dp{world} (independent heads per rank, no collective)"},
            "roofline": roofline, "parity": parity, "cpu_baseline": cpu, "e2e": e2e, "decode": decode,
            "backward": backward, "workloads": workloads, "clocks": clk,
            "gpu_launches": launches_per_step * args.steps, "device_status": status,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


TOLERANCE = {"f32": 1e-4, "bf16": 2e-2}     # max row-wise relative L2 error against the fp64 oracle
FIVE = ("hla2_f32_1x2x256x32", "hla2n_bf16_4x16x4096x64", "hla2d_bf16_2x16x16384x64", "ahla_bf16_4x16x8192x64",
        "hla3_f32_2x8x4096x32")


def parity_against_oracle(w, out, q, k, v, g):
    """Max row-wise relative L2 error of a GPU output against the fp64 oracle over every head and
    token of the workload (the oracle runs on all host cores, one thread per head)."""
    import oracle
    ref = oracle.recur(w.op, q, k, v, gamma=g, eps=w.eps)
    err = oracle.max_row_rel_err(out.detach().cpu(), ref)
    return {"max_row_rel_err": err, "tol": TOLERANCE[w.dtype], "pass": err <= TOLERANCE[w.dtype],
            "rows": int(w.B * w.H * w.T), "against": "fp64 oracle (serial recurrence), every head and token"}


def roofline_of(path, w, out_ms, tokens, peaks, peak_kind):
    model = output_kernel_model(path, w)
    achieved = model["flops_per_token"] * tokens / (out_ms / 1e3) / 1e12
    if model["bound"] == "tensor" and path == "tc-output":
        # fp32 products from three bf16 products each (six for Q K^T): a third of the bf16 rate
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) / 3
        note = f"bf16 dense burst ({peak_kind}) / 3: each fp32 product is three bf16 products"
    elif model["bound"] == "tensor":
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        note = f"bf16 dense burst ({peak_kind})"
    else:
        smax = float(peaks.get("sm_max_mhz", 1965.0))
        peak = alu_peak_tflops(smax)
        note = f"FP32 FFMA 148x128x2 flop at {smax:.0f} MHz (derived)"
    return {"kernel": "output", "bound": model["bound"], "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "peak_source": note, "flops_per_token": model["flops_per_token"],
            "kernel_ms": out_ms}


def measure_workloads(dev, args, peaks, peak_kind, done):
    """Every one of the five workloads at its full size, one after the other on this GPU: forward
    throughput (CUDA events around each step, L2 flushed before it), the output kernel against its
    roofline (phase events), and the full-output parity error against the fp64 oracle."""
    import torch

    import higher_order_linear_chunked_b200 as hla
    res = {}
    flush = torch.empty(512 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)
    for name in FIVE:
        w = hla_inputs.workload(name)
        if name in done:
            value, ms, roof, par = done[name]
            res[name] = {"tokens_per_s": value, "ms_per_step": ms, "roofline_frac": roof["frac"],
                         "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "kernel_ms")},
                         "parity": par, "note": "the headline line above"}
            continue
        q, k, v, g = hla_inputs.make_inputs(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        gd = g.to(dev) if g is not None else None
        out = torch.empty((w.B, w.H, w.T, w.dv), dtype=torch.float32, device=dev)
        op = hla.OP_CODES[w.op]
        ws = hla.make_workspace(op, qd, vd, decayed=gd is not None)
        dcode = hla.HLA_BF16 if w.dtype == "bf16" else hla.HLA_F32
        path = {1: "tc", 2: "tc-output"}.get(hla.uses_tensor_cores(op, dcode, gd is not None, w.B, w.H, w.T, w.d, w.dv), "simt")
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            hla.forward(w.op, qd, kd, vd, gamma=gd, eps=w.eps, out=out, workspace=ws)
        torch.cuda.synchronize()
        bounds = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.workload_steps)]
        for a, b in bounds:
            flush.zero_()
            a.record()
            hla.forward(w.op, qd, kd, vd, gamma=gd, eps=w.eps, out=out, workspace=ws)
            b.record()
        torch.cuda.synchronize()
        ms = statistics.mean(a.elapsed_time(b) for a, b in bounds)
        status = hla.read_device_status(ws)
        par = parity_against_oracle(w, out, q, k, v, g)
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.workload_steps)]
        for ev in evs:
            for e in ev:
                e.record()
        torch.cuda.synchronize()
        for ev in evs:
            flush.zero_()
            hla.forward_profiled(w.op, qd, kd, vd, ev, gamma=gd, eps=w.eps, out=out, workspace=ws)
        torch.cuda.synchronize()
        out_ms = statistics.mean(ev[2].elapsed_time(ev[3]) for ev in evs)
        roof = roofline_of(path, w, out_ms, w.tokens, peaks, peak_kind)
        res[name] = {"tokens_per_s": w.tokens / (ms / 1e3), "ms_per_step": ms, "roofline_frac": roof["frac"],
                     "roofline": {k: roof[k] for k in ("bound", "achieved", "peak", "unit", "frac", "kernel_ms")},
                     "parity": par, "path": path, "dtype": w.dtype, "steps": args.workload_steps,
                     "device_status": status,
                     "config": {"op": w.op, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "dv": w.dv}}
        del qd, kd, vd, out, ws
    return res


def backward_measure(w, qd, kd, vd, flush, steps, peaks, q, k, v, rank, peak_kind="fallback"):
    """The backward pass of the workload's operator (the plain masked second order for hla2 and
    hla2n workloads, hla2_backward; AHLA for ahla workloads, ahla_backward) on its inputs with a
    seeded fp32 output gradient: time per call (CUDA events, L2 flushed before each), tokens/s,
    the gradient products against the peak of the units they run on, and a directional-derivative
    check of the result against the fp64 oracle's forward on one head (rank 0)."""
    import numpy as np
    import torch

    import higher_order_linear_chunked_b200 as hla
    dev = qd.device
    g = torch.Generator("cpu").manual_seed(w.seed + 1234)
    do = torch.randn(tuple(qd.shape[:3]) + (vd.shape[-1],), generator=g, dtype=torch.float32)
    dod = do.to(dev)
    ahla = w.op == "ahla"
    opc = hla.OP_AHLA if ahla else hla.OP_HLA2
    dtc = hla.HLA_BF16 if w.dtype == "bf16" else hla.HLA_F32
    run = hla.ahla_backward if ahla else hla.hla2_backward
    ws = torch.empty(hla.load_library().hla_backward_workspace_bytes(opc, dtc, w.B, w.H, w.T, w.d, w.dv),
                     dtype=torch.uint8, device=dev)
    for _ in range(3):
        grads = run(qd, kd, vd, dod, workspace=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        grads = run(qd, kd, vd, dod, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    ms = statistics.mean(times)
    D = w.d
    smax = float(peaks.get("sm_max_mhz", 1965.0))
    tensor = not ahla and w.dtype == "bf16" and D == 64
    if tensor:
        # tensor-core path, 128-token chunks, in multiply-adds per chunk (the two-term splits of dO
        # and dZ are precision work, not counted): adjoint terms (dO V^T, Q^T dO, Q^T V, dW Q,
        # Q^T (dW Q)), the cross term C dR'^T, and the gradients in the Z form (A, Q S0, A K, dO V^T,
        # dW^T Q, V dR'^T, Q Z^T, dZ K^T, K dS', A^T dZ, dO R0^T, dZ S0, W^T dO, Z dR', dW Z, dA K,
        # dA^T Q); the carried states it recomputes are not counted
        c = 128
        macs = (2 * c * c * D + 3 * c * D * D) + D ** 3 + (11 * c * c * D + 6 * c * D * D)
        peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
        bound, peak_source = "tensor", f"bf16 dense burst ({peak_kind})"
    elif ahla:
        # AHLA, CUDA cores, 64-token chunks: chunk terms (A, Q^T dO, Q^T K, A^T dO, Q^T (A^T dO)), the
        # cross term M dE', and the gradients (A, Y, dY, dA, dV, dQ, dK)
        c = 64
        macs = (2 * c * c * D + 3 * c * D * D) + D ** 3 + (8 * c * c * D + 7 * c * D * D)
        peak, bound = alu_peak_tflops(smax), "alu"
        peak_source = f"FP32 FFMA 148x128x2 flop at {smax:.0f} MHz (derived)"
    else:
        # second order, CUDA cores, 64-token chunks: chunk terms (Q^T dO, Q^T V, dO V^T, dW Q,
        # Q^T (dW Q)), the cross term C dR'^T, and the chunk gradients (A, P, dW, W, Z, dV, dZ, dP,
        # dA, dQ, dK); the forward summaries it recomputes are not counted
        c = 64
        macs = (3 * c * D * D + 2 * c * c * D) + D ** 3 + (8 * c * c * D + 6 * c * D * D + 2 * c ** 3 + 3 * c * c * D)
        peak, bound = alu_peak_tflops(smax), "alu"
        peak_source = f"FP32 FFMA 148x128x2 flop at {smax:.0f} MHz (derived)"
    flops_per_token = 2 * macs / c
    achieved = flops_per_token * w.tokens / (ms / 1e3) / 1e12
    check = None
    if rank == 0:
        b_, h_ = 0, 0
        rng = np.random.default_rng(0)
        import oracle
        qh, kh, vh, doh = (x[b_, h_].double().numpy() for x in (q, k, v, do))
        dirs = [rng.standard_normal(x.shape) for x in (qh, kh, vh)]
        eps = 1e-4

        def f(s):
            o = oracle.recur("ahla" if ahla else "hla2", (qh + s * dirs[0])[None, None],
                             (kh + s * dirs[1])[None, None], (vh + s * dirs[2])[None, None])[0, 0]
            return float(np.sum(o * doh))
        num = (f(eps) - f(-eps)) / (2 * eps)
        ana = sum(float(np.sum(gr[b_, h_].double().cpu().numpy() * dr)) for gr, dr in zip(grads, dirs))
        check = {"directional_derivative_rel_err": abs(ana - num) / max(1.0, abs(num)), "head": [b_, h_],
                 "against": "central difference of the fp64 oracle forward"}
    return {"op": "ahla" if ahla else "hla2 (plain masked second order)", "ms": ms,
            "tokens_per_s": w.tokens / (ms / 1e3),
            "gpu_launches_per_step": hla.load_library().hla_backward_kernel_launches(opc, dtc, w.B, w.H, w.T, w.d,
                                                                                     w.dv),
            "roofline": {"bound": bound, "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                         "frac": achieved / peak, "flops_per_token": flops_per_token, "scope": "whole call",
                         "peak_source": peak_source},
            "check": check, "l2": "flushed before every call (outside the events)"}


def decode_measure(w, qd, kd, vd, gd, flush, steps, peaks, peak_kind):
    """Streaming form: the prefill state of the workload's T tokens (hla_state), then `steps`
    one-token decode steps per head (hla_step), each timed alone with CUDA events after an L2
    flush.  A step reads and writes every head's state once: HBM-bound."""
    import torch

    import higher_order_linear_chunked_b200 as hla
    B, H, T, d = qd.shape
    dev = qd.device
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    st = hla.state(w.op, qd, kd, vd, gamma=gd)                      # warm-up prefill (not timed)
    flush.zero_()
    ev[0].record()
    st = hla.state(w.op, qd, kd, vd, gamma=gd, out=st)
    ev[1].record()
    torch.cuda.synchronize()
    prefill_ms = ev[0].elapsed_time(ev[1])
    toks = [(qd[:, :, t].contiguous(), kd[:, :, t].contiguous(), vd[:, :, t].contiguous()) for t in range(steps)]
    o = torch.empty((B, H, vd.shape[-1]), dtype=torch.float32, device=dev)
    for t in range(3):                                              # warm-up on a copy of the state
        hla.step(w.op, st.clone(), *toks[t % steps], gamma=gd, eps=w.eps, out=o)
    times = []
    for t in range(steps):
        flush.zero_()
        # a spin kernel keeps the stream busy while the host enqueues the step (the Python call
        # takes longer than the kernel), so the events time the device, not the host
        torch.cuda._sleep(200000)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        hla.step(w.op, st, *toks[t], gamma=gd, eps=w.eps, out=o)
        b.record()
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    step_ms = statistics.mean(times)
    host = []                                                       # host time of one call
    for t in range(steps):
        h0 = time.perf_counter()
        hla.step(w.op, st, *toks[t], gamma=gd, eps=w.eps, out=o)
        host.append(time.perf_counter() - h0)
        torch.cuda.synchronize()
    esz = qd.element_size()
    nbytes = B * H * (2 * st.shape[-1] * 4 + 3 * d * esz + vd.shape[-1] * 4)   # state in and out, q k v, o
    gbs = nbytes / (step_ms / 1e3) / 1e9
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    return {"prefill_ms": prefill_ms, "prefill_note": "second call (the first is a warm-up), L2 flushed before it",
            "prefill_tokens": B * H * T, "steps": steps, "us_per_step": step_ms * 1e3,
            "host_us_per_call": statistics.median(host) * 1e6,
            "timing": "events around each step with the stream kept busy before it (device time, the "
                      "event pair included); the host time of the Python call is reported apart",
            "tokens_per_s": B * H / (step_ms / 1e3), "gpu_launches_per_step": 1,
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "bytes_per_step": nbytes, "peak_source": f"HBM copy ({peak_kind})"},
            "l2": "flushed before every step (outside the events)"}


def _traffic_from_profiles(path, w):
    """DRAM bytes per launch of the output kernel from the committed ncu summary, when it was
    taken on this workload and on the kernel source as it is now (else None)."""
    import hashlib
    f = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(f):
        return None
    try:
        rec = json.load(open(f)).get(f"{path}:{w.name}")
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    src = os.path.join(ROOT, rec.get("kernel_source", "higher_order_linear_chunked_b200/csrc/tc_hla.cu"))
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest() if os.path.exists(src) else None
    if rec.get("kernel_source_sha256") != sha:
        return None
    return rec.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# CPU baseline and the reference arm: the fp64 oracle on the host cores
# ---------------------------------------------------------------------------

def cpu_baseline(w, q, k, v, g, max_tokens: int = 1 << 30):
    import oracle
    threads = os.cpu_count() or 1
    B, H, T = w.B, w.H, w.T
    # the whole workload (every head, every token) unless it is larger than max_tokens
    Ts = min(T, max(1, max_tokens // (B * H)))
    qs, ks, vs = q[:, :, :Ts], k[:, :, :Ts], v[:, :, :Ts]
    t0 = time.perf_counter()
    oracle.recur(w.op, qs, ks, vs, gamma=g, eps=w.eps, nthreads=threads)
    dt = time.perf_counter() - t0
    n = B * H * Ts
    return {"value": n / dt, "unit": UNIT, "cores": min(threads, B * H), "kind": "oracle",
            "sample": f"{B}x{H} heads x {Ts} tokens ({n} tokens) of the same workload, serial fp64 "
                      f"recurrence, one host thread per head, {dt:.2f} s"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = hla_inputs.workload(args.workload)
    q, k, v, g = hla_inputs.make_inputs(w)
    threads = os.cpu_count() or 1
    Ts = min(w.T, 1024)                         # bounded sample per step: every head, first Ts tokens
    qs, ks, vs = q[:, :, :Ts], k[:, :, :Ts], v[:, :, :Ts]
    n = w.B * w.H * Ts
    for _ in range(args.warmup):
        oracle.recur(w.op, qs, ks, vs, gamma=g, eps=w.eps, nthreads=threads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.recur(w.op, qs, ks, vs, gamma=g, eps=w.eps, nthreads=threads)
    dt = time.perf_counter() - t0
    value = n * args.steps / dt
    sample = (f"{w.B}x{w.H} heads x first {Ts} tokens ({n} tokens) per step, serial fp64 recurrence "
              f"(the oracle), one host thread per head")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "op": w.op, "B": w.B, "H": w.H, "T": w.T, "d": w.d, "dv": w.dv},
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": min(threads, w.B * w.H), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
