#!/usr/bin/env python
"""Benchmark of the direct NVFP4 Newton-Schulz step (Q-Root, "Full-Stack FP4"
Section 3.4) on B200: one JSON line on rank 0.

A step is one fs4_root_ns_batched call over every matrix of the workload
(normalise + clip + quantise, then K iterations of the three NVFP4 products),
inputs resident in HBM.  Default workload: the full 28-block set of a 3B-class
decoder (196 matrices: per block Q/K/V/O 3072x3072, gate/up 8192x3072, down
3072x8192), Student-t (nu = 3) momenta at RMS 0.02, the Muon coefficients passed
per matrix, K = 5, one batched call; the largest workload that fits one GPU.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]
                  [--shard replicas|lpt]

Multi-GPU (torchrun): every rank runs the whole workload on its own GPU (the
matrices are independent; no collective on the data path), so per-GPU work is
fixed and the scaling is weak; the step time is the max over ranks.  With
--shard lpt the ranks instead split one workload (longest processing time first
over the algorithmic FLOPs) and one NCCL all-gather returns every update to every
rank: strong scaling.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "3b_28blocks_student"
METRIC = "NVFP4 Newton-Schulz matrices/s (K=5 iterations per matrix)"
UNIT = "matrices/s"


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--source", default="fp32", choices=["fp32", "nvfp4"],
                    help="ns: the momenta as FP32 matrices, or as NVFP4 first-moment states "
                         "(fs4_root_ns_batched_nvfp4; states written once by fs4_momentum_nvfp4)")
    ap.add_argument("--per-matrix", action="store_true",
                    help="--op quantize: one fs4_nvfp4_quantize call per matrix instead of one "
                         "fs4_nvfp4_quantize_batched call per step")
    ap.add_argument("--no-bf16", action="store_true",
                    help="skip the BF16 comparison step (same plan, BF16 operands)")
    ap.add_argument("--op", default="ns", choices=["ns", "quantize", "dequantize", "momentum"],
                    help="ns: the Newton-Schulz step (default); quantize / dequantize: the standalone "
                         "NVFP4 calls over every matrix of the workload (row axis); momentum: one "
                         "NVFP4 first-moment step (fs4_momentum_nvfp4) per matrix")
    ap.add_argument("--layout", default="plain", choices=["plain", "tiled"],
                    help="NVFP4 layout of --op quantize / dequantize")
    ap.add_argument("--clip", default="rms", choices=["rms", "p99"],
                    help="clip rule of the preamble: 3 x RMS (default) or the 0.99 quantile of "
                         "|X_0| (Section 3.4 p99 outlier clipping, FS4_NS_CLIP_QUANTILE)")
    ap.add_argument("--graph", action="store_true",
                    help="ns: capture one call in a CUDA graph and replay it per step (for the "
                         "launch-bound small workloads; per-phase times then come from a "
                         "separate untimed pass of the event-recording call)")
    ap.add_argument("--quant", default="plain", choices=["plain", "rht46", "rht", "a46"],
                    help="quantiser of the step: plain NVFP4 (default) or the Section 3.4 options "
                         "(random Hadamard transform with fresh seeded sign masks, adaptive 4/6)")
    ap.add_argument("--shard", default="replicas", choices=["replicas", "lpt"],
                    help="ns across ranks: replicas (default; every rank runs the whole workload on "
                         "its own matrices, weak scaling, no collective) or lpt (one model's matrices "
                         "split by longest processing time over the algorithmic FLOPs, one NCCL "
                         "all-gather of the updates, strong scaling)")
    return ap.parse_args()


def rank_seed(base_seed: int, rank: int) -> int:
    """Seed of the workload matrices of one rank: every rank runs the whole workload on
    its own matrices (replicas; the matrices are independent, no collective)."""
    return base_seed + 1000 * rank


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The largest value over all ranks (step times: the job is as slow as its slowest
    rank).  Uses the default process group; `device` is "cuda" under NCCL, "cpu" under gloo."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(world: int, units_per_rank: float, ms_step: float) -> float:
    """Whole-job throughput: the units every rank processed per step over the slowest
    rank's step time."""
    return world * units_per_rank / (ms_step * 1e-3)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "of measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "of fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


def phase_kinds(K):
    """Kernel launched in each timed phase of one call (3 + 3K events)."""
    kinds = ["reduce", "preamble"]
    for _ in range(K):
        kinds += ["gram_x", "gram_a", "update"]
    return kinds


def flops_per_launch(w, kind):
    tot = 0.0
    for (r, c) in w.shapes:
        m, n = min(r, c), max(r, c)
        if kind == "gram_x":
            tot += m * (m + 1) * n
        elif kind == "gram_a":
            tot += m * (m + 1) * m
        elif kind == "update":
            tot += 2 * m * m * n
    return tot


def bytes_per_launch(w, kind):
    """Algorithmic HBM bytes of one launch of each phase: every tensor the phase must read
    or write once (for the products: their FP32 inputs and outputs and their NVFP4
    operands and views; the re-reads of operand tiles between output tiles are an
    implementation cost and not counted).  Per matrix in working orientation m <= n:
      reduce    4 mn (G)
      preamble  4 mn (G) + 4 mn (X_0) + 2 x 0.5625 mn (both views)
      gram_x    0.5625 mn (qX) + 4 m^2 (T+1)/(2T) (A, the 256 x 256 tiles on and above the
                diagonal, T = m/256) + 0.5625 m^2 (qA, both triangles)
      gram_a    4 m^2 (T+1)/(2T) (A) + 0.5625 m^2 (qA) + 0.5625 m^2 (qB)
      update    0.5625 m^2 (qB) + 0.5625 mn (qX16x1) + 4 mn (X) + 4 mn (X') + 2 x 0.5625 mn
                (both views of X'; the last update writes the FP32 output instead)"""
    tot = 0.0
    for (r, c) in w.shapes:
        m, n = min(r, c), max(r, c)
        e = m * n
        tiles = max(1, (m + 255) // 256)
        upper = 4.0 * m * m * (tiles + 1) / (2 * tiles)
        if kind == "reduce":
            tot += 4 * e
        elif kind == "preamble":
            tot += 4 * e + 4 * e + 2 * (e / 2 + e / 16)
        elif kind == "gram_x":
            tot += 0.5625 * e + upper + 0.5625 * m * m
        elif kind == "gram_a":
            tot += upper + 2 * 0.5625 * m * m
        elif kind == "update":
            tot += 0.5625 * m * m + 0.5625 * e + 8 * e + 2 * 0.5625 * e
    return tot


def bf16_comparator(F, Gs, w, steps: int, flush, l2_bytes: int):
    """Time the BF16 comparison step (fs4_root_ns_bf16_batched: the same Newton-Schulz
    plan with BF16 operands on tcgen05 kind::f16) on the same matrices, per phase with
    CUDA events on the launching stream; the pages compare Q-Root with an optimized
    BF16 implementation of the same step (Full-Stack FP4, Section 4.4, Table 6)."""
    import torch
    lib = F._lib.lib()
    K = w.K
    outs = [torch.empty_like(G) for G in Gs]
    arr = F._descs(Gs, outs, w.coeffs)
    need = int(lib.fs4_root_ns_bf16_batched_workspace_size(len(Gs), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    n_ev = 3 + 3 * K
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(steps)]
    for row in evs:
        for e in row:
            e.record(stream)

    def call(row=None):
        if row is None:
            st = lib.fs4_root_ns_bf16_batched(len(Gs), arr, K, w.clip_k, 0, ws.data_ptr(), need,
                                              stream.cuda_stream)
        else:
            ev_arr = (F._lib.c_vp * n_ev)(*[e.cuda_event for e in row])
            st = lib.fs4_root_ns_bf16_batched_timed(len(Gs), arr, K, w.clip_k, 0, ws.data_ptr(), need,
                                                    stream.cuda_stream, ev_arr, n_ev)
        F.check(st, "fs4_root_ns_bf16_batched")

    for _ in range(3):
        call()
    torch.cuda.synchronize()
    for row in evs:
        if flush is not None:
            flush.zero_()
        call(row)
    torch.cuda.synchronize()
    F.check(F.device_status(ws), "device status after the BF16 comparison steps")
    ms = statistics.mean(row[0].elapsed_time(row[-1]) for row in evs)
    kinds = phase_kinds(K)
    per_kind = {}
    for row in evs:
        for i, kind in enumerate(kinds):
            per_kind.setdefault(kind, []).append(row[i].elapsed_time(row[i + 1]))
    phase = {k: statistics.mean(v) * (1 if k in ("reduce", "preamble") else K) for k, v in per_kind.items()}
    del ws, outs
    torch.cuda.empty_cache()
    return ms, phase


QUANT_NAMES = {"plain": "NVFP4 RTN (H = I, M = 6)",
               "rht46": "NVFP4 RTN with H16^r (fresh signs per step) and adaptive 4/6",
               "rht": "NVFP4 RTN with H16^r (fresh signs per step)",
               "a46": "NVFP4 RTN with adaptive 4/6"}


def ns_config(w, quant: str, clip: str, world: int) -> dict:
    """The workload keys of a Newton-Schulz bench line (the same for both arms)."""
    return {"workload": w.name, "matrices": len(w.shapes), "shapes": sorted(set(map(tuple, w.shapes))),
            "K": w.K, "coeffs": "Muon (3.4445, -4.7750, 2.0315)",
            "clip": "3 x RMS" if clip == "rms" else "0.99 quantile of |X_0| (nearest rank)",
            "quantiser": QUANT_NAMES[quant],
            "parallelism": f"replicas x{world} (independent matrices, no collective)"}


def oracle_sample_rate(w, budget_s: float, quant: str = "plain", clip: str = "rms"):
    """Time the oracle (as it stands) on one bounded sample of the workload:
    one NVFP4 Newton-Schulz iteration of an m x n slice of its first matrix (the whole
    matrix when that fits the budget), with the quantiser options and clip rule of the run.
    It runs the C++ oracle (OpenMP over rows, float64 triple loops, no BLAS), which
    implements the plain step and every option (H16^r, adaptive 4/6, the quantile clip).
    Returns (matrices/s extrapolated by algorithmic FLOPs, seconds, description, cores)."""
    import numpy as np
    from oracle import cpp_oracle as C
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, generate
    r0, c0 = w.shapes[0]
    m_full, n_full = min(r0, c0), max(r0, c0)
    G = generate((m_full, n_full), w.dist, BASE_SEED, "cpu").numpy()
    masks = None
    if quant in ("rht", "rht46"):
        masks = [int(v) for v in np.random.default_rng(BASE_SEED + 7).integers(0, 1 << 16, 3)]
    a46 = quant in ("a46", "rht46")
    cores = C.threads()
    m = m_full
    while True:
        if clip == "p99":
            X0 = C.normalise_and_clip(G[:m], None, clip_quantile=0.99)[0]
        else:
            X0 = C.normalise_and_clip(G[:m], w.clip_k)[0]
        t0 = time.perf_counter()
        C.ns_iterations_nvfp4(X0, 1, *w.coeffs[0], rht_masks=masks, adaptive46=a46)
        dt = time.perf_counter() - t0
        if dt <= budget_s or m <= 256:
            break
        m //= 2
    f_sample = m * (m + 1) * n_full + m * (m + 1) * m + 2 * m * m * n_full
    f_matrix = w.K * (m_full * (m_full + 1) * n_full + m_full * (m_full + 1) * m_full
                      + 2 * m_full * m_full * n_full)
    per_matrix_s = dt * f_matrix / f_sample
    which = "C++ oracle (OpenMP over rows, float64 triple loops, no BLAS, exact NVFP4 emulation)"
    desc = (f"{which}: one NVFP4 NS iteration of a {m}x{n_full} slice of the first "
            f"{m_full}x{n_full} matrix, {dt:.2f} s on {cores} threads, extrapolated by algorithmic "
            f"FLOPs to K={w.K} iterations of one full matrix")
    return 1.0 / per_matrix_s, dt, desc, cores


QD_BYTES = 4.5625          # algorithmic bytes per element: 4 B of FP32 + 0.5 B of codes + 1/16 B of scale
MO_BYTES = 9.125   # momentum step: read g (4 B) and the state (0.5625 B), write m_t (4 B) and the state
MO_METRIC = "NVFP4 first-moment step GB/s (9.125 B per element)"
QD_METRIC = {"quantize": "NVFP4 standalone quantise GB/s (4.5625 B per element)",
             "dequantize": "NVFP4 standalone dequantise GB/s (4.5625 B per element)"}


def oracle_qd_rate(w, op: str, budget_s: float):
    """Time the C++ oracle's quantiser (or dequantiser) on leading rows of the workload's
    first matrix, growing the slice until it takes about budget_s / 4 seconds.
    Returns (algorithmic GB/s, seconds, description, cores)."""
    from oracle import cpp_oracle as C
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, generate
    G = generate(w.shapes[0], w.dist, BASE_SEED, "cpu").numpy()
    rows = 16
    while True:
        x = np.ascontiguousarray(G[:rows])
        if op == "quantize":
            t0 = time.perf_counter()
            C.quantize_rows(x)
            dt = time.perf_counter() - t0
        else:
            c, sc, g = C.quantize_rows(x)
            t0 = time.perf_counter()
            C.dequantize_rows(c, sc, g)
            dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or rows >= G.shape[0]:
            break
        rows = min(G.shape[0], rows * 4)
    rate = x.size * QD_BYTES / dt / 1e9
    cores = C.threads()
    desc = (f"C++ oracle {op} (exact NVFP4 emulation, OpenMP over rows) of the first {rows} rows "
            f"of a {G.shape[0]}x{G.shape[1]} workload matrix, {dt:.2f} s on {cores} threads")
    return rate, dt, desc, cores


def run_reference(args):
    from nvfp4_precision_optimizer_b200.workloads import WORKLOADS
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    if args.op == "momentum":
        run_momentum_reference(args, w)
        return
    if args.op != "ns":
        rates, desc, cores = [], "", 1
        for i in range(args.warmup + args.steps):
            rate, dt, desc, cores = oracle_qd_rate(w, args.op, max(2.0, 120.0 / max(1, args.steps + args.warmup)))
            if i >= args.warmup:
                rates.append(rate)
        value = statistics.median(rates)
        total = sum(r * c for r, c in w.shapes) * QD_BYTES
        line = {
            "impl": "reference", "metric": QD_METRIC[args.op], "value": value, "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1000.0 * total / (value * 1e9), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32 values, exact NVFP4 emulation",
            "data": "synthetic", "config": {"workload": w.name, "matrices": len(w.shapes), "op": args.op,
                                            "layout": "plain"},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        }
        print(json.dumps(line), flush=True)
        return
    budget = max(5.0, 150.0 / max(1, args.steps + args.warmup))
    rates, secs = [], []
    desc, cores = "", 1
    for i in range(args.warmup + args.steps):
        rate, dt, desc, cores = oracle_sample_rate(w, budget, args.quant, args.clip)
        if i >= args.warmup:
            rates.append(rate)
            secs.append(dt)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        # each timed step is one bounded sample (one iteration of one matrix slice): its
        # own wall time; the value is that sample's rate extrapolated to the workload
        "ms_per_step": 1000.0 * statistics.median(secs),
        "step": "one bounded sample per step (see cpu_baseline.sample); value extrapolated by FLOPs",
        "ms_per_workload_extrapolated": 1000.0 * len(w.shapes) / value,
        "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64 products, fp32 tensors",
        "data": "synthetic", "config": ns_config(w, args.quant, args.clip, args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    import torch
    import torch.distributed as dist

    import nvfp4_precision_optimizer_b200 as F
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, WORKLOADS, matrices

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(v: float) -> float:
        return max_over_ranks(v, world, "cuda")

    w = WORKLOADS[args.workload]
    if args.op == "momentum":
        run_momentum(args, w, rank, world, local, barrier, ranks_max)
        if world > 1:
            dist.destroy_process_group()
        return
    if args.op != "ns":
        run_standalone(args, w, rank, world, local, barrier, ranks_max)
        if world > 1:
            dist.destroy_process_group()
        return
    if args.shard == "lpt":
        run_sharded(args, w, rank, world, local, barrier, ranks_max)
        if world > 1:
            dist.destroy_process_group()
        return
    K = w.K
    Gs = matrices(w, device="cuda", seed=rank_seed(BASE_SEED, rank))
    outs = [torch.empty_like(G) for G in Gs]
    arr = F._descs(Gs, outs, w.coeffs)
    lib = F._lib.lib()
    need = int(lib.fs4_root_ns_batched_workspace_size(len(Gs), arr))
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()
    n_ev = 3 + 3 * K

    qflags = {"plain": 0, "rht46": F.FS4_NS_RHT | F.FS4_NS_ADAPTIVE46, "rht": F.FS4_NS_RHT,
              "a46": F.FS4_NS_ADAPTIVE46}[args.quant]
    clip_arg = w.clip_k
    if args.clip == "p99":
        qflags |= F.FS4_NS_CLIP_QUANTILE
        clip_arg = 0.99
    mask_rng = np.random.default_rng(BASE_SEED + 7)

    if args.graph and qflags & F.FS4_NS_RHT:
        raise SystemExit("--graph: a captured call would replay the same H16^r signs every step")

    states = sarr = None
    if args.source == "nvfp4":
        # the momenta as NVFP4 first-moment states (one fs4_momentum_nvfp4 step from an empty
        # state each); the step then reads the states in place of FP32 G
        states = [F.momentum_nvfp4(G, 0.9, None, mask=0x5A5A, seed=BASE_SEED + i, want_m=False)[1]
                  for i, G in enumerate(Gs)]
        sarr = (F._lib.Nvfp4State * len(Gs))()
        for i, (G, st) in enumerate(zip(Gs, states)):
            sarr[i] = F._lib.Nvfp4State(st[0].data_ptr(), st[1].data_ptr(), st[2].data_ptr(), 0x5A5A)
            arr[i].G = None
        torch.cuda.synchronize()
        del Gs
        Gs = [torch.empty((1, 1), device="cuda") for _ in sarr]   # shapes come from the descriptors
        need = int(lib.fs4_root_ns_batched_workspace_size(len(sarr), arr))

    def call(events=None):
        masks = None
        if qflags & F.FS4_NS_RHT:        # fresh signs for every step (Section 3.4)
            masks = (ctypes.c_uint16 * (3 * K))(*[int(v) for v in mask_rng.integers(0, 1 << 16, 3 * K)])
        mptr = ctypes.cast(masks, ctypes.c_void_p) if masks is not None else None
        cur = torch.cuda.current_stream().cuda_stream   # the capture stream under --graph
        if sarr is not None:
            ev_arr = None if events is None else (F._lib.c_vp * n_ev)(*[e.cuda_event for e in events])
            if ev_arr is None:
                st = lib.fs4_root_ns_batched_nvfp4(len(sarr), arr, sarr, K, clip_arg, qflags, mptr,
                                                   ws.data_ptr(), need, cur)
            else:
                st = lib.fs4_root_ns_batched_nvfp4_timed(len(sarr), arr, sarr, K, clip_arg, qflags, mptr,
                                                         ws.data_ptr(), need, cur, ev_arr, n_ev)
            F.check(st, "fs4_root_ns_batched_nvfp4")
            return
        if events is None:
            st = lib.fs4_root_ns_batched_ex(len(Gs), arr, K, clip_arg, qflags, mptr, ws.data_ptr(),
                                            need, cur)
        else:
            ev_arr = (F._lib.c_vp * n_ev)(*[e.cuda_event for e in events])
            st = lib.fs4_root_ns_batched_timed(len(Gs), arr, K, clip_arg, qflags, mptr, ws.data_ptr(),
                                               need, cur, ev_arr, n_ev)
        F.check(st, "fs4_root_ns_batched")

    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    F.check(F.device_status(ws), "device status after warm-up")
    graph = None
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            call()
        for _ in range(max(3, args.warmup)):
            graph.replay()
        torch.cuda.synchronize()
        F.check(F.device_status(ws), "device status after graph warm-up")

    step_events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)] for _ in range(args.steps)]
    for evs in step_events:          # torch creates the CUDA event on its first record
        for e in evs:
            e.record(stream)
    # Inputs that fit in L2 would be read from L2 by the next step: then L2 is flushed
    # (a zero-fill of twice its size) before every step, and the step time is taken from
    # the events around each call, so that the fill stays outside the timed work.
    in_bytes = (sum(G.numel() for G in Gs) * 4 if states is None
                else sum(st[0].numel() + st[1].numel() for st in states))
    l2_bytes = int(torch.cuda.get_device_properties(local).L2_cache_size)
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device="cuda") if in_bytes <= 2 * l2_bytes else None
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    replay_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(args.steps)] if graph is not None else []
    with sampler:
        time.sleep(0.3)
        t_start.record(stream)
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()
            if graph is not None:
                replay_events[s][0].record(stream)
                graph.replay()
                replay_events[s][1].record(stream)
            else:
                call(step_events[s])
        t_end.record(stream)
        torch.cuda.synchronize()
    barrier()
    F.check(F.device_status(ws), "device status after timed steps")
    if graph is not None:
        total_ms = ranks_max(sum(a.elapsed_time(b) for a, b in replay_events))
    elif flush is None:
        total_ms = ranks_max(t_start.elapsed_time(t_end))
    else:
        total_ms = ranks_max(sum(evs[0].elapsed_time(evs[-1]) for evs in step_events))
    if flush is None:
        l2_note = "inputs larger than L2 (%.2f GB per step)" % (in_bytes / 1e9)
    else:
        l2_note = ("L2 flushed before every step (zero-fill of %d MB; inputs %.1f MB); step time "
                   "from events around each call" % (2 * l2_bytes >> 20, in_bytes / 1e6))
    ms_step = total_ms / args.steps
    if graph is not None:
        # per-phase times (roofline entry): a separate, untimed pass of the event-recording call
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()
            call(step_events[s])
        torch.cuda.synchronize()
        F.check(F.device_status(ws), "device status after the per-phase pass")

    # per-phase kernel durations (CUDA events on the launching stream)
    kinds = phase_kinds(K)
    per_kind = {}
    for evs in step_events:
        for i, kind in enumerate(kinds):
            per_kind.setdefault(kind, []).append(evs[i].elapsed_time(evs[i + 1]))
    totals = {k: sum(v) for k, v in per_kind.items()}
    dom = max(totals, key=totals.get)
    dom_ms = statistics.mean(per_kind[dom])
    peaks, peak_src = measured_peaks()
    # The GEMM kernels are timed one launch at a time (milliseconds each), so the
    # burst figure is the denominator: dense FP4 = 4 x the burst bf16 GEMM rate.
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    # The dominant kernel's roofline is the larger of its two floors: algorithmic FLOPs at
    # the dense-FP4 peak and algorithmic bytes at the HBM peak.  (The update product of the
    # 3072-row matrices moves 9.7 bytes of epilogue data per element of X for 2m FLOPs, so
    # at m = 3072 its HBM floor is above its tensor floor.)
    hbm_ach = bytes_per_launch(w, dom) / (dom_ms * 1e-3) / 1e9
    hbm = {"bound": "hbm", "achieved": hbm_ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
           "frac": hbm_ach / peaks["hbm_gbs"], "bytes_per_launch": bytes_per_launch(w, dom)}
    if dom in ("gram_x", "gram_a", "update"):
        achieved = flops_per_launch(w, dom) / (dom_ms * 1e-3) / 1e12
        ten = {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
               "frac": achieved / fp4_peak, "flops_per_launch": flops_per_launch(w, dom)}
        t_flop = flops_per_launch(w, dom) / (fp4_peak * 1e12)
        t_byte = bytes_per_launch(w, dom) / (peaks["hbm_gbs"] * 1e9)
        roof = dict(hbm if t_byte > t_flop else ten)
        roof["other_bound"] = ten if t_byte > t_flop else hbm
    else:
        roof = dict(hbm)
    roof["kernel"] = dom
    roof["ms_per_launch"] = dom_ms
    roof["peak_source"] = (f"dense FP4 = 4 x bf16_tflops, the burst figure ({peak_src} MEASURED_PEAKS.json; "
                           f"4 = nominal FP4/BF16 dense ratio); HBM = hbm_gbs ({peak_src} "
                           f"MEASURED_PEAKS.json)")
    roof["traffic"] = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
        ent = tr.get(args.workload, {}).get(dom)
        files = F.GEMM_SOURCES if dom in ("gram_x", "gram_a", "update") else F.ELEMENTWISE_SOURCES
        if ent and ent.get("source_sha") == F._source_digest(files):
            roof["traffic"] = ent["bytes_per_launch"]

    value = job_rate(world, len(Gs), ms_step)
    tflops = world * w.flops_algorithmic() / (ms_step * 1e-3) / 1e12
    phase_ms = {k: statistics.mean(v) * (1 if k in ("reduce", "preamble") else K) for k, v in per_kind.items()}

    comparator = None
    if not args.no_bf16 and args.quant == "plain" and args.clip == "rms" and states is None:
        bms, bphase = bf16_comparator(F, Gs, w, max(2, min(args.steps, 5)), flush, l2_bytes)
        peaks_b, _ = measured_peaks()
        bf16_tflops = w.flops_algorithmic() / (bms * 1e-3) / 1e12
        comparator = {
            "precision": "bf16 operands (tcgen05 kind::f16), fp32 accumulate, same plan and fusion",
            "ms_per_step": bms, "value": job_rate(world, len(Gs), bms), "unit": UNIT,
            "tflops_algorithmic": bf16_tflops,
            "frac_bf16_peak": bf16_tflops / peaks_b["bf16_tflops"],
            "nvfp4_speedup": bms / ms_step,
            "phase_ms_per_step": bphase,
            "context": "Full-Stack FP4 Table 6 (RTX 5090, d = 4096): Root BF16 344.55 ms vs NVFP4 "
                       "109.80 ms per optimizer step (3.14x)",
        }

    # end to end through the public API with host buffers: every step copies its inputs
    # in from pinned host memory, runs the call and copies its outputs back.  Steps are
    # pipelined on three streams (copy-in, compute, copy-out) with double-buffered
    # device tensors, so step i's copies overlap steps i - 1 and i + 1.
    e2e = None
    if not args.no_e2e and states is None:
        host_in = [G.cpu().pin_memory() for G in Gs]
        # one pinned host set for the results: the copy-out stream writes it step after
        # step in order (nothing reads it in between), so the device side alone is
        # double-buffered and the pinned host memory stays at twice the input size
        host_out = [torch.empty(G.shape, dtype=torch.float32).pin_memory() for G in Gs]
        dev_in = [Gs, [torch.empty_like(G) for G in Gs]]
        dev_out = [outs, [torch.empty_like(o) for o in outs]]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        e2e_steps = max(2, min(args.steps, 6))
        ev = {key: [torch.cuda.Event() for _ in range(2)] for key in ("in", "done", "out")}
        for key in ev:                   # create the CUDA events before the timed region
            for e in ev[key]:
                e.record(stream)

        def e2e_step(i):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev["done"][b])        # step i - 2 finished reading dev_in[b]
                for G, h in zip(dev_in[b], host_in):
                    G.copy_(h, non_blocking=True)
                ev["in"][b].record(s_in)
            stream.wait_event(ev["in"][b])
            if i >= 2:
                stream.wait_event(ev["out"][b])           # step i - 2's outputs were copied out
            masks = ([int(v) for v in mask_rng.integers(0, 1 << 16, 3 * K)]
                     if qflags & F.FS4_NS_RHT else None)
            F.root_ns_batched(dev_in[b], K=K, coeffs=w.coeffs, clip_k=w.clip_k, outs=dev_out[b],
                              workspace=ws, stream=stream, rht_masks=masks,
                              adaptive46=bool(qflags & F.FS4_NS_ADAPTIVE46),
                              clip_quantile=0.99 if args.clip == "p99" else None)
            ev["done"][b].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev["done"][b])
                for o, h in zip(dev_out[b], host_out):
                    h.copy_(o, non_blocking=True)
                ev["out"][b].record(s_out)

        e2e_step(0)                      # warm-up of the pipeline's streams
        e2e_step(1)
        torch.cuda.synchronize()
        barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        for i in range(e2e_steps):
            e2e_step(i)
        stream.wait_event(ev["out"][0])
        stream.wait_event(ev["out"][1])
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        F.check(F.device_status(ws), "device status after the end-to-end steps")
        e2e_ms = ranks_max(e0.elapsed_time(e1)) / e2e_steps
        nbytes = sum(G.numel() * 4 for G in Gs)
        e2e = {"value": job_rate(world, len(Gs), e2e_ms), "unit": UNIT,
               "h2d_bytes_per_step": nbytes, "d2h_bytes_per_step": nbytes,
               "ms_per_step": e2e_ms,
               "pipeline": "copy-in, compute and copy-out of consecutive steps overlap on three "
                           "streams (double-buffered device tensors)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, desc, cores = oracle_sample_rate(w, 20.0, args.quant, args.clip)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": desc}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "nvfp4 (e2m1 x e4m3/16) products, fp32 accumulate",
            "data": "synthetic",
            "config": {**ns_config(w, args.quant, args.clip, world),
                       "source": ("NVFP4 first-moment states (fs4_root_ns_batched_nvfp4)"
                                  if states is not None else "FP32 momenta"),
                       "l2": l2_note,
                       "launch": ("one CUDA graph replay per step (the call captured once); per-phase "
                                  "times from a separate event-recording pass" if graph is not None
                                  else "one library call per step (stream launches)")},
            "tflops_algorithmic": tflops,
            "frac_fp4_peak_algorithmic": tflops / world / fp4_peak,
            "tflops_dense_equivalent": world * w.flops_dense() / (ms_step * 1e-3) / 1e12,
            "phase_ms_per_step": phase_ms,
            "roofline": roof,
            "comparator": comparator,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": args.steps * (2 + 6 * K + (3 if args.clip == "p99" else 0)),
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def run_sharded(args, w, rank, world, local, barrier, ranks_max):
    """--shard lpt: one model's matrices split across the ranks (longest processing time
    first over the algorithmic FLOPs; nvfp4_precision_optimizer_b200.shard).  Each rank runs
    the step (fs4_root_ns_batched) on its share, then one NCCL all-gather returns every
    update to every rank.  A step is both; its time is the maximum over ranks of the CUDA
    events around them, and the value is the model's matrices over that time.  The total
    work is fixed as N grows ("scaling": "strong").  The plain step on FP32 momenta only."""
    import torch

    import nvfp4_precision_optimizer_b200 as F
    from nvfp4_precision_optimizer_b200 import shard
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, generate
    if args.quant != "plain" or args.clip != "rms" or args.source != "fp32" or args.graph:
        raise SystemExit("--shard lpt runs the plain step on FP32 momenta "
                         "(no --quant, --clip, --source or --graph)")
    K = w.K
    S = shard.ShardedRootNS(w.shapes, K=K, coeffs=w.coeffs, rank=rank, world=world, device="cuda",
                            clip_k=w.clip_k)
    mine = set(S.local)
    # one model on every rank: matrix i is seeded with BASE_SEED + i everywhere; a rank
    # holds only the momenta it owns
    Gs = [generate(s, w.dist, BASE_SEED + i, "cuda") if i in mine else None
          for i, s in enumerate(w.shapes)]
    stream = torch.cuda.current_stream()

    def status(what):
        if S.workspace is not None:
            F.check(F.device_status(S.workspace), what)

    for _ in range(max(3, args.warmup)):
        S(Gs)
    torch.cuda.synchronize()
    status("device status after warm-up")
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for evs in ev:                   # torch creates the CUDA event on its first record
        for e in evs:
            e.record(stream)
    in_bytes = sum(G.numel() * 4 for G in Gs if G is not None)
    l2_bytes = int(torch.cuda.get_device_properties(local).L2_cache_size)
    flush = torch.empty(2 * l2_bytes, dtype=torch.uint8, device="cuda") if in_bytes <= 2 * l2_bytes else None
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler:
        time.sleep(0.3)
        for s in range(args.steps):
            if flush is not None:
                flush.zero_()
            ev[s][0].record(stream)
            S.compute_local(Gs)
            ev[s][1].record(stream)
            S.gather()
            ev[s][2].record(stream)
        torch.cuda.synchronize()
    barrier()
    status("device status after timed steps")
    ms_step = ranks_max(sum(e[0].elapsed_time(e[2]) for e in ev)) / args.steps
    ns_ms = ranks_max(statistics.mean(e[0].elapsed_time(e[1]) for e in ev))
    ag_ms = ranks_max(statistics.mean(e[1].elapsed_time(e[2]) for e in ev))
    n = len(w.shapes)
    value = n / (ms_step * 1e-3)
    gathered = world * S.plan.chunk * 4 if world > 1 else 0
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None,
            "dtype": "nvfp4 (e2m1 x e4m3/16) products, fp32 accumulate", "data": "synthetic",
            "config": {**ns_config(w, args.quant, args.clip, world),
                       "parallelism": (f"lpt x{world}: the model's {n} matrices split by longest "
                                       f"processing time over algorithmic FLOPs, one NCCL all-gather "
                                       f"of the updates" if world > 1 else "one GPU, no collective"),
                       "load_imbalance": S.plan.imbalance,
                       "l2": ("inputs larger than L2 (%.2f GB per rank per step)" % (in_bytes / 1e9)
                              if flush is None else "L2 flushed before every step")},
            "split_ms": {"share_step_max_over_ranks": ns_ms, "all_gather_max_over_ranks": ag_ms},
            "all_gather_recv_bytes_per_rank": gathered,
            "tflops_algorithmic": w.flops_algorithmic() / (ms_step * 1e-3) / 1e12,
            "roofline": None, "cpu_baseline": None, "e2e": None,
            "note": "per-phase roofline, CPU baseline and end-to-end figures come from the default mode",
            "gpu_launches": args.steps * (2 + 6 * K) if S.local else 0,
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)


def run_standalone(args, w, rank, world, local, barrier, ranks_max):
    """--op quantize / dequantize: one step = one fs4_nvfp4_quantize_batched call over every
    matrix of the workload (--per-matrix: one fs4_nvfp4_quantize call per matrix), or one
    fs4_nvfp4_dequantize call per matrix; row axis, outputs preallocated."""
    import torch
    import nvfp4_precision_optimizer_b200 as F
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, matrices

    lib = F._lib.lib()
    tiled = args.layout == "tiled"
    flags = F.FS4_LAYOUT_TILED if tiled else 0
    Gs = matrices(w, device="cuda", seed=rank_seed(BASE_SEED, rank))
    stream = torch.cuda.current_stream()
    qws_bytes = int(lib.fs4_nvfp4_quantize_workspace_size())
    bufs = []
    for G in Gs:
        R, C = G.shape
        nc, ns = F.tiled_shape(R, C) if tiled else (R * C // 2, R * C // 16)
        bufs.append({"codes": torch.empty(nc, dtype=torch.uint8, device="cuda"),
                     "scales": torch.empty(ns, dtype=torch.uint8, device="cuda"),
                     "sg": torch.empty(1, dtype=torch.float32, device="cuda"),
                     "ws": torch.zeros(qws_bytes, dtype=torch.uint8, device="cuda"),
                     "y": torch.empty_like(G) if args.op == "dequantize" else None})

    def quantize(i, x, st):
        G, b = Gs[i], bufs[i]
        F.check(lib.fs4_nvfp4_quantize(x.data_ptr(), G.shape[0], G.shape[1], G.shape[1], 0,
                                       b["codes"].data_ptr(), b["scales"].data_ptr(), b["sg"].data_ptr(),
                                       flags, b["ws"].data_ptr(), qws_bytes, st.cuda_stream),
                "fs4_nvfp4_quantize")

    def dequantize(i, y, st):
        G, b = Gs[i], bufs[i]
        F.check(lib.fs4_nvfp4_dequantize(b["codes"].data_ptr(), b["scales"].data_ptr(), b["sg"].data_ptr(),
                                         G.shape[0], G.shape[1], y.data_ptr(), G.shape[1], flags,
                                         st.cuda_stream), "fs4_nvfp4_dequantize")

    batched = args.op == "quantize" and not args.per_matrix
    qarr = (F._lib.QuantDesc * len(Gs))()
    for i, (G, b) in enumerate(zip(Gs, bufs)):
        qarr[i] = F._lib.QuantDesc(G.data_ptr(), G.shape[0], G.shape[1], G.shape[1], 0, b["codes"].data_ptr(),
                                   b["scales"].data_ptr(), b["sg"].data_ptr())
    bws_bytes = int(lib.fs4_nvfp4_quantize_batched_workspace_size(len(Gs)))
    bws = torch.zeros(max(bws_bytes, 256), dtype=torch.uint8, device="cuda")

    def quantize_all(st):
        F.check(lib.fs4_nvfp4_quantize_batched(len(Gs), qarr, flags, bws.data_ptr(), bws.numel(),
                                               st.cuda_stream), "fs4_nvfp4_quantize_batched")

    def step():
        if batched:
            quantize_all(stream)
            return
        for i in range(len(Gs)):
            if args.op == "quantize":
                quantize(i, Gs[i], stream)
            else:
                dequantize(i, bufs[i]["y"], stream)

    for i in range(len(Gs)):              # codes for the dequantiser; warms the quantiser
        quantize(i, Gs[i], stream)
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    for b in bufs:
        F.check(F.device_status(b["ws"]), "device status after warm-up")
    F.check(F.device_status(bws), "device status after warm-up")

    call_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(Gs) + 1)] for _ in range(args.steps)]
    for evs in call_ev:
        for e in evs:
            e.record(stream)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler:
        time.sleep(0.3)
        for s in range(args.steps):
            call_ev[s][0].record(stream)
            if batched:
                quantize_all(stream)
                call_ev[s][-1].record(stream)
                continue
            for i in range(len(Gs)):
                if args.op == "quantize":
                    quantize(i, Gs[i], stream)
                else:
                    dequantize(i, bufs[i]["y"], stream)
                call_ev[s][i + 1].record(stream)
        torch.cuda.synchronize()
    if batched:
        F.check(F.device_status(bws), "device status after the timed steps")
    barrier()
    total_ms = ranks_max(call_ev[0][0].elapsed_time(call_ev[-1][-1]))
    ms_step = total_ms / args.steps
    elems = sum(G.numel() for G in Gs)
    value = job_rate(world, elems * QD_BYTES / 1e9, ms_step)

    # roofline of one call (the amax and quantise launches of fs4_nvfp4_quantize, or
    # the one dequantise launch), averaged over every call of the timed steps
    if batched:
        call_ms = [evs[0].elapsed_time(evs[-1]) for evs in call_ev]
        call_bytes = elems * QD_BYTES
    else:
        call_ms = [evs[i].elapsed_time(evs[i + 1]) for evs in call_ev for i in range(len(Gs))]
        call_bytes = elems * QD_BYTES / len(Gs)
    mean_call = statistics.mean(call_ms)
    peaks, peak_src = measured_peaks()
    achieved = call_bytes / (mean_call * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None,
            "kernel": ("fs4_nvfp4_quantize_batched call (quantize_batched_kernel: amax pass, grid "
                       "barrier, quantise pass over every matrix)" if batched
                       else "fs4_nvfp4_quantize call (quantize_fused_kernel: amax pass, grid barrier, quantise pass)"
                       if args.op == "quantize" else "fs4_nvfp4_dequantize call (dequantize_kernel)"),
            "ms_per_launch": mean_call, "peak_source": f"hbm_gbs ({peak_src} MEASURED_PEAKS.json)"}

    # end to end with host buffers: per matrix, copy in, call, copy out, pipelined over a
    # copy-in, a compute and a copy-out stream (each matrix has its own device buffers)
    e2e = None
    if not args.no_e2e:
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        if args.op == "quantize":
            host_in = [G.cpu().pin_memory() for G in Gs]
            dev_in = [torch.empty_like(G) for G in Gs]
            host_out = [(torch.empty(b["codes"].shape, dtype=torch.uint8).pin_memory(),
                         torch.empty(b["scales"].shape, dtype=torch.uint8).pin_memory(),
                         torch.empty(1, dtype=torch.float32).pin_memory()) for b in bufs]
            dev_out = [(b["codes"], b["scales"], b["sg"]) for b in bufs]
        else:
            host_in = [(b["codes"].cpu().pin_memory(), b["scales"].cpu().pin_memory(),
                        b["sg"].cpu().pin_memory()) for b in bufs]
            dev_in = [(b["codes"], b["scales"], b["sg"]) for b in bufs]
            host_out = [torch.empty(G.shape, dtype=torch.float32).pin_memory() for G in Gs]
            dev_out = [b["y"] for b in bufs]
        ev_in = [torch.cuda.Event() for _ in Gs]
        ev_done = [torch.cuda.Event() for _ in Gs]
        ev_out = [torch.cuda.Event() for _ in Gs]
        for e in ev_in + ev_done + ev_out:
            e.record(stream)

        def copy(dst, src):
            if isinstance(dst, tuple):
                for d, h in zip(dst, src):
                    d.copy_(h, non_blocking=True)
            else:
                dst.copy_(src, non_blocking=True)

        def e2e_step():
            for i in range(len(Gs)):
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_done[i])        # the previous step's call read dev_in[i]
                    copy(dev_in[i], host_in[i])
                    ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                stream.wait_event(ev_out[i])           # the previous step's outputs were copied out
                if args.op == "quantize":
                    quantize(i, dev_in[i], stream)
                else:
                    dequantize(i, dev_out[i], stream)
                ev_done[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[i])
                    copy(host_out[i], dev_out[i])
                    ev_out[i].record(s_out)

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e2e_steps = max(2, min(args.steps, 5))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        for _ in range(e2e_steps):
            e2e_step()
        for e in ev_out:
            stream.wait_event(e)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = ranks_max(e0.elapsed_time(e1)) / e2e_steps
        nb_fp32 = elems * 4
        nb_q = sum(b["codes"].numel() + b["scales"].numel() + 4 for b in bufs)
        e2e = {"value": job_rate(world, elems * QD_BYTES / 1e9, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": nb_fp32 if args.op == "quantize" else nb_q,
               "d2h_bytes_per_step": nb_q if args.op == "quantize" else nb_fp32,
               "ms_per_step": e2e_ms,
               "pipeline": "per matrix: copy-in, call and copy-out overlap on three streams"}
    for b in bufs:
        F.check(F.device_status(b["ws"]), "device status after the timed steps")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, desc, cores = oracle_qd_rate(w, args.op, 20.0)
        cpu = {"value": rate, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        line = {
            "metric": QD_METRIC[args.op], "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 <-> nvfp4 (e2m1 x e4m3/16, fp32 tensor scale)", "data": "synthetic",
            "config": {"workload": w.name, "matrices": len(Gs), "op": args.op, "layout": args.layout,
                       "axis": "row (1x16 blocks)", "s_g": "power of two",
                       "parallelism": f"replicas x{world} (independent matrices, no collective)",
                       "l2": ("inputs larger than L2 (%.2f GB of FP32 per step)" % (elems * 4 / 1e9)
                              if elems * 4 > torch.cuda.get_device_properties(local).L2_cache_size
                              else "inputs of %.1f MB fit in L2 (not flushed)" % (elems * 4 / 1e6))},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * (1 if batched else len(Gs)),   # one kernel per call
            "clocks": sampler.summary(),
        }
        print(json.dumps(line), flush=True)


def oracle_momentum_rate(w, budget_s: float):
    """Time the C++ oracle's momentum step (with a previous state) on leading rows of the
    workload's first matrix.  Returns (algorithmic GB/s, seconds, description, cores)."""
    from oracle import cpp_oracle as C
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, generate
    G = generate(w.shapes[0], w.dist, BASE_SEED, "cpu").numpy()
    rows = 16
    while True:
        g = G[:rows]
        _, state = C.momentum_update(g, 0.95, None, 0, 0x5A5A, 1)
        t0 = time.perf_counter()
        C.momentum_update(g, 0.95, state, 0x5A5A, 0xC3C3, 2)
        dt = time.perf_counter() - t0
        if dt >= budget_s / 4 or rows >= G.shape[0]:
            break
        rows = min(G.shape[0], rows * 4)
    cores = C.threads()
    desc = (f"C++ oracle momentum step (exact emulation; OpenMP over rows) of the first {rows} rows "
            f"of a {G.shape[0]}x{G.shape[1]} workload matrix, {dt:.2f} s on {cores} threads")
    return g.size * MO_BYTES / dt / 1e9, dt, desc, cores


def run_momentum_reference(args, w):
    rates, desc, cores = [], "", 1
    for i in range(args.warmup + args.steps):
        rate, dt, desc, cores = oracle_momentum_rate(w, max(2.0, 120.0 / max(1, args.steps + args.warmup)))
        if i >= args.warmup:
            rates.append(rate)
    value = statistics.median(rates)
    total = sum(r * c for r, c in w.shapes) * MO_BYTES
    print(json.dumps({
        "impl": "reference", "metric": MO_METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * total / (value * 1e9), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 values, exact NVFP4 emulation", "data": "synthetic",
        "config": {"workload": w.name, "matrices": len(w.shapes), "op": "momentum"},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def run_momentum(args, w, rank, world, local, barrier, ranks_max):
    """--op momentum: one step = one fs4_momentum_nvfp4 call per matrix of the workload
    (previous state present, updated in place; m_t written in FP32)."""
    import torch
    import nvfp4_precision_optimizer_b200 as F
    from nvfp4_precision_optimizer_b200.workloads import BASE_SEED, matrices

    lib = F._lib.lib()
    Gs = matrices(w, device="cuda", seed=rank_seed(BASE_SEED, rank))
    stream = torch.cuda.current_stream()
    wsz = int(lib.fs4_momentum_workspace_size())
    bufs = []
    for G in Gs:
        R, C = G.shape
        bufs.append({"codes": torch.empty((R, C // 2), dtype=torch.uint8, device="cuda"),
                     "scales": torch.empty((R, C // 16), dtype=torch.uint8, device="cuda"),
                     "sg": torch.empty(1, dtype=torch.float32, device="cuda"),
                     "m": torch.empty_like(G),
                     "ws": torch.zeros(wsz, dtype=torch.uint8, device="cuda")})
    step_no = [0]

    def call(i, g, st, first=False):
        b = bufs[i]
        prev = (None, None, None) if first else (b["codes"].data_ptr(), b["scales"].data_ptr(),
                                                 b["sg"].data_ptr())
        k = step_no[0]
        F.check(lib.fs4_momentum_nvfp4(g.data_ptr(), g.shape[0], g.shape[1], g.shape[1], 0.95,
                                       prev[0], prev[1], prev[2], (0x5A5A + k) & 0xFFFF,
                                       b["codes"].data_ptr(), b["scales"].data_ptr(), b["sg"].data_ptr(),
                                       (0x5A5A + k + 1) & 0xFFFF, 1000 * k + i, b["m"].data_ptr(),
                                       g.shape[1], b["ws"].data_ptr(), wsz, st.cuda_stream),
                "fs4_momentum_nvfp4")

    for i, G in enumerate(Gs):
        call(i, G, stream, first=True)
    step_no[0] += 1
    for _ in range(max(3, args.warmup)):
        for i, G in enumerate(Gs):
            call(i, G, stream)
        step_no[0] += 1
    torch.cuda.synchronize()
    for b in bufs:
        F.check(F.device_status(b["ws"]), "device status after warm-up")
    call_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(Gs) + 1)] for _ in range(args.steps)]
    for evs in call_ev:
        for e in evs:
            e.record(stream)
    barrier()
    torch.cuda.synchronize()
    sampler = ClockSampler(local)
    with sampler:
        time.sleep(0.3)
        for s in range(args.steps):
            call_ev[s][0].record(stream)
            for i, G in enumerate(Gs):
                call(i, G, stream)
                call_ev[s][i + 1].record(stream)
            step_no[0] += 1
        torch.cuda.synchronize()
    barrier()
    total_ms = ranks_max(call_ev[0][0].elapsed_time(call_ev[-1][-1]))
    ms_step = total_ms / args.steps
    elems = sum(G.numel() for G in Gs)
    value = job_rate(world, elems * MO_BYTES / 1e9, ms_step)
    call_ms = [evs[i].elapsed_time(evs[i + 1]) for evs in call_ev for i in range(len(Gs))]
    mean_call = statistics.mean(call_ms)
    peaks, peak_src = measured_peaks()
    achieved = elems * MO_BYTES / len(Gs) / (mean_call * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": None,
            "kernel": "fs4_momentum_nvfp4 call (momentum_pass1_kernel + momentum_pass2_kernel)",
            "ms_per_launch": mean_call, "peak_source": f"hbm_gbs ({peak_src} MEASURED_PEAKS.json)"}

    # end to end: each matrix's gradient copied in from pinned host memory, the step, and
    # m_t copied back (the state stays on the device), pipelined over three streams
    e2e = None
    if not args.no_e2e:
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        host_g = [G.cpu().pin_memory() for G in Gs]
        dev_g = [torch.empty_like(G) for G in Gs]
        host_m = [torch.empty(G.shape, dtype=torch.float32).pin_memory() for G in Gs]
        ev_in = [torch.cuda.Event() for _ in Gs]
        ev_done = [torch.cuda.Event() for _ in Gs]
        ev_out = [torch.cuda.Event() for _ in Gs]
        for e in ev_in + ev_done + ev_out:
            e.record(stream)

        def e2e_step():
            for i in range(len(Gs)):
                with torch.cuda.stream(s_in):
                    s_in.wait_event(ev_done[i])
                    dev_g[i].copy_(host_g[i], non_blocking=True)
                    ev_in[i].record(s_in)
                stream.wait_event(ev_in[i])
                stream.wait_event(ev_out[i])
                call(i, dev_g[i], stream)
                ev_done[i].record(stream)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev_done[i])
                    host_m[i].copy_(bufs[i]["m"], non_blocking=True)
                    ev_out[i].record(s_out)
            step_no[0] += 1

        e2e_step()
        torch.cuda.synchronize()
        barrier()
        e2e_steps = max(2, min(args.steps, 5))
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_event(e0)
        for _ in range(e2e_steps):
            e2e_step()
        for e in ev_out:
            stream.wait_event(e)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = ranks_max(e0.elapsed_time(e1)) / e2e_steps
        e2e = {"value": job_rate(world, elems * MO_BYTES / 1e9, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": elems * 4, "d2h_bytes_per_step": elems * 4, "ms_per_step": e2e_ms,
               "pipeline": "per matrix: gradient copy-in, step and m_t copy-out overlap on three streams"}
    for b in bufs:
        F.check(F.device_status(b["ws"]), "device status after the timed steps")
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, dt, desc, cores = oracle_momentum_rate(w, 20.0)
        cpu = {"value": rate, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps({
            "metric": MO_METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "f32 momentum, nvfp4 state (e2m1 x e4m3/16, SR, adaptive 4/6, H16^r)",
            "data": "synthetic",
            "config": {"workload": w.name, "matrices": len(Gs), "op": "momentum", "beta": 0.95,
                       "state": "previous state present, updated in place; m_t written in FP32",
                       "parallelism": f"replicas x{world} (independent matrices, no collective)",
                       "l2": ("inputs larger than L2 (%.2f GB of FP32 per step)" % (elems * 4 / 1e9)
                              if elems * 4 > torch.cuda.get_device_properties(local).L2_cache_size
                              else "inputs of %.1f MB fit in L2 (not flushed)" % (elems * 4 / 1e6))},
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": args.steps * len(Gs) * 2, "clocks": sampler.summary(),
        }), flush=True)


if __name__ == "__main__":
    main()
