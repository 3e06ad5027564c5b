"""Benchmark: converged sequence-steps x batch per second of parallel Newton evaluation.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl pn|reference]
                    [--workload I] [--mode M] [--all]

A step is one full evaluation (pn_eval: input projection, the device-side
convergence loop of fused iteration kernels, result copy) of one synthetic
workload, by default the tanh RNN D=64, T=16384, B=16 with diagonal
quasi-Newton (tol 1e-5).  The timed region holds exactly K steps between a
barrier + device synchronisation on both sides, timed with CUDA events; for N>1
(launched by torch.distributed.run, one rank per GPU) every rank evaluates its
own copy of the workload (independent problem instances, no collective in the
data path: weak scaling) and the time is the max over ranks.

Also reported, on rank 0: the end-to-end number through pn_eval_host_many
(K batches from pinned host buffers, every batch's host<->device copies inside
the timed region, overlapped with the neighbouring batches' evaluations); the
roofline of the fused iteration kernel (algorithmic bytes per iteration / its
mean time per iteration, CUDA events on the library's stream); and the fp64
oracle timed on this host's cores on a bounded sample of the same workload,
with the oracle's plain sequential loop beside it for context.
``--impl reference`` times that oracle alone as the reference arm.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import pn_inputs as pi  # noqa: E402

METRIC = "converged sequence-steps x batch /sec per mode; % of HBM roofline"
UNIT = "steps*batch/s"
DEFAULT_WORKLOAD = 1
CSRC = os.path.join(ROOT, "newton_evaluation_nonlinear_b200", "csrc")
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="pn", choices=["pn", "reference"])
    ap.add_argument("--workload", type=int, default=DEFAULT_WORKLOAD)
    ap.add_argument("--mode", default=None, help="jacobi|picard|quasi|newton (default: the workload's first)")
    ap.add_argument("--all", action="store_true", help="one line per workload and mode (report runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--window", type=int, default=0,
                    help="time the windowed solve (pn_eval_windowed) with windows of this many steps instead")
    ap.add_argument("--band", type=int, default=-1,
                    help="newton: banded Jacobian with this half-bandwidth (PN_OPT_NEWTON_BAND)")
    ap.add_argument("--damping", type=float, default=1.0, help="damping coefficient lambda in (0, 1]")
    ap.add_argument("--adaptive", type=float, default=-1.0,
                    help="adaptive switching with this stall ratio (>= 0; default off)")
    ap.add_argument("--store", default="f32", choices=["f32", "bf16", "f16"],
                    help="iterate storage while the residual is above --store-until")
    ap.add_argument("--store-until", type=float, default=0.0)
    ap.add_argument("--run-length", type=int, default=0, help="PN_OPT_RUN_LENGTH (0: automatic)")
    ap.add_argument("--host-loop", action="store_true",
                    help="host-driven convergence loop (plain kernel launches, e.g. for ncu) instead of the "
                         "device-side CUDA graph loop")
    return ap.parse_args()


# ----------------------------------------------------------------------------
# algorithmic cost model of one fused iteration launch (per sequence step)
# ----------------------------------------------------------------------------

def alg_bytes_per_step(prob) -> int:
    """Bytes one iteration must move per (b, t): read the step input (u_t, gx_t or c_t), read
    s^(i)_t (s^(i)_{t-1} is the previous step's row), write s^(i+1)_t; float32."""
    rin = 3 if prob.cell == pi.CELL_GRU else 1
    return 4 * (rin * prob.D + 2 * prob.D)


def alg_flops_per_step(prob, mode) -> int:
    R = 3 if prob.cell == pi.CELL_GRU else 1
    f = 2 * R * prob.D * prob.D
    if mode == pi.MODE_NEWTON:
        f += 2 * prob.D * prob.D * (prob.D + 1)   # prefix chain [P|q] <- A [P|q]
    return f


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_sha() -> str:
    """Hash of the device code: the kernel headers and the per-cell kernel units (host code excluded)."""
    h = hashlib.sha256()
    for name in sorted(os.listdir(CSRC)):
        if name.endswith(".cuh") or (name.startswith("pn_k_") and name.endswith(".cu")):
            with open(os.path.join(CSRC, name), "rb") as f:
                h.update(f.read())
    return h.hexdigest()[:16]


def traffic_from_profile(prob, mode):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current source."""
    path = os.path.join(PROFILES, "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(f"{prob.name}:{pi.MODE_NAMES[mode]}")
    if not e or e.get("source_sha") != kernel_source_sha():
        return None
    return float(e["dram_bytes_per_launch"])


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampling (read-only) of the SM clock and clock-event reasons every 20 ms, started
    before the warm-up; samples whose timestamp falls inside [mark_start, mark_end] are the ones
    taken during the timed region."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None
        self.lines = []

    def __enter__(self):
        import subprocess
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.5)   # let it start sampling before the timed region
        except Exception:
            self.proc = None
        return self

    def mark_start(self):
        self.t0 = time.time()

    def mark_end(self):
        self.t1 = time.time()
        time.sleep(0.05)

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        import datetime
        rows = []
        for l in self.lines:
            parts = [p.strip() for p in l.split(",")]
            if len(parts) < 7:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[3:7]))
            except ValueError:
                continue
        inside = [r for r in rows if self.t0 is not None and self.t0 <= r[0] <= (self.t1 or 0)]
        window = inside
        if not window and rows and self.t0 is not None:   # region shorter than the sampling period
            window = sorted(rows, key=lambda r: abs(r[0] - 0.5 * (self.t0 + (self.t1 or self.t0))))[:2]
        reasons = set()
        for r in window:
            for n, v in zip(self.NAMES, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median([r[1] for r in window]) if window else None,
                "sm_max_mhz": window[0][2] if window else None, "reasons": sorted(reasons),
                "samples": len(inside), "nearest_used": bool(window) and not inside}


# ----------------------------------------------------------------------------
# the oracle on the host cores (CPU baseline / reference arm)
# ----------------------------------------------------------------------------

def cpu_sample(prob, mode, b_sample, args=None):
    """The oracle's iteration in the same mode (and variant: band, damping, adaptive switching,
    storage format) on the first b_sample sequences."""
    import oracle
    m = oracle.Model.from_problem(prob)
    x = np.ascontiguousarray(prob.x[:b_sample])
    s0 = np.ascontiguousarray(prob.s0[:b_sample])
    threads = oracle.default_threads(b_sample)
    v = variant(args) if args is not None else {}
    t0 = time.perf_counter()
    if {k: val for k, val in v.items() if k != "run_length"}:
        band = v.get("newton_band", -1)
        omode, oband = (oracle.BANDED, band) if (mode == pi.MODE_NEWTON and 0 <= band < prob.D - 1) else (mode, 0)
        store = {"bf16": oracle.STORE_BF16, "f16": oracle.STORE_F16}.get(v.get("store"), oracle.STORE_F64)
        # the library holds lambda, the stall ratio and store_until in float32
        f32 = lambda a: float(np.float32(a))   # noqa: E731
        _, it, _, _, _, _, _ = m.iterate_ex(omode, x, s0, prob.iters_cap, prob.tol, band=oband,
                                            damping=f32(v.get("damping", 1.0)),
                                            adapt="adaptive_stall" in v, stall=f32(v.get("adaptive_stall", 0.9)),
                                            store=store, store_until=f32(v.get("store_until", 0.0)),
                                            nthreads=threads)
    else:
        _, it, _, _, _ = m.iterate(mode, x, s0, prob.iters_cap, prob.tol, nthreads=threads)
    wall = time.perf_counter() - t0
    return prob.T * b_sample / wall, wall, it, threads


def cpu_sequential(prob, b_sample, threads):
    """The oracle's plain sequential loop s_t = f_t(s_{t-1}) on the first b_sample sequences."""
    import oracle
    m = oracle.Model.from_problem(prob)
    x = np.ascontiguousarray(prob.x[:b_sample])
    s0 = np.ascontiguousarray(prob.s0[:b_sample])
    t0 = time.perf_counter()
    m.sequential(x, s0, nthreads=threads)
    return prob.T * b_sample / (time.perf_counter() - t0)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def cpu_baseline(prob, mode, args=None):
    b_sample = max(1, min(prob.B, os.cpu_count() or 1))
    v, wall, it, threads = cpu_sample(prob, mode, b_sample, args)
    # context: the sequential loop the method replaces, on the same sample and threads, and on one
    # sequence with one thread
    seq = cpu_sequential(prob, b_sample, threads)
    seq1 = cpu_sequential(prob, 1, 1)
    return {"value": v, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"fp64 oracle {pi.MODE_NAMES[mode]} iteration (serial over t, threads over b) on the "
                      f"first {b_sample} of {prob.B} sequences at full T={prob.T}: {it} iterations, "
                      f"{wall:.1f} s wall",
            "sequential": {"value": seq, "unit": UNIT, "cores": threads, "value_1_thread_1_sequence": seq1},
            "cpu_model": cpu_model(), "nproc": os.cpu_count()}


def variant(args) -> dict:
    """Settings beyond the plain iteration (banded Jacobian, damping, adaptive switching, narrow
    iterate storage, run length); empty for the plain one."""
    v = {}
    if getattr(args, "band", -1) >= 0:
        v["newton_band"] = args.band
    if getattr(args, "damping", 1.0) != 1.0:
        v["damping"] = args.damping
    if getattr(args, "adaptive", -1.0) >= 0:
        v["adaptive_stall"] = args.adaptive
    if getattr(args, "store", "f32") != "f32":
        v["store"] = args.store
        v["store_until"] = args.store_until
    if getattr(args, "run_length", 0) > 0:
        v["run_length"] = args.run_length
    return v


L2_BYTES = 126 * 1024 * 1024


def working_set_bytes(prob) -> int:
    """x, the hoisted step inputs and two iterate buffers."""
    rin = 3 if prob.cell == pi.CELL_GRU else 1
    return int(prob.x.nbytes + (rin + 2) * prob.B * prob.T * prob.D * 4)


def flush_l2_needed(prob) -> bool:
    return working_set_bytes(prob) < 2 * L2_BYTES


def workload_config(prob, mode, world, args=None):
    """The workload a line measures; both arms print the same dict for the same workload."""
    v = variant(args) if args is not None else {}
    return {"workload": prob.name + "".join(f"_{k}{val}" for k, val in v.items()), **v, "mode": pi.MODE_NAMES[mode], "cell": pi.CELL_NAMES[prob.cell],
            "D": prob.D, "d_in": prob.d_in, "T": prob.T, "B": prob.B, "tol": prob.tol,
            "max_iters": prob.iters_cap, "parallelism": f"independent instances x{world}",
            "l2": (f"L2 flushed before every timed step (a {2 * L2_BYTES >> 20} MB write outside the events): "
                   f"working set {working_set_bytes(prob) / 1e6:.1f} MB"
                   if flush_l2_needed(prob) else
                   f"inputs larger than L2 (x, step inputs, two iterate buffers: "
                   f"{working_set_bytes(prob) / 1e6:.0f} MB)")}


def reference_arm(args, prob, mode, rank, world):
    if rank != 0:
        return
    b_sample = max(1, min(prob.B, os.cpu_count() or 1))
    for _ in range(args.warmup):
        cpu_sample(prob, mode, b_sample, args)
    walls, its = [], []
    for _ in range(args.steps):
        _, wall, it, threads = cpu_sample(prob, mode, b_sample, args)
        walls.append(wall)
        its.append(it)
    tot = sum(walls)
    value = prob.T * b_sample * args.steps / tot
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": workload_config(prob, mode, world, args),
            "run": {"iters": its[-1], "sample_sequences": b_sample, "loop": "host (serial over t)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": f"fp64 oracle {pi.MODE_NAMES[mode]} iteration on the first {b_sample} "
                                       f"of {prob.B} sequences at full T={prob.T}, {its[-1]} iterations per step"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# multi-rank aggregation (independent instances, one per rank: weak scaling)
# ----------------------------------------------------------------------------

def max_over_ranks(ms: float, dist, device) -> float:
    """The slowest rank's time for the same timed region; every rank calls this at the same point
    (a collective). Without a process group it is the local time."""
    if dist is None:
        return ms
    import torch
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed over the slowest rank's time."""
    return units_per_rank * world / (ms_max / 1e3)


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------

def bench_pn(args, prob, mode, rank, world, local_rank, dist, with_extras=True):
    import torch

    import newton_evaluation_nonlinear_b200 as pn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    solver = pn.Solver.from_problem(prob, stream=stream, device=dev)
    if args.host_loop:
        solver.set_option(pn.PN_OPT_DEVICE_LOOP, 0)
    if args.band >= 0:
        solver.set_option(pn.PN_OPT_NEWTON_BAND, args.band)
    if args.run_length > 0:
        solver.set_option(pn.PN_OPT_RUN_LENGTH, args.run_length)
    if args.damping != 1.0:
        solver.set_damping(args.damping)
    if args.adaptive >= 0:
        solver.set_adaptive(args.adaptive)
    if args.store != "f32":
        solver.set_storage({"bf16": pn.PN_STORE_BF16, "f16": pn.PN_STORE_F16}[args.store], args.store_until)
    x = torch.from_numpy(prob.x).to(dev)
    s0 = torch.from_numpy(prob.s0).to(dev)
    states = torch.empty((prob.B, prob.T, prob.D), device=dev, dtype=torch.float32)
    mi, tol = prob.iters_cap, prob.tol

    for _ in range(max(3, args.warmup)):
        _, iters, resid, st = solver.eval(x, s0, mode, mi, tol, states)
    torch.cuda.synchronize(dev)
    solver.reset_stats()

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush = flush_l2_needed(prob)
    scrub = torch.empty(2 * L2_BYTES // 4, device=dev, dtype=torch.float32) if flush else None
    with ClockSampler(local_rank) as clk:
        barrier()
        clk.mark_start()
        if flush:
            # a working set below twice the L2: every step starts from a flushed L2, timed step by step
            t_ms = 0.0
            for _ in range(args.steps):
                scrub.fill_(1.0)
                e0.record(stream)
                _, iters, resid, st = solver.eval(x, s0, mode, mi, tol, states)
                e1.record(stream)
                e1.synchronize()
                t_ms += e0.elapsed_time(e1)
        else:
            e0.record(stream)
            for _ in range(args.steps):
                _, iters, resid, st = solver.eval(x, s0, mode, mi, tol, states)
            e1.record(stream)
        barrier()
        clk.mark_end()
    ms = max_over_ranks(t_ms if flush else e0.elapsed_time(e1), dist, dev)
    del scrub
    stats = solver.stats()
    value = job_throughput(prob.T * prob.B * args.steps, world, ms)
    loop_kind = pn.pn_dim(solver.h, 5 + mode)
    looping = loop_kind >= 1 and not args.host_loop
    single = loop_kind == 2 and not args.host_loop
    # projection (not for the Euler cell), init, the iteration kernel(s), result copy; or the one
    # single-CTA launch of the small solve
    launches_per_step = 1 if single else (1 if looping else iters + 1) + 2 + (0 if prob.cell == pi.CELL_EULER else 1)

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": workload_config(prob, mode, world, args),
            "run": {"iters": iters, "final_resid": resid, "status": st,
                    "loop": "host" if args.host_loop else (
                        "device (one single-CTA launch: projection, iterations, stop rule, result copy)" if single
                        else "device (one launch iterating to the stop rule)" if looping
                        else "device (CUDA graph WHILE node)")},
            "clocks": clk.summary(), "gpu_launches": launches_per_step * args.steps}
    if not with_extras:
        solver.close()
        return line

    # roofline of the fused iteration kernel: CUDA events around back-to-back launches
    n_l = max(10, 3 * (iters + 1))
    kms = solver.time_iterations(mode, n_l)
    in_eval_us = stats["iteration_ns"] / max(1, stats["iteration_launches"]) / 1e3
    hbm, src = peaks()
    bytes_launch = alg_bytes_per_step(prob) * prob.B * prob.T
    achieved = bytes_launch / (kms / 1e3) / 1e9
    traffic = traffic_from_profile(prob, mode)
    line["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                        "frac": achieved / hbm, "traffic": traffic, "peak_source": src,
                        "kernel": "fused iteration (cell + Jacobian + chunked scan + residual)"
                                  + (", one launch looping over iterations: figures per iteration" if looping else ""),
                        "alg_bytes_per_launch": bytes_launch, "launch_ms": kms,
                        "in_eval_us_per_iteration": in_eval_us,
                        "fp32_tflops": alg_flops_per_step(prob, mode) * prob.B * prob.T / (kms / 1e3) / 1e12}

    # end to end through the pipelined host-buffer entry point: every step copies its batch's
    # inputs in from pinned host memory and its states out, inside the timed region; the copies
    # of neighbouring steps overlap each step's evaluation
    hx = torch.from_numpy(prob.x).pin_memory()
    hs0 = torch.from_numpy(prob.s0).pin_memory()
    hst = torch.empty((prob.B, prob.T, prob.D), dtype=torch.float32).pin_memory()
    hxn, hs0n, hstn = hx.numpy(), hs0.numpy(), hst.numpy()
    solver.eval_host_many([hxn] * 2, [hs0n] * 2, mode, mi, tol, [hstn] * 2)
    barrier()
    e0.record(stream)
    solver.eval_host_many([hxn] * args.steps, [hs0n] * args.steps, mode, mi, tol, [hstn] * args.steps)
    e1.record(stream)
    barrier()
    ems = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    line["e2e"] = {"value": job_throughput(prob.T * prob.B * args.steps, world, ems), "unit": UNIT, "h2d_bytes_per_step": int(prob.x.nbytes + prob.s0.nbytes),
                   "d2h_bytes_per_step": int(prob.B * prob.T * prob.D * 4), "ms_per_step": ems / args.steps}
    solver.close()
    return line


def bench_windowed(args, prob, mode, rank, world, local_rank, dist):
    """The same metric for the windowed solve: each step solves the whole sequence window by
    window (windows of args.window steps, the ragged last one by a second handle)."""
    import torch

    import newton_evaluation_nonlinear_b200 as pn
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    W = min(int(args.window), prob.T)
    rem = prob.T % W
    win = pn.Solver(prob.cell, prob.D, prob.d_in, W, prob.B, prob.params, prob.eps, stream=stream, device=dev)
    tail = (pn.Solver(prob.cell, prob.D, prob.d_in, rem, prob.B, prob.params, prob.eps, stream=stream, device=dev)
            if rem else None)
    x = torch.from_numpy(prob.x).to(dev)
    s0 = torch.from_numpy(prob.s0).to(dev)
    states = torch.empty((prob.B, prob.T, prob.D), device=dev, dtype=torch.float32)
    mi, tol = min(prob.iters_cap, W), prob.tol
    for _ in range(max(3, args.warmup)):
        _, iters, resid, st, wit = win.eval_windowed(x, s0, mode, mi, tol, tail=tail, states=states)
    torch.cuda.synchronize(dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        clk.mark_start()
        e0.record(stream)
        for _ in range(args.steps):
            _, iters, resid, st, wit = win.eval_windowed(x, s0, mode, mi, tol, tail=tail, states=states)
        e1.record(stream)
        barrier()
        clk.mark_end()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    nwin = len(wit)
    loop_kind = pn.pn_dim(win.h, 5 + mode)
    per_window = [1 if loop_kind == 2 else (1 if loop_kind == 1 else int(n) + 1) + 2 +
                  (0 if prob.cell == pi.CELL_EULER else 1) for n in wit]
    line = {"metric": METRIC, "value": job_throughput(prob.T * prob.B * args.steps, world, ms), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": prob.name + f"_window{W}", "mode": pi.MODE_NAMES[mode],
                       "cell": pi.CELL_NAMES[prob.cell], "D": prob.D, "d_in": prob.d_in, "T": prob.T,
                       "B": prob.B, "tol": prob.tol, "max_iters_per_window": mi, "window": W,
                       "windows": nwin, "iters": iters, "window_iters": [int(n) for n in wit],
                       "final_resid": resid, "status": st,
                       "parallelism": f"independent instances x{world}",
                       "l2": (f"inputs larger than L2 (the whole sequence, {working_set_bytes(prob) / 1e6:.0f} MB "
                              "of x, step inputs and iterates, is read and written once per step)"
                              if not flush_l2_needed(prob) else
                              f"L2 not flushed: working set {working_set_bytes(prob) / 1e6:.1f} MB")},
            "clocks": clk.summary(), "gpu_launches": sum(per_window) * args.steps}
    win.close()
    if tail is not None:
        tail.close()
    return line


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime

        import torch
        import torch.distributed as tdist
        backend = "nccl" if args.impl == "pn" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local_rank)
        tdist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        dist = tdist
    try:
        jobs = []
        if args.all:
            for idx in range(5):
                for m in pi.WORKLOAD_MODES[idx]:
                    jobs.append((idx, m))
        else:
            m = pi.MODE_BY_NAME[args.mode] if args.mode else pi.WORKLOAD_MODES[args.workload][0]
            jobs.append((args.workload, m))
        for idx, mode in jobs:
            prob = pi.benchmark_workload(idx)
            if args.impl == "reference":
                reference_arm(args, prob, mode, rank, world)
                continue
            if args.window > 0:
                line = bench_windowed(args, prob, mode, rank, world, local_rank, dist)
            else:
                line = bench_pn(args, prob, mode, rank, world, local_rank, dist)
            if rank == 0:
                if world == 1 and not args.no_cpu_baseline and args.window <= 0:
                    line["cpu_baseline"] = cpu_baseline(prob, mode, args)
                print(json.dumps(line), flush=True)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
