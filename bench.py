#!/usr/bin/env python
"""Benchmark of the fused diagonal-GMM EM iteration (N=1M, d=128, K=256, fp32).

A step is one EM iteration over the workload: the fused E-step + statistics
(gmm_em_step) and the M-step finalise (gmm_finalize), through the C ABI, with
X resident in HBM.  X is 512 MB (larger than the 126 MB L2), so every step
streams it from HBM.  With --gpus N (torchrun, one rank per GPU) every rank
holds its own 1M-point shard of an N x 1M-point data set (weak scaling); the
statistics are summed across ranks with one NCCL all-reduce per iteration and
every rank runs the same finalise.

Prints one JSON line (rank 0).  `--impl reference` times the float64 CPU
oracle on a bounded sample instead (the reference arm).
"""
from __future__ import annotations

import argparse
import hashlib
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

from synth import WORKLOADS, gmm_data, gmm_init  # noqa: E402

METRIC = "EM iters/s and N·K·d/s (% roofline) for diag GMM N=1M d=128 K=256"
TF32_OVER_BF16 = 1.1 / 2.25   # nominal dense ratio (profiling recipe)


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", type=int, default=2)
    p.add_argument("--flags", type=int, default=0, help="GMM_FLAG_* (testing)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--points", type=int, default=0,
                   help="override N per GPU (small cases for profiling only)")
    p.add_argument("--cpu-sample", type=int, default=16384,
                   help="points per step of the reference arm (at least 1024 per thread)")
    p.add_argument("--cpu-budget", type=float, default=30.0,
                   help="seconds of oracle work for the cpu_baseline leg")
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, \
        "fallback"


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 20 ms over the timed
    region: the sampler is started, and entry waits until it has produced its
    first line (up to 3 s); only the lines written after that count, so a
    region of a few tens of milliseconds still gets samples of its own."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.out = None
        self.skip = 0

    def __enter__(self):
        try:
            self.out = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 3.0 and self._lines() == 0:
                time.sleep(0.01)
            self.skip = self._lines()
        except (FileNotFoundError, OSError):
            self.proc = None
        return self

    def _lines(self):
        self.out.flush()
        with open(self.out.name) as f:
            return sum(1 for _ in f)

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.05)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or self.out is None:
            return None
        self.out.flush()
        rows = []
        with open(self.out.name) as f:
            for i, ln in enumerate(f):
                parts = [x.strip() for x in ln.split(",")]
                if i >= self.skip and len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def pipelined_e2e(Xh, Xbuf, n_steps, compute):
    """Time n_steps end-to-end steps.  Every step copies its X from pinned host
    memory (Xh) and runs compute(X_device), which copies the step's other
    inputs in and its results back on the current stream.  The X copies go on
    a second stream into two device buffers, so that step s + 1's copy runs
    while step s computes.  Returns the milliseconds between an event
    recorded before the first copy and one after the last step's results."""
    import torch
    cur = torch.cuda.current_stream()
    cs = torch.cuda.Stream()
    bufs = [Xbuf, torch.empty_like(Xbuf)]
    copied = [torch.cuda.Event(), torch.cuda.Event()]
    used = [torch.cuda.Event(), torch.cuda.Event()]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def copy_into(k, s):
        with torch.cuda.stream(cs):
            if s >= 2:
                cs.wait_event(used[k])   # step s - 2 is done with this buffer
            bufs[k].copy_(Xh, non_blocking=True)
            copied[k].record(cs)

    a.record(cur)
    cs.wait_event(a)
    copy_into(0, 0)
    for s in range(n_steps):
        k = s % 2
        if s + 1 < n_steps:
            copy_into((s + 1) % 2, s + 1)
        cur.wait_event(copied[k])
        compute(bufs[k])
        used[k].record(cur)
    b.record(cur)
    torch.cuda.synchronize()
    return a.elapsed_time(b)


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "means_clustering_gmm_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel_key: str, src_hash: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current source of the kernel; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    e = t.get(kernel_key)
    if e and e.get("source_hash") == src_hash:
        return e.get("dram_bytes_per_launch")
    return None


def cpu_sample_points(w, X, mu, var, lw, budget_s: float) -> tuple[int, float]:
    """Points of the workload the oracle can run one EM iteration on within
    about budget_s seconds (calibrated on a prefix that gives every OpenMP
    thread two row blocks); the whole workload when it fits."""
    import oracle
    oracle.build()
    n0 = min(2048 * oracle.num_threads(), X.shape[0])   # row blocks for every thread
    t0 = time.perf_counter()
    oracle.gmm_em_iteration(X[:n0], mu, var, lw)
    t = time.perf_counter() - t0
    n = int(n0 * budget_s / max(t, 1e-6))
    return max(n0, min(X.shape[0], n)), t


def cpu_baseline(w, X, mu, var, lw, budget_s: float):
    """The oracle as it stands (float64, OpenMP on every host core), one EM
    iteration on the whole workload when that takes at most about budget_s,
    else on a prefix scaled to the workload."""
    import oracle
    n, _ = cpu_sample_points(w, X, mu, var, lw, budget_s)
    t0 = time.perf_counter()
    oracle.gmm_em_iteration(X[:n], mu, var, lw)
    t = time.perf_counter() - t0
    per_iter_full = t * (X.shape[0] / n)
    what = (f"one float64 EM iteration (E-step, two-pass M-step) on all {n} points"
            if n == X.shape[0] else
            f"one float64 EM iteration (E-step, two-pass M-step) on the first {n} of "
            f"{X.shape[0]} points, scaled by N/{n}")
    return {"value": 1.0 / per_iter_full, "unit": "EM iters/s", "cores": oracle.num_threads(),
            "kind": "oracle", "sample": f"{what} (d={w.d}, K={w.K}), {t:.2f} s"}


def gmm_config(w, N: int, world: int) -> dict:
    """The workload description both arms print (same keys, same values)."""
    x_bytes = N * w.d * (4 if w.dtype == "f32" else 2)
    return {"workload": w.name, "N_per_gpu": N, "d": w.d, "K": w.K, "input_dtype": w.dtype,
            "parallelism": f"dp{world}",
            "l2": "inputs larger than L2 (X = %d MB per GPU)" % (x_bytes >> 20)}


def run_reference(args):
    """Reference arm: the float64 oracle as it stands, on the host cores.  Each
    step is one EM iteration on a bounded prefix of the workload (at least
    1024 points per OpenMP thread, so every thread has row blocks); `value` is
    scaled to the whole workload, `ms_per_step` is the measured time of one
    such step."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = WORKLOADS[args.workload]
    if w.kind != "gmm":
        print(json.dumps({"impl": "reference", "unavailable":
                          "the reference arm times the GMM workloads only"}), flush=True)
        return 0
    N = args.points or w.N
    threads = oracle.num_threads()
    n = min(N, max(args.cpu_sample, 1024 * threads))
    X, *_ = gmm_data(w, N=max(n, w.K))
    mu, var, lw = gmm_init(w, X)
    X = X[:n]
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        it = oracle.gmm_em_iteration(X, mu, var, lw)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
        mu, var, lw = it["means"], it["vars"], it["logw"]
    step_s = statistics.median(times)
    value = 1.0 / (step_s * (N / n))
    cb = {"value": value, "unit": "EM iters/s", "cores": threads, "kind": "oracle",
          "sample": f"each step: one float64 EM iteration (E-step, two-pass M-step) on the "
                    f"first {n} of {N} points (d={w.d}, K={w.K}); value scaled by N/{n}"}
    print(json.dumps({
        "impl": "reference", "metric": gmm_metric(w), "value": value, "unit": "EM iters/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_s * 1e3,
        "ms_per_step_p95": float(np.percentile(np.array(times) * 1e3, 95)),
        "sample_points": n, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": gmm_config(w, N, world),
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "EM iters/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)
    return 0


def gmm_metric(w) -> str:
    return METRIC if w.number == 2 else METRIC.replace("N=1M d=128 K=256", w.name)


KMEANS_METRIC = "k-means Lloyd iters/s (B problems x N points, one iteration = assign + update)"


def run_kmeans(args):
    """The k-means workload (a secondary measurement): one step = one Lloyd
    iteration of kmeans_step over all B problems; the centroids evolve."""
    import torch
    import torch.distributed as dist

    import means_clustering_gmm_b200 as gmm
    from means_clustering_gmm_b200 import _lib
    from synth import kmeans_data, kmeans_init

    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    rank = int(os.environ.get("RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    lib = _lib.load()
    w = WORKLOADS[args.workload]
    N = args.points or w.N
    X = kmeans_data(w, N=N)
    C0 = kmeans_init(w, X)
    B, _, d = X.shape
    K = w.K
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[w.dtype]
    Xd = torch.from_numpy(X).to(tdt).to(dev)
    Ca = torch.from_numpy(C0).to(dev)
    Cb = torch.empty_like(Ca)
    ids = torch.empty((B, N), dtype=torch.int32, device=dev)
    counts = torch.empty((B, K), dtype=torch.int32, device=dev)
    inertia = torch.empty(B, dtype=torch.float64, device=dev)
    ws = gmm.Workspace.for_kmeans(B, N, d, K, device=dev)
    bufs = [Ca, Cb]

    def step(i):
        gmm.kmeans_step(Xd, bufs[i % 2], ws, ids=ids, new_centroids=bufs[(i + 1) % 2],
                        counts=counts, inertia=inertia, flags=args.flags)

    for i in range(args.warmup):
        step(i)
    assert gmm.gmm_last_error(ws) == 0, "device error during warm-up"
    ev_k = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for a, b in ev_k:
        a.record()
        b.record()
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    for e in ev_s:
        e.record()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = lib.gmm_kernel_launch_count()
    with ClockSampler(local) as clk:
        ev_s[0].record()
        for i in range(args.steps):
            lib.gmm_set_kernel_timer(ev_k[i][0].cuda_event, ev_k[i][1].cuda_event)
            step(args.warmup + i)
            ev_s[i + 1].record()
        torch.cuda.synchronize()
    lib.gmm_set_kernel_timer(None, None)
    launches = lib.gmm_kernel_launch_count() - launches0
    elapsed = ev_s[0].elapsed_time(ev_s[-1])
    step_ms = [ev_s[i].elapsed_time(ev_s[i + 1]) for i in range(args.steps)]
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_k)
    stats_ms = [statistics.median(step_ms), float(np.percentile(step_ms, 95))]
    if world > 1:
        t = torch.tensor([elapsed, kern_ms, *stats_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed, kern_ms = float(t[0]), float(t[1])
        stats_ms = [float(x) for x in t[2:]]
    assert gmm.gmm_last_error(ws) == 0, "device error during the timed steps"
    value = world * args.steps / (elapsed / 1e3)
    peaks, peak_src = load_peaks()
    tc = d in (64, 128) and not (args.flags & 2)
    flops = 2.0 * B * N * K * d
    achieved = flops / (kern_ms * 1e-3) / 1e12
    peak = peaks["bf16_tflops"]
    # DRAM bytes per launch at the full workload, from the committed capture
    traffic = (traffic_for("km_tc_assign_kernel", source_hash("kmeans_tc.cu", "tc_ptx.cuh"))
               if tc and not args.points else None)
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": "km_tc_assign_kernel" if tc else "km_simt_assign_kernel",
                "kernel_ms": kern_ms, "flops_per_launch": flops,
                # x_hi c_hi + x_hi c_lo (+ x_lo c_hi for fp32 X), each 2d per pair
                "issued_mma_flops_per_launch": ((3 if w.dtype == "f32" else 2) * flops
                                                if tc else None),
                "peak_source": f"bf16 burst (fp16 runs at the same rate), {peak_src}"}
    e2e = None
    if not args.no_e2e:
        Xh = torch.from_numpy(X).to(tdt).pin_memory()
        Ch = torch.from_numpy(C0).pin_memory()
        ih = torch.empty(B, dtype=torch.float64).pin_memory()
        Xe = torch.empty_like(Xd)

        def e2e_compute(Xb):
            Ca.copy_(Ch, non_blocking=True)
            gmm.kmeans_step(Xb, Ca, ws, ids=ids, new_centroids=Cb, counts=counts,
                            inertia=inertia, flags=args.flags)
            ih.copy_(inertia, non_blocking=True)

        pipelined_e2e(Xh, Xe, 2, e2e_compute)   # untimed warm-up
        e_steps = max(3, min(args.steps, 5))
        e_ms = pipelined_e2e(Xh, Xe, e_steps, e2e_compute)
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t[0])
        e2e = {"value": world * e_steps / (e_ms / 1e3), "unit": "Lloyd iters/s",
               "h2d_bytes_per_step": Xh.numel() * Xh.element_size() + Ch.numel() * 4,
               "d2h_bytes_per_step": B * 8}
    cb = None
    if not args.no_cpu_baseline and world == 1:
        import oracle
        oracle.build()
        # calibrate on 4096 points, then time whole problems: all B when one
        # full iteration fits the budget, else as many as do (scaled by B/b)
        n = min(N, 4096)
        t0 = time.perf_counter()
        oracle.kmeans_step(X[:1, :n], C0[:1])
        per_point = (time.perf_counter() - t0) / n
        b = max(1, min(B, int(args.cpu_budget / max(per_point * N, 1e-9))))
        t0 = time.perf_counter()
        oracle.kmeans_step(X[:b], C0[:b])
        t = time.perf_counter() - t0
        what = (f"one float64 Lloyd iteration on all {B} problems" if b == B else
                f"one float64 Lloyd iteration on {b} of {B} problems, scaled by {B}/{b}")
        cb = {"value": 1.0 / (t * B / b), "unit": "Lloyd iters/s",
              "cores": oracle.num_threads(), "kind": "oracle",
              "sample": f"{what} (N={N}, K={K}, d={d}), {t:.2f} s"}
    out = {
        "metric": KMEANS_METRIC, "value": value, "unit": "Lloyd iters/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed / args.steps,
        "ms_per_step_median": stats_ms[0], "ms_per_step_p95": stats_ms[1],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name, "B": B, "N": N, "d": d, "K": K, "input_dtype": w.dtype,
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs larger than L2 (X = {Xd.numel() * Xd.element_size() >> 20} MB)",
                   "path": "tcgen05-assign" if tc else "simt-assign"},
        "roofline": roofline, "cpu_baseline": cb, "e2e": e2e, "gpu_launches": int(launches),
        "clocks": clk.summary(),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if WORKLOADS[args.workload].kind == "kmeans":
        return run_kmeans(args)

    import torch
    import torch.distributed as dist

    import means_clustering_gmm_b200 as gmm
    from means_clustering_gmm_b200 import _lib, sharded

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    lib = _lib.load()

    w = WORKLOADS[args.workload]
    assert w.kind == "gmm", "bench times the GMM EM iteration"
    if args.points:
        import dataclasses
        w = dataclasses.replace(w, N=args.points)
    X, *_ = gmm_data(w, shard=rank)
    if rank == 0:
        mu, var, lw = gmm_init(w, X)
    else:
        mu = np.empty((w.K, w.d), np.float32)
        var = np.empty((w.K, w.d), np.float32)
        lw = np.empty(w.K, np.float32)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[w.dtype]
    Xd = torch.from_numpy(X).to(tdt).to(dev)
    m0 = torch.from_numpy(mu).to(dev)
    v0 = torch.from_numpy(var).to(dev)
    l0 = torch.from_numpy(lw).to(dev)
    if world > 1:
        for t in (m0, v0, l0):
            dist.broadcast(t, 0)
    N = X.shape[0]
    N_global = N * world
    m, v, lw_d = m0.clone(), v0.clone(), l0.clone()
    ws = gmm.Workspace.for_gmm(N, w.d, w.K, tdt, device=dev)
    stats = torch.empty(w.K * (1 + 2 * w.d), dtype=torch.float64, device=dev)
    tot = torch.empty(1, dtype=torch.float64, device=dev)

    def step():
        sharded.em_iteration(Xd, m, v, lw_d, ws, N_global, stats, tot, flags=args.flags)

    for _ in range(args.warmup):
        step()
    assert gmm.gmm_last_error(ws) == 0, "device error during warm-up"
    ev_s = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    for e in ev_s:   # torch creates the CUDA event on first record
        e.record()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = lib.gmm_kernel_launch_count()
    # the library brackets its dominant kernel(s) with events of its own on
    # its stream, once per point chunk of a step
    with ClockSampler(local) as clk, gmm.KernelTimer() as ktimer:
        ev_s[0].record()
        for i in range(args.steps):
            step()
            ev_s[i + 1].record()
        torch.cuda.synchronize()
    launches = lib.gmm_kernel_launch_count() - launches0
    if world > 1:
        dist.barrier()
    elapsed = ev_s[0].elapsed_time(ev_s[-1])
    step_ms = [ev_s[i].elapsed_time(ev_s[i + 1]) for i in range(args.steps)]
    regions = len(ktimer.ms) // args.steps
    assert regions >= 1 and regions * args.steps == len(ktimer.ms), "kernel regions per step"
    kern_list = [sum(ktimer.ms[i * regions:(i + 1) * regions]) for i in range(args.steps)]
    kern_ms = statistics.mean(kern_list)
    stats_ms = [statistics.median(step_ms), float(np.percentile(step_ms, 95)),
                statistics.median(kern_list), float(np.percentile(kern_list, 95))]
    if world > 1:
        t = torch.tensor([elapsed, kern_ms, *stats_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        elapsed, kern_ms = float(t[0]), float(t[1])
        stats_ms = [float(x) for x in t[2:]]
    assert gmm.gmm_last_error(ws) == 0, "device error during the timed steps"

    ms_per_step = elapsed / args.steps
    value = world * args.steps / (elapsed / 1e3)   # 1M-point EM iterations per second
    nkd = N * w.K * w.d
    path = lib_path_name(lib, N, w, args.flags)

    # e2e: host X (pinned) and host parameters copied in, results read back, every step
    e2e = None
    if not args.no_e2e:
        Xh = torch.from_numpy(X).to(tdt).pin_memory()
        mh, vh, lh = (t.cpu().pin_memory() for t in (m0, v0, l0))
        mo, vo, lo = (torch.empty_like(t).pin_memory() for t in (mh, vh, lh))
        toth = torch.empty(1, dtype=torch.float64).pin_memory()
        Xe = torch.empty_like(Xd)

        def e2e_compute(Xb):
            m.copy_(mh, non_blocking=True)
            v.copy_(vh, non_blocking=True)
            lw_d.copy_(lh, non_blocking=True)
            sharded.em_iteration(Xb, m, v, lw_d, ws, N_global, stats, tot, flags=args.flags)
            mo.copy_(m, non_blocking=True)
            vo.copy_(v, non_blocking=True)
            lo.copy_(lw_d, non_blocking=True)
            toth.copy_(tot, non_blocking=True)

        pipelined_e2e(Xh, Xe, 2, e2e_compute)   # untimed warm-up
        if world > 1:
            dist.barrier()
        e_steps = max(3, min(args.steps, 5))
        e_ms = pipelined_e2e(Xh, Xe, e_steps, e2e_compute)
        if world > 1:
            t = torch.tensor([e_ms], dtype=torch.float64, device=dev)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            e_ms = float(t[0])
        h2d = Xh.numel() * Xh.element_size() + sum(t.numel() * 4 for t in (mh, vh, lh))
        d2h = sum(t.numel() * 4 for t in (mo, vo, lo)) + 8
        e2e = {"value": world * e_steps / (e_ms / 1e3), "unit": "EM iters/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    peaks, peak_src = load_peaks()
    tc = path.startswith("tcgen05")
    mma_dtype = "f16" if tc else "f32"
    peak_bf16 = peaks["bf16_tflops"]
    # The tensor-core kernels issue tcgen05.mma kind::f16 (split fp16
    # products), so the tensor peak is the measured bf16 burst figure (f16
    # runs at the same rate).  The TF32 figure (the data dtype's own tensor
    # kind for fp32 inputs, bf16 x 1.1/2.25) is reported beside it, labelled.
    peak = peak_bf16
    achieved = 6.0 * nkd / (kern_ms / 1e3) / 1e12
    kernel_key, kernel_src = KERNEL_SOURCES[path]
    per_pair = issued_mma_flops_per_pair(path, w.dtype, w.d, w.K)
    issued = per_pair * N * w.K if per_pair else None
    # (per launch at the full workload: not for a --points prefix)
    traffic = None if args.points else traffic_for(kernel_key, source_hash(*kernel_src))
    sweeps = 2 if path.endswith("two-sweep") else 1
    x_bytes = N * w.d * (4 if w.dtype == "f32" else 2)
    tensor_us = 6.0 * nkd / (peak * 1e12) * 1e6
    hbm_us = sweeps * x_bytes / (peaks["hbm_gbs"] * 1e9) * 1e6
    if tensor_us >= hbm_us:
        bound, r_ach, r_peak, r_unit = "tensor", achieved, peak, "TFLOP/s"
    else:   # the X stream binds: bytes per launch over the measured copy bandwidth
        bound, r_unit = "hbm", "GB/s"
        r_ach = sweeps * x_bytes / (kern_ms / 1e3) / 1e9
        r_peak = peaks["hbm_gbs"]
    roofline = {"bound": bound,
                "achieved": r_ach, "peak": r_peak, "unit": r_unit,
                "frac": r_ach / r_peak, "traffic": traffic,
                "kernel": kernel_key, "kernel_ms": kern_ms,
                "kernel_ms_median": stats_ms[2], "kernel_ms_p95": stats_ms[3],
                "kernel_regions_per_step": regions,
                "flops_per_launch": 6.0 * nkd, "bytes_per_launch": sweeps * x_bytes,
                "tensor_tflops": achieved,
                "flops_8nkd_per_launch": 8.0 * nkd,
                "issued_mma_flops_per_launch": issued,
                "issued_mma_tflops": (issued / (kern_ms / 1e3) / 1e12) if issued else None,
                "peak_source": (f"bf16/f16 dense burst (the tcgen05 kind::f16 the kernels issue), "
                                f"{peak_src}") if bound == "tensor"
                               else f"hbm copy bandwidth, {peak_src}",
                "frac_vs_tf32_literal": (achieved / (peak_bf16 * TF32_OVER_BF16)
                                         if w.dtype == "f32" else None),
                "bound_us": {"tensor": tensor_us, "hbm": hbm_us, "sweeps": sweeps},
                "step_frac": max(tensor_us, hbm_us) / (ms_per_step * 1e3)}
    cb = None
    if not args.no_cpu_baseline and world == 1:
        cb = cpu_baseline(w, X, mu, var, lw, args.cpu_budget)
    clocks = clk.summary()
    out = {
        "metric": gmm_metric(w),
        "value": value, "unit": "EM iters/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "ms_per_step_median": stats_ms[0], "ms_per_step_p95": stats_ms[1],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": mma_dtype, "data": "synthetic",
        "config": gmm_config(w, N, world),
        "path": path,
        "point_chunk": gmm.point_chunk(N, w.d, w.K, tdt, args.flags),
        "workspace_bytes": ws.nbytes,
        "nkd_per_s": world * nkd * args.steps / (elapsed / 1e3),
        "roofline": roofline,
        "cpu_baseline": cb,
        "e2e": e2e,
        "gpu_launches": int(launches),
        "clocks": clocks,
    }
    print(json.dumps(out), flush=True)
    return 0


# dominant kernel of each path: (name in the roofline object, its source files)
KERNEL_SOURCES = {
    "simt-two-sweep": ("gmm_simt_lse_kernel+gmm_simt_stats_kernel", ("gmm_simt.cu",)),
    "tcgen05-single-sweep": ("gmm_tc_fused_kernel", ("gmm_tc.cu", "tc_ptx.cuh")),
    "tcgen05-single-sweep-cluster": ("gmm_tc_cluster_kernel",
                                     ("gmm_tc.cu", "gmm_tc_cluster.cuh", "tc_ptx.cuh")),
    "tcgen05-two-sweep": ("gmm_tc_fused_kernel<kLse>+gmm_tc_stats_kernel",
                          ("gmm_tc.cu", "gmm_tc_stats.cuh", "tc_ptx.cuh")),
    "tcgen05-single-sweep-smallk": ("gmm_tc_smallk_kernel",
                                    ("gmm_tc.cu", "gmm_tc_smallk.cuh", "tc_ptx.cuh")),
}


def issued_mma_flops_per_pair(path: str, dtype: str, d: int, K: int):
    """FLOPs the tensor-core kernels issue per (point, component) pair, from
    their MMA programs (split fp16 pieces; the metric counts 6d and the dense
    contractions are 8d): None for the paths not listed.
      E-step: 6 products of depth d for fp32 X (x_lo is zero for 16-bit X: 5).
      M-step: r_hi, r_lo against [x | x^2] hi pieces and r_hi against the lo
        pieces: 6 columns of d for fp32 X, 5 for 16-bit X; S0: r_hi and r_lo
        against 16 columns of ones (64 FLOPs).
      Cluster kernel: one E-step + M-step.  Two sweeps: sweep 1's E-step, then
        sweep 2's E-step again + M-step.  Small-mixture kernel: E-step N = 2 KP
        columns over 3d operand features, M-step 4 KP rows over 128 operand
        features, KP = 16 or 32 component slots."""
    e = (10 if dtype != "f32" else 12) * d
    m = (10 if dtype != "f32" else 12) * d + 64
    if path == "tcgen05-single-sweep-cluster":
        return e + m
    if path == "tcgen05-two-sweep":
        return 2 * e + m
    if path == "tcgen05-single-sweep-smallk":
        kp = 16 if K <= 16 else 32
        return (2 * 2 * kp * 3 * d + 2 * 4 * kp * 128) / K
    return None


def lib_path_name(lib, N, w, flags=0) -> str:
    """Which kernels gmm_em_step runs for this shape (the library's regime rule)."""
    r = lib.gmm_regime(N, w.d, w.K, {"f32": 0, "bf16": 1, "f16": 2}[w.dtype], flags)
    if int(r) == 1 and w.K > 128:
        return "tcgen05-single-sweep-cluster"
    if int(r) == 1 and w.dtype != "f32" and w.d == 32 and w.K <= 32:
        return "tcgen05-single-sweep-smallk"
    return {0: "simt-two-sweep", 1: "tcgen05-single-sweep", 2: "tcgen05-two-sweep"}[int(r)]


if __name__ == "__main__":
    sys.exit(main())
