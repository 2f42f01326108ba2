#!/usr/bin/env python
"""Benchmark of the batch-1 LUT binary GEMV on B200.

Workload (the headline): M = N = 4096, K = 2 global +/-1 bases, g = 4, 128
salient columns with 2 extra bases, batch 1, fp16 x ~ N(0,1),
alpha ~ |N(0,0.02)| + 1e-3.  64 distinct weight sets of that shape (285 MB,
more than twice the 126 MB L2) are rotated so every GEMV streams its weights
from HBM.  One step = 1024 back-to-back GEMVs (16 passes over the 64 sets),
captured in a CUDA graph of fb_gemv launches with programmatic dependent
launch.  Every GEMV has its own freshly drawn x and its own y, so the GEMVs
are independent and are launched with FB_GEMV_INDEPENDENT (each may overlap
its predecessor; completion order is kept).  The same graph with every GEMV
waiting for its predecessor before reading x (a dependent decode chain) is
timed too and reported as "dependent_chain".

Printed: one JSON line (rank 0).  value = achieved GB/s of algorithmic bytes
(packed planes, scales, salient data, x, y) over all ranks; also GEMV us, the
g = 8 variant on the same weights, the 7B-shaped decode step (224 GEMVs), the
roofline of the GEMV kernel against the measured HBM peak, every workload at
its own shape, a dense fp16 comparator with energy per call, e2e through the
public API with pinned host buffers copied in and out every step (graph-replayed
and eager calls), the fitter (a whole 4096 x 4096 fit from a dense layer), and
the fp64 CPU oracle as baseline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""

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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GEMV µs & achieved HBM GB/s (% peak) at 4096×4096 K=2; 7B-shaped step ms"
WEIGHT_SETS = 64
PASSES_PER_STEP = 16
FALLBACK_HBM_GBS = 6650.0
SM_MAX_GHZ = 1.965   # clocks.max.sm of this machine's B200s


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-7b", action="store_true", help="skip the 7B-shaped step measurement")
    ap.add_argument("--no-cpu", action="store_true", help="skip the CPU oracle baseline")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-workload timings")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--profile", action="store_true",
                    help="small case for ncu: 32 weight sets (142 MB), one pass per step, headline graph only")
    ap.add_argument("--dependent", action="store_true",
                    help="with --profile: the graph as a dependent chain (the dependent-call plan)")
    ap.add_argument("--profile-batched", action="store_true",
                    help="for ncu: batch-16 calls on two 8192^2 K=3 layers (a few calls, independent flags)")
    ap.add_argument("--profile-fit", action="store_true",
                    help="for ncu --profile-from-start off: one whole 4096^2 fit inside a profiler range, nothing else")
    return ap.parse_args()


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest():
    h = hashlib.sha256()
    for f in ("lut_binary_gemv_b200/csrc/gemv.cu", "lut_binary_gemv_b200/csrc/fb_internal.cuh"):
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()


def ncu_traffic(kernel_tag):
    """DRAM bytes per launch from the committed ncu summary, only if it was
    taken on the current kernel source."""
    try:
        d = json.load(open(os.path.join(ROOT, "profiles", "ncu_traffic.json")))
        e = d[kernel_tag]
        if e["source_sha256"] == source_digest():
            return float(e["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.out = os.path.join("/tmp", f"fb_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.gpu_id)], stdout=open(self.out, "w"), stderr=subprocess.DEVNULL)
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
        for line in open(self.out):
            parts = [s.strip() for s in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], swp=parts[8]))
            except ValueError:
                continue
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("swp", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows),
                "power_w_mean": round(statistics.mean(r["power"] for r in rows), 1)}


def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if args.impl == "ours" else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=180))
    if args.impl == "ours":
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    device = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_config():
    return {"workload": "layer_4096x4096_k2_g4_s128", "M": 4096, "N": 4096, "K": 2, "g": 4, "nS": 128,
            "Ks": 2, "batch": 1, "x_dtype": "f16", "weight_sets": WEIGHT_SETS,
            "gemvs_per_step": WEIGHT_SETS * PASSES_PER_STEP,
            "l2": "inputs larger than L2: 64 distinct weight sets (285 MB) rotated, no flush",
            "launch": "CUDA graph of fb_gemv, PDL + FB_GEMV_INDEPENDENT (fresh x and own y per GEMV)"}


# --------------------------------------------------------------------------
def cpu_baseline(seconds):
    """The fp64 oracle (dense dequantisation + fp64 dot) on this host's cores:
    all cores (OpenMP over rows), and one core on a bounded row sample."""
    import oracle
    import workloads as wl
    p = wl.layer4096()
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    cores = oracle.num_threads()
    oracle.gemv(w, x)                        # warm (page in, thread pool)
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.gemv(w, x)
        n += 1
        dt = time.perf_counter() - t0
        if dt >= seconds:
            break
    per = dt / n
    # one core: a bounded sample of rows (about a third of the time budget)
    oracle.set_num_threads(1)
    try:
        rows = 512
        sel = np.arange(rows)
        oracle.gemv(w, x, sel)
        n1, t1 = 0, time.perf_counter()
        while True:
            oracle.gemv(w, x, sel)
            n1 += 1
            dt1 = time.perf_counter() - t1
            if dt1 >= seconds / 3:
                break
        per1 = dt1 / n1 * (p.M / rows)       # scaled to a whole GEMV
    finally:
        oracle.set_num_threads(cores)
    return {"value": round(p.algorithmic_bytes() / per / 1e9, 4), "unit": "GB/s", "cores": cores,
            "affinity_cpus": len(os.sched_getaffinity(0)), "kind": "oracle", "sample": f"{n} full 4096x4096 K=2 GEMVs (all rows) of the same workload, "
            f"{per * 1e3:.1f} ms each", "ms_per_gemv": round(per * 1e3, 3),
            "single_core": {"value": round(p.algorithmic_bytes() / per1 / 1e9, 4), "unit": "GB/s", "cores": 1,
                            "ms_per_gemv": round(per1 * 1e3, 3),
                            "sample": f"{n1} passes over rows 0..{rows - 1} of the same GEMV, scaled to 4096 rows"}}


def run_reference(args):
    if int(os.environ.get("RANK", "0")) != 0:
        return                              # the oracle runs once, on rank 0's host

    import oracle
    import workloads as wl
    p = wl.layer4096()
    w = oracle.OracleWeights.from_problem(p)
    x = oracle.x_to_f64(p.x, p.x_dtype)
    oracle.gemv(w, x)
    t1 = time.perf_counter()
    oracle.gemv(w, x)
    one = time.perf_counter() - t1
    # each step: a bounded row sample so the whole run stays within a few minutes
    budget = 150.0 / max(1, args.steps + args.warmup)
    rows = p.M if one <= budget else max(32, int(p.M * budget / one) // 32 * 32)
    sel = np.arange(rows)
    for _ in range(args.warmup):
        oracle.gemv(w, x, sel)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemv(w, x, sel)
    dt = time.perf_counter() - t0
    frac_rows = rows / p.M
    gbs = p.algorithmic_bytes() * frac_rows * args.steps / dt / 1e9
    cores = oracle.num_threads()
    sample = f"rows 0..{rows - 1} of the 4096x4096 K=2 GEMV per step ({rows / p.M:.3f} of the matrix)"
    line = {"impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(),
            "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                             "affinity_cpus": len(os.sched_getaffinity(0)), "kind": "oracle", "sample": sample},
            "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------
def make_sets(n, device):
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    Ws, xs, bytes_per = [], [], None
    for r in range(n):
        p = wl.layer4096(seed=1 if r == 0 else (1, r))
        Ws.append(fb.Weights.from_problem(p, device=device))
        xs.append(torch.from_numpy(p.x[0]).to(device))
        bytes_per = p.algorithmic_bytes()
    torch.cuda.synchronize()
    return Ws, xs, bytes_per


def capture(stream, body):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        body()                         # warm-up launch outside capture (sets kernel attributes)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            body()
    torch.cuda.synchronize()
    return g


def time_graph(graph, stream, steps, warmup, world, sampler=None):
    import torch
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        for _ in range(steps):
            graph.replay()
        end.record(stream)
    end.synchronize()
    torch.cuda.synchronize()
    clocks = sampler.stop() if sampler else None
    barrier(world)
    ms = start.elapsed_time(end)
    return max_over_ranks(ms, world), clocks


def run_ours(args):
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    from lut_binary_gemv_b200 import build as fb_build

    rank, world, local = dist_setup(args)
    if rank == 0:
        fb_build.build()
    barrier(world)
    device = f"cuda:{local}"
    peak, peak_src = measured_peak()

    if args.profile_fit:
        profile_fit(device)
        return
    if args.profile_batched:
        profile_batched(device)
        return

    global WEIGHT_SETS, PASSES_PER_STEP
    if args.profile:
        WEIGHT_SETS, PASSES_PER_STEP = 32, 1
    Ws, xs, bytes_per = make_sets(WEIGHT_SETS, device)
    ys = [torch.empty(4096, dtype=torch.float32, device=device) for _ in range(WEIGHT_SETS)]
    stream = torch.cuda.Stream(device=device)

    indep = fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT

    def step(sets, flags):
        def body():
            for _ in range(PASSES_PER_STEP):
                for r in range(WEIGHT_SETS):
                    fb.fb_gemv(sets[r], xs[r], y=ys[r], flags=flags)
        return body

    gemvs = WEIGHT_SETS * PASSES_PER_STEP
    graph = capture(stream, step(Ws, fb.FB_GEMV_PDL if (args.profile and args.dependent) else indep))
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_id = vis.split(",")[local] if vis else str(local)
    sampler = ClockSampler(gpu_id)
    ms, clocks = time_graph(graph, stream, args.steps, args.warmup, world, sampler)
    us_per_gemv = ms * 1e3 / (args.steps * gemvs)
    gbs_rank = bytes_per / (us_per_gemv * 1e-6) / 1e9
    value = gbs_rank * world
    if args.profile:
        # one more replay of the whole graph inside a profiler range, so that
        # `ncu --profile-from-start off --graph-profiling graph` measures the
        # calls as they run together (overlapped or chained), not one by one
        torch.cuda.synchronize()
        torch.cuda.profiler.start()
        with torch.cuda.stream(stream):
            graph.replay()
        torch.cuda.synchronize()
        torch.cuda.profiler.stop()
    del graph
    if args.profile:
        if rank == 0:
            print(json.dumps({"profile_run": True, "gemv_us": round(us_per_gemv, 4),
                              "gemvs": args.steps * gemvs}), flush=True)
        return

    def side(sets, flags):
        g = capture(stream, step(sets, flags))
        n = max(20, args.steps // 4)
        t, _ = time_graph(g, stream, n, args.warmup, world)
        us = t * 1e3 / (n * gemvs)
        gbs = bytes_per / (us * 1e-6) / 1e9
        return {"gemv_us": round(us, 4), "gbs": round(gbs, 2), "frac": round(gbs / peak, 4)}

    # the same GEMVs as a dependent chain (each waits for the previous before reading x)
    dependent = side(Ws, fb.FB_GEMV_PDL)
    dependent["note"] = "each GEMV reads x only after the previous kernel completes"
    # g = 8 tables on the same weights (the layout does not depend on g)
    Wg = [W.with_g(8) for W in Ws]
    g8 = side(Wg, indep)
    g8["note"] = ("same weights declared with g = 8: the GEMV builds the same 256-entry byte tables for every g, "
                  "so this times the headline kernel again (g changes neither the work nor the result bits)")
    g8_dep = side(Wg, fb.FB_GEMV_PDL)
    g8["dependent_chain_gemv_us"] = g8_dep["gemv_us"]

    # e2e through the public API, every step: the step's x copied in from
    # pinned host memory, its 64 fb_gemv calls (independent calls, replayed
    # from a captured CUDA graph), its y read back into pinned host memory.
    # Steps rotate through three buffer sets: step k's copies and GEMVs run
    # on their own streams (host-to-device, compute k % 3, device-to-host), so they
    # overlap the neighbouring steps' work; events keep each buffer's copy in
    # -> GEMVs -> copy out order.  The timed region spans the first step's
    # copy in to the last step's copy out.  The same with 64 eager Python
    # calls per step on one stream, not overlapped, is reported beside it.
    n_e2e = WEIGHT_SETS
    x_host = torch.stack([x.cpu() for x in xs]).pin_memory()
    NBUF = 3   # buffer sets (and compute streams) the steps rotate through
    y_hosts = [torch.empty((n_e2e, 4096), dtype=torch.float32).pin_memory() for _ in range(NBUF)]
    y_host = y_hosts[0]
    x_devs = [torch.empty_like(x_host, device=device) for _ in range(NBUF)]
    y_devs = [torch.empty((n_e2e, 4096), dtype=torch.float32, device=device) for _ in range(NBUF)]
    x_dev, y_dev = x_devs[0], y_devs[0]
    e2e_steps = max(10, args.steps // 10)

    def e2e_run(step_fn, steps):
        with torch.cuda.stream(stream):
            for _ in range(3):
                step_fn()
            torch.cuda.synchronize()
            barrier(world)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            for _ in range(steps):
                step_fn()
            s1.record(stream)
            s1.synchronize()
        ms_e = max_over_ranks(s0.elapsed_time(s1), world)
        return bytes_per * n_e2e * steps / (ms_e * 1e-3) / 1e9 * world

    def gemvs_e2e(b):
        def body():
            for r in range(n_e2e):
                fb.fb_gemv(Ws[r], x_devs[b][r], y=y_devs[b][r], flags=indep)
        return body
    g_e2e = [capture(stream, gemvs_e2e(b)) for b in range(NBUF)]
    h2d, d2h = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    comp = [torch.cuda.Stream(device=device) for _ in range(NBUF)]
    ev_in = [torch.cuda.Event() for _ in range(NBUF)]
    ev_comp = [torch.cuda.Event() for _ in range(NBUF)]
    ev_out = [torch.cuda.Event() for _ in range(NBUF)]

    def e2e_pipelined(steps):
        for _ in range(3):   # warm-up, one buffer at a time
            for b in range(NBUF):
                x_devs[b].copy_(x_host, non_blocking=True)
                g_e2e[b].replay()
                y_hosts[b].copy_(y_devs[b], non_blocking=True)
        torch.cuda.synchronize()
        barrier(world)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(h2d)
        for st in (d2h, *comp):
            st.wait_event(s0)
        for k in range(steps):
            b = k % NBUF
            with torch.cuda.stream(h2d):
                h2d.wait_event(ev_comp[b])          # step k - NBUF has finished reading x_devs[b]
                x_devs[b].copy_(x_host, non_blocking=True)
                ev_in[b].record(h2d)
            with torch.cuda.stream(comp[b]):
                comp[b].wait_event(ev_in[b])
                comp[b].wait_event(ev_out[b])       # step k - NBUF's y has left y_devs[b]
                g_e2e[b].replay()
                ev_comp[b].record(comp[b])
            with torch.cuda.stream(d2h):
                d2h.wait_event(ev_comp[b])
                y_hosts[b].copy_(y_devs[b], non_blocking=True)
                ev_out[b].record(d2h)
        s1.record(d2h)                              # after the last step's copy out (and so all before it)
        s1.synchronize()
        ms_e = max_over_ranks(s0.elapsed_time(s1), world)
        return bytes_per * n_e2e * steps / (ms_e * 1e-3) / 1e9 * world

    def eager_step():
        x_dev.copy_(x_host, non_blocking=True)
        for r in range(n_e2e):
            fb.fb_gemv(Ws[r], x_dev[r], y=y_dev[r])
        y_host.copy_(y_dev, non_blocking=True)

    e2e_gbs = e2e_pipelined(e2e_steps)
    e2e_eager_gbs = e2e_run(eager_step, e2e_steps)
    del g_e2e
    torch.cuda.synchronize()

    step7b = None
    if not args.no_7b:
        step7b = bench_7b(args, device, stream, world, peak)
    configs = None if args.no_configs else bench_configs(args, device, stream, world, peak)
    ours_energy = round(clocks["power_w_mean"] * us_per_gemv, 2) if clocks and clocks.get("power_w_mean") else None
    fp16 = None if args.no_configs else bench_vs_fp16(args, device, stream, world, gpu_id)
    fitter = None if args.no_configs else bench_fit(args, device, stream, peak)
    group_scales = None if args.no_configs else bench_group_scales(args, device, stream, world, peak)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        cpu = cpu_baseline(args.cpu_seconds)

    traffic = ncu_traffic("gemv_g4_f16_layer4096")
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": dict(workload_config(), parallelism=f"replicas{world}"),
        "gemv_us": round(us_per_gemv, 4),
        "roofline": {"bound": "hbm", "achieved": round(gbs_rank, 2), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs_rank / peak, 4), "traffic": traffic,
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": bytes_per},
        "dependent_chain": dependent,
        "variants": {"g8_pair_tables": g8},
        "step_7b": step7b,
        "configs": configs,
        "energy_uj_per_gemv": ours_energy,
        "fp16_dense_comparator": fp16,
        "fitter": fitter,
        "group_scales": group_scales,
        "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s", "h2d_bytes_per_step": int(x_host.numel() * 2),
                "d2h_bytes_per_step": int(y_host.numel() * 4),
                "note": (f"per step: pinned host x ({n_e2e} x 4096 fp16) copied in, {n_e2e} fb_gemv calls "
                         "(PDL + FB_GEMV_INDEPENDENT, replayed from a CUDA graph), y read back to pinned host; "
                         "steps rotate through three buffer sets on their own streams, so one step's copies "
                         "overlap its neighbours' GEMVs")},
        "e2e_eager": {"value": round(e2e_eager_gbs, 2), "unit": "GB/s",
                      "note": f"the same with {n_e2e} eager Python fb_gemv calls per step (dependent-call plan)"},
        "gpu_launches": args.steps * gemvs,
        "clocks": clocks,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def bench_7b(args, device, stream, world, peak):
    """The 7B-shaped decode step: 32 layers x (q,k,v,o 4096x4096; gate, up
    11008x4096; down 4096x11008), K=2, g=4, 3% salient, fresh fp16 x per GEMV;
    224 GEMVs in one CUDA graph with programmatic dependent launch."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    Ws, xs, ys, total = [], [], [], 0
    for layer in range(wl.STEP7B_LAYERS):
        for m in range(len(wl.STEP7B_MATRICES)):
            p = wl.step7b_matrix(layer, m)
            Ws.append(fb.Weights.from_problem(p, device=device))
            xs.append(torch.from_numpy(p.x[0]).to(device))
            ys.append(torch.empty(p.M, dtype=torch.float32, device=device))
            total += p.algorithmic_bytes()
    def run(flags, steps):
        def body():
            for W, x, y in zip(Ws, xs, ys):
                fb.fb_gemv(W, x, y=y, flags=flags)
        graph = capture(stream, body)
        ms, _ = time_graph(graph, stream, steps, args.warmup, world)
        return ms / steps

    steps = max(30, args.steps // 4)
    per = run(fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT, steps)
    per_dep = run(fb.FB_GEMV_PDL, steps)
    per_plain = run(0, steps)               # ordinary launches: no programmatic dependent launch
    gbs = total / (per * 1e-3) / 1e9

    # Grouped: per layer q,k,v in one launch, o, gate,up in one launch, down
    # (4 launches; x shared within a group, as in a decoder layer).
    nm = len(wl.STEP7B_MATRICES)
    groups = []
    for layer in range(wl.STEP7B_LAYERS):
        base = layer * nm
        for ms in ((0, 1, 2), (3,), (4, 5), (6,)):
            groups.append(([Ws[base + m] for m in ms], xs[base + ms[0]], [ys[base + m] for m in ms]))
    xb = 2   # fp16 x
    total_g = total - sum((len(Wg) - 1) * Wg[0].N * xb for Wg, _, _ in groups)

    def run_grouped(flags, steps):
        def body():
            for Wg, x, yg in groups:
                fb.fb_gemv_grouped(Wg, x, yg, flags=flags)
        graph = capture(stream, body)
        ms, _ = time_graph(graph, stream, steps, args.warmup, world)
        return ms / steps

    per_g = run_grouped(fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT, steps)
    per_g_dep = run_grouped(fb.FB_GEMV_PDL, steps)
    return {"ms": round(per, 5), "gbs": round(gbs, 2), "frac": round(gbs / peak, 4),
            "ms_dependent_chain": round(per_dep, 5),
            "frac_dependent_chain": round(total / (per_dep * 1e-3) / 1e9 / peak, 4),
            "ms_plain_chain": round(per_plain, 5),
            "frac_plain_chain": round(total / (per_plain * 1e-3) / 1e9 / peak, 4),
            "algorithmic_bytes": total, "gemvs": len(Ws), "steps": steps,
            "note": "224 GEMVs, fresh x per GEMV (independent); dependent chain: each waits for its predecessor "
                    "(programmatic dependent launch); plain chain: the same with ordinary launches",
            "grouped": {"ms": round(per_g, 5), "frac": round(total_g / (per_g * 1e-3) / 1e9 / peak, 4),
                        "ms_dependent_chain": round(per_g_dep, 5),
                        "frac_dependent_chain": round(total_g / (per_g_dep * 1e-3) / 1e9 / peak, 4),
                        "launches": len(groups), "algorithmic_bytes": total_g,
                        "note": "fb_gemv_grouped: q,k,v and gate,up each one launch reading one x"}}


def bench_configs(args, device, stream, world, peak):
    """Every workload of the build at its own shape: µs per call and the
    fraction of the HBM roofline (algorithmic bytes per call, all tokens'
    x and y included).  Distinct weight sets are rotated so that each config
    streams more than the 126 MB L2 (except the 256x256 case, which fits in
    L2 whatever is done).  Calls are launched as in the headline: a CUDA
    graph of independent calls (PDL + FB_GEMV_INDEPENDENT)."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    indep = fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT
    l2 = 126e6
    out = {}

    def measure(name, make, batches=(1,)):
        p0 = make(0)
        per_set = p0.algorithmic_bytes() - p0.batch * (p0.N * {"f32": 4, "f16": 2, "bf16": 2}[p0.x_dtype] + 4 * p0.M)
        nsets = max(1, min(16, int(2 * l2 // per_set) + 1)) if per_set * 2 < 16 * l2 else 1
        ps = [p0] + [make(i) for i in range(1, nsets)]
        Ws = [fb.Weights.from_problem(p, device=device) for p in ps]
        Xs = [torch.from_numpy(p.x.view(np.int16)).to(device).view(torch.bfloat16) if p.x_dtype == "bf16"
              else torch.from_numpy(p.x).to(device) for p in ps]
        del ps
        res = {}
        for B in batches:
            Ys = [torch.empty((B, p0.M), dtype=torch.float32, device=device) for _ in Ws]
            reps = max(-(-32 // len(Ws)), int(4 * l2 // (per_set * len(Ws))))   # >= 32 calls per graph

            def body():
                for _ in range(reps):
                    for W, X, Y in zip(Ws, Xs, Ys):
                        if B == 1:
                            fb.fb_gemv(W, X[0], y=Y[0], flags=indep)
                        else:
                            fb.fb_gemv_batched(W, X[:B], Y=Y, flags=indep)
            g = capture(stream, body)
            n = max(5, args.steps // 20)
            ms, _ = time_graph(g, stream, n, args.warmup, world)
            calls = n * reps * len(Ws)
            us = ms * 1e3 / calls
            xb = {"f32": 4, "f16": 2, "bf16": 2}[p0.x_dtype]
            nbytes = per_set + B * (p0.N * xb + 4 * p0.M)
            gbs = nbytes / (us * 1e-6) / 1e9
            r = {"us_per_call": round(us, 3), "us_per_token": round(us / B, 3), "gbs": round(gbs, 1),
                 "frac": round(gbs / peak, 4), "weight_sets": len(Ws), "fits_l2": per_set * len(Ws) < l2}
            if B > 1:
                # shared-memory roof: every weight byte is one 4-byte table
                # lookup per token; 148 SMs x 128 B per clock at the top clock
                wbytes = p0.K * p0.M * p0.N // 8 + (p0.Ks * p0.M * p0.nS_pad // 8 if p0.nS else 0)
                roof_us = B * wbytes * 4 / (148 * 128 * SM_MAX_GHZ * 1e9) * 1e6
                r["smem_roof"] = {"us": round(roof_us, 3), "frac": round(roof_us / us, 4),
                                  "basis": "B x weight bytes x 4 B lookups / (148 SMs x 128 B/clk x 1.965 GHz)"}
            res[f"batch{B}"] = r
            del g, Ys
        out[name] = res if len(batches) > 1 else res["batch1"]
        del Ws, Xs
        torch.cuda.synchronize()

    measure("tiny_256x256_k2_g4", lambda i: wl.make_problem(256, 256, 2, g=4, nS=0, x_dtype="f32", alpha_dist="unit",
                                                             seed=(5, i)))
    measure("ternary_11008x4096", lambda i: wl.ternary11008() if i == 0 else
            wl.make_problem(11008, 4096, 2, g=4, nS=0, x_dtype="bf16", seed=(6, i), ternary=True))
    for si, (M, N) in enumerate(wl.SHAPES70B):
        measure(f"layer70b_{M}x{N}_k3_g8", lambda i, si=si: wl.layer70b(si, 16) if i == 0 else
                wl.make_problem(M, N, 3, g=8, nS=wl.salient_count(0.05, N), Ks=2, batch=16, x_dtype="f16",
                                alpha_dist="small", seed=(7, si, i)), batches=wl.BATCHES70B)
    return out


def bench_group_scales(args, device, stream, world, peak):
    """The group-wise row-scale format at 4096 x 4096 (K = 2, 128 salient
    columns with 2 bases, fp16 x): one row scale per 128 input columns
    (fb_gemv_group_scales, G = 128), independent and dependent graphs over
    rotating weight sets.  Algorithmic bytes as for the ordinary format with
    the row scales K * N/G * M * 4 bytes instead of K * M * 4."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    G, nsets = 128, 48
    ps = [wl.layer4096(seed=1 if i == 0 else (1, i)) for i in range(nsets)]
    p0 = ps[0]
    Ws = [fb.Weights.from_problem(p, device=device) for p in ps]
    ars = [torch.from_numpy(np.ascontiguousarray(np.transpose(
        wl.group_row_scales(p.K, p.M, p.N // G, seed=(43, i)), (0, 2, 1)))).to(device) for i, p in enumerate(ps)]
    xs = [torch.from_numpy(p.x[0]).to(device) for p in ps]
    ys = [torch.empty(p0.M, dtype=torch.float32, device=device) for _ in ps]
    nbytes = p0.algorithmic_bytes() - 4 * p0.K * p0.M + 4 * p0.K * (p0.N // G) * p0.M
    del ps
    out = {"workload": "layer_4096x4096_k2_s128_G128", "G": G, "algorithmic_bytes": nbytes}
    for name, flags in (("independent", fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT), ("dependent", fb.FB_GEMV_PDL)):
        def body():
            for _ in range(4):
                for W, a, x, y in zip(Ws, ars, xs, ys):
                    fb.fb_gemv_group_scales(W, G, x, a, y=y, flags=flags)
        g = capture(stream, body)
        n = max(10, args.steps // 10)
        ms, _ = time_graph(g, stream, n, args.warmup, world)
        del g
        us = ms * 1e3 / (n * 4 * nsets)
        gbs = nbytes / (us * 1e-6) / 1e9
        out[name] = {"gemv_us": round(us, 3), "gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    return out


def profile_batched(device):
    """A small case of the batched kernel for ncu: batch-16 calls on two
    8192 x 8192 K = 3 layers (5% salient columns), three passes over both,
    eagerly (PDL + FB_GEMV_INDEPENDENT)."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    ps = [wl.layer70b(0, 16)] + [wl.make_problem(8192, 8192, 3, g=8, nS=wl.salient_count(0.05, 8192), Ks=2,
                                                 batch=16, x_dtype="f16", alpha_dist="small", seed=(7, 0, 1))]
    Ws = [fb.Weights.from_problem(p, device=device) for p in ps]
    Xs = [torch.from_numpy(p.x).to(device) for p in ps]
    Ys = [torch.empty((16, p.M), dtype=torch.float32, device=device) for p in ps]
    for _ in range(3):
        for W, X, Y in zip(Ws, Xs, Ys):
            fb.fb_gemv_batched(W, X, Y=Y, flags=fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT)
    torch.cuda.synchronize()
    print(json.dumps({"profile_batched": True, "calls": 6}), flush=True)


FIT_SHAPE = dict(M=4096, N=4096, K=2, Ks=2, nS=128, sweeps=8, T=64)


def profile_fit(device):
    """One whole fit of the bench's 4096^2 layer inside a profiler range
    (after two untimed fits), for a launch list of the fitter's kernels."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    f = FIT_SHAPE
    fi = wl.fit_inputs(f["M"], f["N"], T=f["T"], seed=21)
    W = torch.from_numpy(fi.W).to(device)
    X = torch.from_numpy(fi.X).to(device)
    for _ in range(2):
        fb.fit(W, X, f["K"], f["Ks"], f["nS"], f["sweeps"])
    torch.cuda.synchronize()
    torch.cuda.profiler.start()
    fb.fit(W, X, f["K"], f["Ks"], f["nS"], f["sweeps"])
    torch.cuda.synchronize()
    torch.cuda.profiler.stop()
    print(json.dumps({"profile_fit": True}), flush=True)


def bench_fit(args, device, stream, peak):
    """The fitter on a 4096 x 4096 layer (K = 2, 128 salient columns with Ks =
    2, 8 alternating sweeps, 64 calibration rows): ms per whole fit on the
    GPU, and the bytes its passes over the residual must move."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    M, N, K, Ks, nS, sweeps, T = (FIT_SHAPE[k] for k in ("M", "N", "K", "Ks", "nS", "sweeps", "T"))
    fi = wl.fit_inputs(M, N, T=T, seed=21)
    W = torch.from_numpy(fi.W).to(device)
    X = torch.from_numpy(fi.X).to(device)
    nS_pad = (nS + 31) // 32 * 32
    per_base = lambda m, n: (8 * sweeps + 9) * m * n        # 2 passes per sweep + read/write R + signs
    nbytes = (8 * M * N                                      # R = W
              + 4 * M * N + 4 * T * N                        # saliency: W and X once each
              + K * per_base(M, N)
              + 8 * M * nS_pad                               # gather of the salient columns
              + Ks * per_base(M, nS_pad))
    with torch.cuda.stream(stream):
        for _ in range(2):
            fb.fit(W, X, K, Ks, nS, sweeps)
        torch.cuda.synchronize()
        times = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            fb.fit(W, X, K, Ks, nS, sweeps)
            b.record(stream)
            b.synchronize()
            times.append(a.elapsed_time(b))
    ms_eager = statistics.median(times)
    # the same fit replayed from a CUDA graph (no host launch gaps)
    graph = capture(stream, lambda: fb.fit(W, X, K, Ks, nS, sweeps))
    gms, _ = time_graph(graph, stream, 10, 2, 1)
    del graph
    ms = gms / 10
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"workload": "fit_4096x4096_k2_ks2_s128_sweeps8_t64", "ms_per_fit": round(ms, 3),
           "ms_per_fit_eager": round(ms_eager, 3),
           "algorithmic_bytes": nbytes, "gbs": round(gbs, 1), "frac": round(gbs / peak, 4),
           "launches_per_fit": 3 + (K + Ks) * (2 * sweeps + 1) + 1,
           "note": "fb.fit: saliency, K greedy bases on R = W, gather of the salient columns, Ks bases on them; "
                   "ms_per_fit: the fit's launches replayed from a CUDA graph (mean of 10); eager: C-ABI calls from "
                   "Python, median of 5"}
    if not args.no_cpu:
        import oracle.fit as ofit
        t0 = time.perf_counter()
        ofit.fit(fi.W, fi.X, K, Ks, nS, sweeps)
        out["cpu_baseline"] = {"ms_per_fit": round((time.perf_counter() - t0) * 1e3, 1), "kind": "oracle",
                               "cores": len(os.sched_getaffinity(0)), "sample": "one whole fit of the same layer (numpy fp64)"}
    return out


def bench_vs_fp16(args, device, stream, world, gpu_id):
    """The comparison the FluxBin page draws against uncompressed fp16
    weights, restated per GEMV on this GPU and like for like: on each shape,
    our GEMV (its own workload of that shape) and a dense fp16 matrix-vector
    product (torch.mv, i.e. cuBLAS) are each timed in the same two regimes:
      * dependent: one call after another on one stream, each waiting for
        the previous (ours: FB_GEMV_PDL; fp16: a plain stream of torch.mv);
      * overlapped: independent calls allowed to run at once (ours:
        FB_GEMV_PDL | FB_GEMV_INDEPENDENT; fp16: calls spread over 8 streams).
    Weight copies larger than twice L2 are rotated.  Energy per call = mean
    board power sampled during that arm's timed region x time per call."""
    import torch
    import lut_binary_gemv_b200 as fb
    import workloads as wl
    l2 = 126e6
    shapes = {
        "4096x4096": lambda i: wl.layer4096(seed=1 if i == 0 else (1, i)),
        "11008x4096": lambda i: wl.step7b_matrix(i, 4),
        "8192x8192": lambda i: wl.make_problem(8192, 8192, 3, g=8, nS=wl.salient_count(0.05, 8192), Ks=2,
                                               batch=1, x_dtype="f16", alpha_dist="small", seed=(7, 0, i)),
    }

    def arm(body, calls):
        graph = capture(stream, body)
        one, _ = time_graph(graph, stream, 2, 1, world)
        n = max(10, int(400.0 / max(one / 2, 1e-3)))        # about 0.4 s of timed work for the power samples
        sampler = ClockSampler(gpu_id)
        ms, clocks = time_graph(graph, stream, n, args.warmup, world, sampler)
        del graph
        us = ms * 1e3 / (n * calls)
        e = {"us": round(us, 3)}
        if clocks and clocks.get("power_w_mean"):
            e["power_w"] = clocks["power_w_mean"]
            e["energy_uj_per_gemv"] = round(clocks["power_w_mean"] * us, 2)
        return e

    out = {}
    for name, make in shapes.items():
        p0 = make(0)
        M, N = p0.M, p0.N
        per_ours = p0.algorithmic_bytes()
        n_ours = max(2, int(2 * l2 // per_ours) + 1)
        ps = [p0] + [make(i) for i in range(1, n_ours)]
        Ws = [fb.Weights.from_problem(p, device=device) for p in ps]
        xs = [torch.from_numpy(p.x[0]).to(device) for p in ps]
        ys = [torch.empty(M, dtype=torch.float32, device=device) for _ in ps]
        del ps
        reps = max(1, 256 // n_ours)

        def ours(flags):
            def body():
                for _ in range(reps):
                    for W, x, y in zip(Ws, xs, ys):
                        fb.fb_gemv(W, x, y=y, flags=flags)
            return body
        r = {"ours_bytes_per_call": per_ours}
        r["ours_dependent"] = arm(ours(fb.FB_GEMV_PDL), reps * n_ours)
        r["ours_overlapped"] = arm(ours(fb.FB_GEMV_PDL | fb.FB_GEMV_INDEPENDENT), reps * n_ours)
        del Ws, xs, ys

        per_fp16 = M * N * 2
        n_fp = max(2, int(2 * l2 // per_fp16) + 1)
        g = torch.Generator(device=device).manual_seed(M * 7 + N)
        Wd = [torch.randn(M, N, device=device, dtype=torch.float16, generator=g) * 0.02 for _ in range(n_fp)]
        xd = torch.randn(N, device=device, dtype=torch.float16, generator=g)
        yd = [torch.empty(M, device=device, dtype=torch.float16) for _ in range(n_fp)]
        reps_fp = max(1, 128 // n_fp)
        side = [torch.cuda.Stream(device=device) for _ in range(8)]

        def fp16_dep():
            for _ in range(reps_fp):
                for W, y in zip(Wd, yd):
                    torch.mv(W, xd, out=y)

        def fp16_overlap():
            cur = torch.cuda.current_stream()
            for s in side:
                s.wait_stream(cur)
            k = 0
            for _ in range(reps_fp):
                for W, y in zip(Wd, yd):
                    with torch.cuda.stream(side[k % len(side)]):
                        torch.mv(W, xd, out=y)
                    k += 1
            for s in side:
                cur.wait_stream(s)
        r["fp16_bytes_per_call"] = per_fp16 + 2 * N + 2 * M
        r["fp16_dependent"] = arm(fp16_dep, reps_fp * n_fp)
        r["fp16_overlapped"] = arm(fp16_overlap, reps_fp * n_fp)
        del Wd, yd
        torch.cuda.synchronize()
        for regime in ("dependent", "overlapped"):
            a, b = r[f"ours_{regime}"], r[f"fp16_{regime}"]
            r[f"speedup_{regime}"] = round(b["us"] / a["us"], 2)
            if "energy_uj_per_gemv" in a and "energy_uj_per_gemv" in b:
                r[f"energy_ratio_{regime}"] = round(b["energy_uj_per_gemv"] / a["energy_uj_per_gemv"], 2)
        out[name] = r
    out["note"] = ("same regime on both sides: speedup = fp16 us / ours us, energy_ratio = fp16 energy / ours; "
                   "ours = the build's workload of that shape (4096: K=2 g=4 128 salient; 11008x4096: 7B gate, "
                   "K=2 3% salient; 8192: K=3 g=8 5% salient); fp16 = torch.mv on random weights")
    return out


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
