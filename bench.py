#!/usr/bin/env python
"""Throughput of exact batched Lloyd k-means on B200 (iterations per second).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config 2] [--impl fkm|reference]

A step is one full Lloyd run of the workload (its configured iterations of
assign + sort-inverse update through fkm_lloyd), inputs resident in HBM.  The
metric is Lloyd iterations/sec on the B x N x K x D problem; the JSON line
also carries the assign kernel's TFLOP/s and the update stages' GB/s, both
from CUDA events recorded on the launching stream inside the timed region.

Default workload (the largest device-resident one): B=1, N=2^24, D=128,
K=4096, bf16 Gaussian mixture with Zipf(1.1) component weights (hot
clusters), 5 iterations, tol=0 (4 GiB of points: larger than L2, so no flush
is needed between steps).  --config 2 is the pages' motivation shape (B=32,
N=65536, D=128, K=1024).  Under torchrun (N > 1) every rank runs its own
independent batch of problems (different seeds): weak scaling, no collective
on the data path.

--impl reference times the fp64 CPU oracle (the reference arm of this build)
on a bounded sample of the same workload on this host's cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import datagen  # noqa: E402

METRIC = "Lloyd iterations/sec (assign+update) per BxNxKxD"
UNIT = "iters/s"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "assign_traffic.json")
ASSIGN_SRC = os.path.join(ROOT, "exact_means_clustering_b200", "csrc", "assign_tc.cu")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

REASON_BITS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}


def workload_config(w: datagen.Workload) -> dict:
    return {"workload": w.name, "B": w.B, "N": w.N, "D": w.D, "K": w.K, "dtype": w.dtype,
            "iters_per_step": w.iters, "tol": w.tol,
            "data": ("seeded Gaussian mixture" if w.n_comp else "seeded standard normal"),
            "l2": f"inputs larger than L2 ({w.x_bytes / 2**20:.0f} MiB of points), no flush"}


def assign_flops(w):
    return 2.0 * w.B * w.N * w.K * w.D


def update_bytes(w):
    # points read once, ids read, new centroids written + previous read, counts written
    return (w.B * w.N * w.D * w.elem_bytes + 4.0 * w.B * w.N + 8.0 * w.B * w.K * w.D
            + 4.0 * w.B * w.K)


def iteration_frac(w, ms_per_iter, peaks):
    """The whole iteration against its roofline: max(assign FLOP at the burst
    bf16 peak, update bytes at the HBM peak) over the measured time."""
    if ms_per_iter <= 0:
        return None
    t_flop = assign_flops(w) * (3 if w.dtype == "f32" else 1) / (peaks["bf16_tflops"] * 1e12)
    t_bytes = update_bytes(w) / (peaks["hbm_gbs"] * 1e9)
    return max(t_flop, t_bytes) / (ms_per_iter / 1e3)


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except OSError:
        return FALLBACK_PEAKS, "fallback"


def source_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def assign_traffic(config_name):
    """DRAM bytes per assign launch from a committed ncu summary, when it was
    taken on the current kernel source for this workload; else None."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except OSError:
        return None
    if t.get("kernel_source_sha") != source_sha(ASSIGN_SRC):
        return None
    return t.get("per_launch_bytes", {}).get(config_name)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms."""

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        q = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def window(self, t0, t1):
        """Keep only samples read between host times t0 and t1 (the timed region)."""
        self.t0, self.t1 = t0, t1

    def __exit__(self, *exc):
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], 0.0, set()
        t0, t1 = getattr(self, "t0", 0.0), getattr(self, "t1", 1e30)
        for ts, ln in self.lines:
            if not (t0 <= ts <= t1 + 0.15):
                continue
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 5:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
                bits = int(parts[4], 16)
            except ValueError:
                continue
            for b, name in REASON_BITS.items():
                if bits & b and name != "gpu_idle":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def rank_workload(w, rank):
    """Rank r's own problems (weak scaling): the same recipe, seed + 1000 r."""
    return w.scaled(seed=w.seed + 1000 * rank)


def over_ranks(torch, dist, dev, t_ms, n_iters):
    """(max over ranks of the timed milliseconds, sum over ranks of the
    iterations done): the whole-job time is the slowest rank's."""
    if dist is None:
        return t_ms, n_iters
    t = torch.tensor([t_ms], device=dev, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    n = torch.tensor([n_iters], device=dev, dtype=torch.float64)
    dist.all_reduce(n, op=dist.ReduceOp.SUM)
    return t.item(), int(n.item())


def oracle_sample(w, iters, rows=None, metric="euclid"):
    """The fp64 oracle on batch 0 of the workload (its first `rows` points when
    given) for `iters` Lloyd iterations under `metric`.  Returns (seconds,
    scale, description): the whole problem's iteration costs `scale` times the
    sample's."""
    import oracle
    n = w.N if rows is None else max(min(int(rows), w.N), w.K)
    ws = w.scaled(B=1, N=n)
    x = datagen.points(ws)
    c0 = datagen.init_centroids(x, datagen.init_indices(ws), ws.dtype)
    mir = w.dtype if w.dtype != "f32" else None
    t0 = time.perf_counter()
    if metric == "euclid":
        oracle.lloyd(x, c0, iters, 0.0, dtype=w.dtype, mirror=mir)
    else:
        oracle.lloyd_sim(x, c0, iters, metric, 0.0, dtype=w.dtype, mirror=mir)
    dt = time.perf_counter() - t0
    scale = w.B * (w.N / n)
    part = "" if n == w.N else f"first {n} points of "
    desc = (f"extrapolated: {part}batch 0 of {w.B} (N={w.N}, K={w.K}, D={w.D}, {w.dtype}), {iters} Lloyd "
            f"iteration(s) of the fp64 oracle; rate scaled by 1/{scale:.4g} to the whole "
            f"problem (cost is linear in B*N at fixed K)")
    return dt, scale, desc


def comparison(fkm, torch, w, xt, c0t, ws, stream, dev, reps=3):
    """Milliseconds of one assign and one update by the pages' "standard"
    path (B x N x K fp32 distance matrix written to HBM then read back for the
    argmin; one fp32 atomicAdd per point per dimension) and by the fused path,
    on the workload's initial centroids."""
    B, N, K, D = w.B, w.N, w.K, w.D
    dist_bytes = 4 * B * N * K
    free, _ = torch.cuda.mem_get_info(dev)
    ids = torch.empty(B, N, dtype=torch.int32, device=dev)
    cen = torch.empty(B, K, D, dtype=torch.float32, device=dev)
    cnt = torch.empty(B, K, dtype=torch.int32, device=dev)

    def t(fn):
        fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        return e0.elapsed_time(e1) / reps

    out = {"centroids": "the initial centroids", "reps": reps}
    out["assign_fused_ms"] = t(lambda: fkm.fkm_assign(xt, c0t, ids, ws=ws, stream=stream))
    out["update_sort_inverse_ms"] = t(lambda: fkm.fkm_update(xt, ids, c0t, cen, cnt, ws=ws,
                                                             stream=stream))
    out["update_scatter_ms"] = t(lambda: fkm.fkm_baseline_update(xt, ids, c0t, cen, cnt, ws=ws,
                                                                 stream=stream))
    out["update_scatter_gbs"] = update_bytes(w) / (out["update_scatter_ms"] / 1e3) / 1e9
    # the optional centring pass (README "Centre your data"): the mean reads x,
    # the subtraction reads and writes it
    xc = torch.empty_like(xt)
    mu = torch.empty(B, D, dtype=torch.float32, device=dev)
    cws = fkm.workspace(fkm.fkm_centre_workspace_size_bytes(B, N, D), dev)
    out["centre_ms"] = t(lambda: fkm.fkm_centre(xt, mu=mu, out=xc, ws=cws, stream=stream))
    out["centre_gbs"] = 3 * w.x_bytes / (out["centre_ms"] / 1e3) / 1e9
    del xc
    if dist_bytes > 0.8 * free:
        out["assign_materialise"] = (f"not run: the distance matrix needs "
                                     f"{dist_bytes / 2**30:.0f} GiB")
    else:
        dist = torch.empty(B, N, K, dtype=torch.float32, device=dev)
        out["assign_materialise_ms"] = t(lambda: fkm.fkm_baseline_assign(xt, c0t, dist, ids,
                                                                         ws=ws, stream=stream))
        out["distance_matrix_bytes"] = dist_bytes
        del dist
    return out


def cpu_baseline(w, max_iters, budget_s=15.0, metric="euclid"):
    """The oracle's iteration rate on a bounded sample of the workload: a probe
    on a few thousand points of batch 0 sizes the sample (points of batch 0,
    and iterations up to max_iters) to about budget_s seconds of CPU work."""
    probe_rows = max(w.K, min(w.N, 4096))
    t_probe, _, _ = oracle_sample(w, 1, probe_rows, metric)
    per_row = max(t_probe, 1e-6) / probe_rows
    rows = int(min(w.N, max(probe_rows, budget_s / per_row)))
    iters = int(max(1, min(max_iters, budget_s / (per_row * rows))))
    dt, scale, desc = oracle_sample(w, iters, rows, metric)
    return iters / (dt * scale), desc


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    cores = cpu_cores()
    # size each step's sample so that the whole run takes about two minutes
    probe_rows = max(w.K, w.N // 64)
    t_probe, _, _ = oracle_sample(w, 1, probe_rows)
    per_step_budget = 120.0 / max(args.steps + args.warmup, 1)
    rows = int(probe_rows * per_step_budget / max(t_probe, 1e-6))
    for _ in range(args.warmup):
        oracle_sample(w, 1, rows)
    total, wall, desc = 0.0, 0.0, ""
    for _ in range(args.steps):
        dt, scale, desc = oracle_sample(w, 1, rows)
        total += dt * scale       # seconds one full-problem iteration would take
        wall += dt
    value = args.steps / total
    # ms_per_step is the time a step (one sample) took on this host; value is
    # the rate the whole problem would run at, extrapolated from the samples
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * wall / args.steps,
            "value_kind": "extrapolated from the samples (cost linear in B*N at fixed K)",
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(w), "impl": "reference",
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


HOST_CHUNK_ROWS = 1 << 23   # rows per streamed chunk of the host-resident workload


def measure_h2d_gbs(torch, dev, nbytes=1 << 30):
    """Pinned host -> device copy bandwidth (best of 5, CUDA events)."""
    src = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    dst = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    best = float("inf")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(6):
        e0.record()
        dst.copy_(src, non_blocking=True)
        e1.record()
        torch.cuda.synchronize(dev)
        best = min(best, e0.elapsed_time(e1))
    return nbytes / (best / 1e3) / 1e9


def run_host(args, w):
    """The host-resident workload: points stay in pinned host memory and every
    iteration streams them through the GPU in chunks (fkm_lloyd_host).  Its
    bound is the host link, so the roofline is taken against the measured
    pinned host-to-device bandwidth."""
    import torch
    import exact_means_clustering_b200 as fkm

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=600),
                                device_id=dev)
    wr = rank_workload(w, rank)
    B, N, D, K = wr.B, wr.N, wr.D, wr.K
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wr.dtype]
    xh = torch.empty((B, N, D), dtype=tdt, pin_memory=True)
    for b in range(B):
        datagen.fill_points(wr, b, xh[b].data_ptr())
    xv = xh.view(torch.int16).numpy().view(np.uint16) if wr.dtype == "bf16" else xh.numpy()
    c0 = datagen.init_centroids(xv, datagen.init_indices(wr), wr.dtype)
    ch = torch.from_numpy(c0).pin_memory()
    c0t = ch.to(dev)
    ids = torch.empty(B, N, dtype=torch.int32, device=dev)
    centers = torch.empty(B, K, D, dtype=torch.float32, device=dev)
    counts = torch.empty(B, K, dtype=torch.int32, device=dev)
    inertia = torch.empty(B, dtype=torch.float64, device=dev)
    ws = fkm.workspace(fkm.fkm_host_workspace_size(B, N, K, D, tdt, HOST_CHUNK_ROWS), dev)
    stream = torch.cuda.current_stream(dev)
    h2d = measure_h2d_gbs(torch, dev)

    def barrier():
        if dist is not None:
            dist.barrier()

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier()
        torch.cuda.synchronize(dev)
        h0 = time.time()
        e0.record(stream)
        n = 0
        for _ in range(args.steps):
            n += fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        h1 = time.time()
        barrier()
        t, n = over_ranks(torch, dist, dev, e0.elapsed_time(e1), n)
        return n, t, (h0, h1)

    def step():
        return fkm.fkm_lloyd_host(xh, c0t, wr.iters, wr.tol, HOST_CHUNK_ROWS, ids, centers,
                                  counts, inertia, ws=ws, stream=stream)

    launches0 = fkm.fkm_kernel_launches()
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        n_it, t_ms, (h0, h1) = timed(step)
        clk.window(h0, h1)
    launches = (fkm.fkm_kernel_launches() - launches0) / max(args.steps + args.warmup, 1) \
        * args.steps
    value = n_it / (t_ms / 1e3)
    per_iter_s = (t_ms / 1e3) / max(n_it / world, 1)
    x_bytes = wr.x_bytes
    achieved = x_bytes / per_iter_s / 1e9
    peaks, _ = load_peaks()
    products = 3 if wr.dtype == "f32" else 1   # fp32 points: split-bf16, three products
    tensor_s = products * assign_flops(wr) / (peaks.get("bf16_tflops_sustained", 1400.0) * 1e12)
    tensor_note = (f"the other bound: {products} x 2*N*K*D tensor-core FLOP per iteration at the "
                   f"measured sustained bf16 peak takes {tensor_s:.3f} s; the larger of the two "
                   f"terms binds")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wr.dtype, "data": "synthetic",
            "config": dict(workload_config(wr), chunk_rows=HOST_CHUNK_ROWS,
                           l2=f"points stream from pinned host memory "
                              f"({x_bytes / 2**30:.0f} GiB per iteration), no flush"),
            "roofline": {"bound": "h2d", "kernel": "whole iteration (host link)",
                         "achieved": achieved, "peak": h2d, "unit": "GB/s",
                         "frac": achieved / h2d, "traffic": None,
                         "peak_source": "measured pinned host-to-device copy, 1 GiB, this run",
                         "terms_s_per_iter": {"h2d": x_bytes / (h2d * 1e9),
                                              "tensor": tensor_s},
                         "note": tensor_note},
            "gpu_launches": int(launches),
            "clocks": clk.summary()}
    if not args.no_e2e:
        ids_h = torch.empty(B, N, dtype=torch.int32).pin_memory()
        cen_h = torch.empty(B, K, D, dtype=torch.float32).pin_memory()
        ine_h = torch.empty(B, dtype=torch.float64).pin_memory()

        def e2e_step():
            c0t.copy_(ch, non_blocking=True)
            n = step()
            ids_h.copy_(ids, non_blocking=True)
            cen_h.copy_(centers, non_blocking=True)
            ine_h.copy_(inertia, non_blocking=True)
            return n

        n_e, t_e, _ = timed(e2e_step)
        line["e2e"] = {"value": n_e / (t_e / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": int(wr.iters * x_bytes + ch.numel() * 4),
                       "d2h_bytes_per_step": int(ids_h.numel() * 4 + cen_h.numel() * 4
                                                 + ine_h.numel() * 8)}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        value_c, desc = cpu_baseline(wr, 1)
        line["cpu_baseline"] = {"value": value_c, "unit": UNIT, "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


def run_sharded(args, w):
    """One workload split over the ranks (README "Multi-GPU Support"): rank r
    holds rows [r*N/R, (r+1)*N/R) of every problem and runs the sharded Lloyd
    loop (assign and partial update on its shard, an NCCL all-reduce of the
    partial sums and counts, the same finalize everywhere).  Strong scaling:
    the whole problem's iterations per second, the time the slowest rank's."""
    import torch
    import exact_means_clustering_b200 as fkm

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    x = datagen.points(w)
    c0 = datagen.init_centroids(x, datagen.init_indices(w), w.dtype)
    r0, r1 = (w.N * rank) // world, (w.N * (rank + 1)) // world
    xs = np.ascontiguousarray(x[:, r0:r1])
    del x
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[w.dtype]
    xt = (torch.from_numpy(xs.view(np.int16)).view(torch.bfloat16) if w.dtype == "bf16"
          else torch.from_numpy(xs)).to(dev)
    c0t = torch.from_numpy(c0).to(dev)
    ws = fkm.workspace(fkm.fkm_workspace_size(w.B, r1 - r0, w.K, w.D, tdt), dev)

    def step():
        return fkm.lloyd_sharded(xt, c0t, w.iters, w.tol, ws=ws)[4]

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if dist is not None:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        time.sleep(0.3)
        h0 = time.time()
        e0.record()
        n = 0
        for _ in range(args.steps):
            n += step()
        e1.record()
        torch.cuda.synchronize(dev)
        clk.window(h0, time.time())
    t_ms = e0.elapsed_time(e1)
    if dist is not None:
        tt = torch.tensor([t_ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        t_ms = tt.item()
    value = n / (t_ms / 1e3)            # every rank ran the same n iterations of one problem
    peaks, src = load_peaks()
    peak_t = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    per_iter_s = t_ms / 1e3 / max(n, 1)
    achieved = assign_flops(w) / world / per_iter_s / 1e12
    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_ms / args.steps,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
            "dtype": w.dtype, "data": "synthetic",
            "config": dict(workload_config(w), sharded=True, rows_per_rank=r1 - r0),
            "roofline": {"bound": "tensor", "kernel": "whole sharded iteration, per GPU",
                         "achieved": achieved, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": achieved / peak_t, "traffic": None,
                         "peak_source": f"{src} (bf16 sustained, MEASURED_PEAKS.json)",
                         "note": "2*N*K*D / GPUs per whole iteration time: a lower bound on "
                                 "the assign kernel's rate"},
            "clocks": clk.summary()}
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", type=int, default=4, choices=sorted(datagen.CONFIGS))
    ap.add_argument("--impl", default="fkm", choices=["fkm", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-comparison", action="store_true")
    ap.add_argument("--sharded", action="store_true",
                    help="one problem split over the ranks' GPUs (strong scaling)")
    ap.add_argument("--oracle-iters", type=int, default=10)
    ap.add_argument("--points", type=int, default=0,
                    help="a smaller case of the workload for profiling: N points per batch "
                         "(same recipe; the line's config names the reduced size)")
    ap.add_argument("--metric", default="euclid", choices=["euclid", "dot", "cosine"],
                    help="similarity of the clustering (dot and cosine k-means: fkm_lloyd_metric)")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = datagen.CONFIGS[args.config]
    if args.points > 0:
        w = w.scaled(N=args.points, name=f"{w.name}_reduced_N{args.points}")
    if args.metric != "euclid" and (w.host_resident or args.sharded or args.impl == "reference"):
        print("bench.py: --metric dot/cosine runs on device-resident workloads with --impl fkm "
              "only (the host-streamed and sharded runs are Euclidean)", file=sys.stderr)
        return 2
    if args.impl == "reference":
        return run_reference(args, w)
    if w.host_resident:
        return run_host(args, w)
    if args.sharded:
        return run_sharded(args, w)

    import torch
    import exact_means_clustering_b200 as fkm

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    # per rank: its own batch of problems (weak scaling)
    wr = rank_workload(w, rank)
    x = datagen.points(wr)
    c0 = datagen.init_centroids(x, datagen.init_indices(wr), wr.dtype)
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[wr.dtype]
    xh = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16) if wr.dtype == "bf16"
          else torch.from_numpy(x)).pin_memory()
    ch = torch.from_numpy(c0).pin_memory()
    dev = torch.device("cuda", local)
    xt = xh.to(dev)
    c0t = ch.to(dev)
    B, N, D, K = wr.B, wr.N, wr.D, wr.K
    ids = torch.empty(B, N, dtype=torch.int32, device=dev)
    centers = torch.empty(B, K, D, dtype=torch.float32, device=dev)
    counts = torch.empty(B, K, dtype=torch.int32, device=dev)
    inertia = torch.empty(B, dtype=torch.float64, device=dev)
    ws = fkm.workspace(fkm.fkm_workspace_size(B, N, K, D, tdt), dev)
    stream = torch.cuda.current_stream(dev)

    def lloyd(xs, cs):
        if args.metric == "euclid":
            return fkm.fkm_lloyd(xs, cs, wr.iters, wr.tol, ids, centers, counts, inertia, ws=ws,
                                 stream=stream)
        return fkm.fkm_lloyd_metric(xs, cs, wr.iters, wr.tol, ids, centers, counts, args.metric,
                                    inertia, ws=ws, stream=stream)

    def step():
        return lloyd(xt, c0t)

    def barrier():
        if dist is not None:
            dist.barrier()

    fkm.fkm_profile(True)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    fkm.fkm_profile_read(reset=True)
    launches0 = fkm.fkm_kernel_launches()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    iters_done = 0
    with ClockSampler(local) as clk:
        time.sleep(0.3)  # let the sampler start
        barrier()
        torch.cuda.synchronize(dev)
        h0 = time.time()
        e0.record(stream)
        for _ in range(args.steps):
            iters_done += step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        clk.window(h0, time.time())
        barrier()
    launches = fkm.fkm_kernel_launches() - launches0
    prof = fkm.fkm_profile_read(reset=True)
    fkm.fkm_profile(False)
    t_max, total_iters = over_ranks(torch, dist, dev, e0.elapsed_time(e1), iters_done)
    value = total_iters / (t_max / 1e3)

    # --- per-stage rates from the events recorded inside the timed region
    it = max(prof["iterations"], 1)
    t_assign = prof["assign"] / it / 1e3
    t_update = (prof["argsort"] + prof["segsum"] + prof["finalize"]) / it / 1e3
    peaks, peak_src = load_peaks()
    tflops = assign_flops(wr) / t_assign / 1e12 if t_assign > 0 else None
    upd_gbs = update_bytes(wr) / t_update / 1e9 if t_update > 0 else None
    # the assign kernel runs at full clock between the update's memory-bound
    # kernels, so it is held to the burst GEMM peak, the stricter denominator
    peak_t = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    if wr.dtype == "f32":
        # split-bf16: the algorithmic FLOPs run as three bf16 products on the tensor cores
        bound_note = "fp32 points as split bf16 (3 tensor-core products per algorithmic one)"
    else:
        bound_note = "bf16/fp16 operands, fp32 accumulate"
    traffic = assign_traffic(wr.name)
    # 16-bit points with rows of at most 256 elements run on CTA pairs
    kname = "assign_pair_kernel" if wr.dtype != "f32" and wr.D <= 256 else "assign_tc_kernel"
    roofline = {"bound": "tensor", "kernel": kname, "achieved": tflops,
                "peak": peak_t, "unit": "TFLOP/s",
                "frac": (tflops / peak_t) if tflops else None, "traffic": traffic,
                "peak_source": f"{peak_src} (bf16 burst, MEASURED_PEAKS.json)",
                "note": bound_note,
                "flops_per_launch": assign_flops(wr),
                "launch_ms": t_assign * 1e3}

    line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": t_max / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": wr.dtype, "data": "synthetic",
            "config": dict(workload_config(wr), **({} if args.metric == "euclid"
                                                    else {"metric": args.metric})),
            "roofline": roofline,
            "stages_ms_per_iter": {k: prof[k] / it for k in fkm.STAGES},
            "assign_tflops": tflops,
            "update_gbs": upd_gbs,
            "update_frac_of_hbm": (upd_gbs / peaks["hbm_gbs"]) if upd_gbs else None,
            "iteration_roofline_frac": iteration_frac(wr, t_max / max(total_iters / world, 1),
                                                      peaks),
            "gpu_launches": int(launches),
            "clocks": clk.summary()}

    # --- the pages' comparison point (not the method): materialised distances
    # + argmin read-back, and the scatter-atomic update, against the fused
    # calls on the same inputs (outside the timed region)
    if not args.no_comparison and args.metric == "euclid":
        line["comparison"] = comparison(fkm, torch, wr, xt, c0t, ws, stream, dev)

    # --- end to end through the C ABI with host buffers.  Every step copies its
    # points and initial centroids from pinned host memory and reads its
    # results back; the copy of step k+1 runs on a copy stream while step k
    # computes (two device buffers), as a service running back-to-back
    # problems would do.
    if not args.no_e2e:
        ids_h = torch.empty(B, N, dtype=torch.int32).pin_memory()
        cen_h = torch.empty(B, K, D, dtype=torch.float32).pin_memory()
        cnt_h = torch.empty(B, K, dtype=torch.int32).pin_memory()
        ine_h = torch.empty(B, dtype=torch.float64).pin_memory()
        x_e = [torch.empty_like(xt), torch.empty_like(xt)]
        c_e = [torch.empty_like(c0t), torch.empty_like(c0t)]
        copy_stream = torch.cuda.Stream(dev)
        ready = [torch.cuda.Event(), torch.cuda.Event()]
        done = [torch.cuda.Event(), torch.cuda.Event()]
        for ev in done:
            ev.record(stream)

        def issue_copy(k):
            s = k % 2
            copy_stream.wait_event(done[s])   # step k-2 is finished with buffer s
            with torch.cuda.stream(copy_stream):
                x_e[s].copy_(xh, non_blocking=True)
                c_e[s].copy_(ch, non_blocking=True)
                ready[s].record(copy_stream)

        def e2e_step(k):
            s = k % 2
            stream.wait_event(ready[s])
            n_it = lloyd(x_e[s], c_e[s])
            done[s].record(stream)
            ids_h.copy_(ids, non_blocking=True)
            cen_h.copy_(centers, non_blocking=True)
            cnt_h.copy_(counts, non_blocking=True)
            ine_h.copy_(inertia, non_blocking=True)
            return n_it

        def e2e_run(steps):
            issue_copy(0)
            n = 0
            for k in range(steps):
                if k + 1 < steps:
                    issue_copy(k + 1)
                n += e2e_step(k)
            return n

        e2e_run(max(args.warmup, 1))
        torch.cuda.synchronize(dev)
        barrier()
        e0.record(stream)
        copy_stream.wait_event(e0)
        n_e = e2e_run(args.steps)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        t_e, n_e = over_ranks(torch, dist, dev, e0.elapsed_time(e1), n_e)
        line["e2e"] = {"value": n_e / (t_e / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": int(xh.numel() * xh.element_size()
                                                 + ch.numel() * ch.element_size()),
                       "d2h_bytes_per_step": int(ids_h.numel() * 4 + cen_h.numel() * 4
                                                 + cnt_h.numel() * 4 + ine_h.numel() * 8)}

    # --- the oracle on this host's cores (rank 0, one GPU only)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        value_c, desc = cpu_baseline(wr, args.oracle_iters, metric=args.metric)
        line["cpu_baseline"] = {"value": value_c, "unit": UNIT, "cores": cpu_cores(),
                                "kind": "oracle", "sample": desc}

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))
    return 0


if __name__ == "__main__":
    sys.exit(main())
