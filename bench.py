#!/usr/bin/env python
"""Benchmark of the fused diagonal-GMM EM step on B200.

One step = one full EM iteration through the C ABI (gmm_em_step: parameter
prep, the fused E-step + statistics pass over all N rows, the deterministic
reduction and the M-step) on the resident synthetic workload.  Default
workload: gauss4096 (N=1e7, D=96, K=4096, fp32 X), the largest single-GPU
configuration by N*K*D; --workload picks any of the five.

Prints ONE JSON line (rank 0).  Timing: W untimed warm-up steps, then exactly
K steps between a barrier + synchronize on both sides, timed with CUDA events
on the stream the library launches on; X (3.84 GB for gauss4096) is larger than
the 126 MB L2, so no flush is needed between steps (a 256 MB buffer is zeroed
between steps for the one workload, gauss8, whose X fits in L2).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (one process per GPU under torchrun) the run is row-sharded weak
scaling: every rank holds its own block of N rows of the same data stream, and
one step is gmm_estep_stats on each rank, an NCCL all-gather of the fp64
statistics and gmm_mstep (which sums the shards in rank order) on every rank.

--impl reference times the CPU oracle (plain fp64 EM) on the host cores, on a
bounded row sample of the same workload per step, scaled to the same unit.
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
sys.path.insert(0, ROOT)

from soft_clustering_em_b200 import synth  # noqa: E402

METRIC = "EM iterations/s and fused E+M N·K·D/s on 1 B200, % of roofline"
UNIT = "EM iterations/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# N*K exponentials at 16 MUFU ex2 per clock per SM, 148 SMs, 1965 MHz: a floor
# for the normalisation, reported beside the tensor roofline
MUFU_EXP_PER_S = 16 * 148 * 1.965e9
FUSED_SOURCES = ["soft_clustering_em_b200/csrc/tc_em.cuh",
                 "soft_clustering_em_b200/csrc/sm100_prims.cuh",
                 "soft_clustering_em_b200/csrc/common.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="gauss4096", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--rows", type=int, default=0, help="override N (0: the workload's N)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--ivf", action="store_true",
                    help="time the IVF list build (gmm_ivf_build) instead of the EM step")
    ap.add_argument("--ivf-tau", type=float, default=0.1)
    ap.add_argument("--topm", action="store_true",
                    help="time the top-2 assignment (gmm_assign_topm) instead of the EM step")
    ap.add_argument("--host-stream", action="store_true",
                    help="time EM with X in pinned host memory (gmm_em_step_host)")
    ap.add_argument("--chunk-rows", type=int, default=1 << 17)
    ap.add_argument("--all", action="store_true",
                    help="one GPU: run every workload in turn (a process each), one JSON line "
                         "per workload")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def measure_tf32_tflops(dev):
    """Dense TF32 rate of this GPU: torch fp32 matmul with TF32 allowed, 8192^3,
    best of 10 after warm-up, CUDA events (a measured TF32 figure beside the bf16 peak)."""
    import torch

    n = 8192
    a = torch.randn(n, n, device=dev)
    b = torch.randn(n, n, device=dev)
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        for _ in range(3):
            torch.matmul(a, b)
        best = float("inf")
        for _ in range(10):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev
    del a, b
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / (best * 1e-3) / 1e12


def fused_source_sha():
    h = hashlib.sha256()
    for f in FUSED_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """Per-launch DRAM bytes of the fused kernel from a committed ncu summary,
    or None if there is none for the current kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    e = d.get(workload)
    if not e or e.get("source_sha") != fused_source_sha():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms during a region."""

    Q = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9 or (self.uuid and f[0] != self.uuid):
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        loaded = [s for s, p in zip(sm, power) if p > 300.0] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm), "samples_under_load": len(loaded)}


def dist_setup(args):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def oracle_sample(wl, X_np, theta, n):
    """One teacher-forced oracle EM step on the first n rows; returns (seconds, result)."""
    import oracle

    X64 = synth.x_as_f64(wl, X_np[:n])
    t0 = time.perf_counter()
    res = oracle.em_step(X64, *theta, var_floor=wl.var_floor)
    return time.perf_counter() - t0, res


def size_sample(wl, X_np, theta, seconds):
    """Rows of an oracle sample that takes about `seconds` on this host."""
    n0 = min(len(X_np), max(256, 2_000_000 // max(1, wl.K * wl.D // 64)))
    t0, _ = oracle_sample(wl, X_np, theta, n0)
    n = int(n0 * seconds / max(t0, 1e-3))
    return max(n0, min(len(X_np), n))


def reference_arm(args):
    """The CPU oracle on the host cores (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    import oracle

    wl = synth.WORKLOADS[args.workload]
    N = args.rows or wl.N
    X_np, _ = synth.make_data(wl, N)
    mode = 0 if wl.var_init == "one" else 1
    theta = oracle.init_seeded(synth.x_as_f64(wl, X_np), wl.init_seed, wl.K, mode, wl.var_floor)
    per_step = min(10.0, 150.0 / max(1, args.steps + args.warmup))
    n = size_sample(wl, X_np, theta, per_step)
    for _ in range(args.warmup):
        oracle_sample(wl, X_np, theta, n)
    t = 0.0
    for _ in range(args.steps):
        dt, _ = oracle_sample(wl, X_np, theta, n)
        t += dt
    sec_per_iter = (t / args.steps) * (N / n)
    value = 1.0 / sec_per_iter
    sample = (f"first {n} of {N} rows, one EM step per timed step from the data-variance init, "
              f"time scaled by N/n = {N / n:.1f}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec_per_iter * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, N),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def workload_config(wl, N):
    xb = N * wl.D * (2 if wl.dtype == "bf16" else 4)
    return {"workload": wl.name, "N": N, "D": wl.D, "K": wl.K, "x_dtype": wl.dtype,
            "x_bytes": xb, "em_iters_per_run": wl.iters,
            "l2": "inputs larger than L2 (no flush)" if xb > 126e6 else "L2 flushed between steps"}


def ours(args):
    import torch
    import torch.distributed as dist

    from soft_clustering_em_b200 import gmm as G
    from soft_clustering_em_b200 import sharded

    world, rank, local = dist_setup(args)
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[args.workload]
    N = args.rows or wl.N  # rows per rank
    N_total = N * world
    X_np, _ = synth.make_data(wl, N, start=rank * N)
    Xh = torch.from_numpy(X_np.view(np.int16) if wl.dtype == "bf16" else X_np)
    if wl.dtype == "bf16":
        Xh = Xh.view(torch.bfloat16)
    Xh = Xh.pin_memory()
    Xd = Xh.to(dev, non_blocking=False)
    p = G.problem_for(Xd, wl.K, wl.var_floor)
    ws = G.workspace(p, dev)
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    w, mu, var = G.gmm_init(Xd, wl.init_seed, wl.K, mode, wl.var_floor, ws=ws)
    if world > 1:
        sharded.broadcast_params(w, mu, var)  # every rank starts from rank 0's parameters
    ll = torch.zeros(1, dtype=torch.float64, device=dev)
    stream = torch.cuda.current_stream(dev)
    theta0 = (w.clone(), mu.clone(), var.clone())
    flush = None if Xd.numel() * Xd.element_size() > 126e6 else torch.empty(
        256 << 20, dtype=torch.uint8, device=dev)
    stats = torch.empty(G.stats_size(wl.K, wl.D), dtype=torch.float64, device=dev)
    xdt = G.xdtype_of(Xd)

    plan = G.gmm_plan(p)
    # a problem whose fit runs in one launch is timed as gmm_fit over the
    # workload's iterations per step; every other as one gmm_em_step per step
    iters_per_step = wl.iters if (world == 1 and plan["fit_one_launch"]) else 1

    def step(X):
        if iters_per_step > 1:
            G.gmm_fit(X, w, mu, var, iters_per_step, wl.var_floor, ws=ws)
        elif world == 1:
            G.gmm_em_step(X, w, mu, var, ll, wl.var_floor, ws=ws)
        else:
            G.gmm_estep_stats(X, w, mu, var, stats, wl.var_floor, ws=ws)
            gathered = sharded.gather_stats(stats)
            G.gmm_mstep(gathered, N_total, w, mu, var, ll, wl.var_floor, xdt)

    def barrier():
        if world > 1:
            dist.barrier(device_ids=[local])

    def max_over_ranks(x):
        if world == 1:
            return x
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    tf32 = measure_tf32_tflops(dev) if rank == 0 else None
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None)
    time.sleep(0.5)
    for _ in range(max(3, args.warmup)):
        step(Xd)
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in starts + stops:
        e.record(stream)
    torch.cuda.synchronize(dev)
    launches0 = G.gmm_launch_count()
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    t_begin.record(stream)
    for i in range(args.steps):
        G.gmm_trace_fused(starts[i], stops[i])
        step(Xd)
        if flush is not None:
            flush.zero_()
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    launches = G.gmm_launch_count() - launches0
    G.gmm_trace_fused(None, None)
    clocks = sampler.stop()
    total_ms = max_over_ranks(t_begin.elapsed_time(t_end))
    fused_ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    rc, flags = G.gmm_device_status(ws)
    if rc != 0:
        raise SystemExit(f"device status {G.status_string(rc)} flags={flags:#x}")

    # ---- end to end: X from pinned host memory every step -------------------
    # One GPU: the public call for host-resident data, gmm_em_step_host. Every
    # step streams all of X over PCIe in chunks (copy stream), overlapping the
    # previous chunk's E-step, and the step's LL is read back to pinned host
    # memory. Several GPUs: each rank's step is gmm_estep_stats + all-gather +
    # gmm_mstep, so X and the parameters are copied per step on a copy stream
    # into one of two device buffers, overlapping the previous step.
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    pbytes = (w.numel() + mu.numel() + var.numel()) * 4
    if world == 1:
        chunk_rows = min(N, args.chunk_rows)
        staging = torch.empty(G.gmm_host_staging_size(p, chunk_rows), dtype=torch.uint8,
                              device=dev)
        cs = G.copy_stream_for(dev)
        ll_hist = torch.zeros(args.steps, dtype=torch.float64).pin_memory()
        G.gmm_em_step_host(Xh, w, mu, var, ll, chunk_rows, wl.var_floor, staging=staging,
                           ws=ws)  # warm-up, untimed
        for t, t0 in zip((w, mu, var), theta0):
            t.copy_(t0)
        torch.cuda.synchronize(dev)
        e0.record(stream)
        cs.wait_event(e0)
        for i in range(args.steps):
            G.gmm_em_step_host(Xh, w, mu, var, ll, chunk_rows, wl.var_floor, staging=staging,
                               ws=ws)
            ll_hist[i].copy_(ll[0], non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / args.steps
        h2d = Xh.numel() * Xh.element_size()
        d2h = 8
        pipeline = (f"gmm_em_step_host: X streamed from pinned host memory in chunks of "
                    f"{chunk_rows} rows on a copy stream, overlapping the E-step; LL read back")
    else:
        w_h = theta0[0].cpu().pin_memory()
        mu_h = theta0[1].cpu().pin_memory()
        var_h = theta0[2].cpu().pin_memory()
        ll_h = torch.zeros(1, dtype=torch.float64).pin_memory()
        xbuf = [torch.empty_like(Xd), torch.empty_like(Xd)]
        cstream = torch.cuda.Stream(dev)
        copied = [torch.cuda.Event(), torch.cuda.Event()]
        used = [torch.cuda.Event(), torch.cuda.Event()]

        def issue_copy(i):
            b = i % 2
            if i >= 2:
                cstream.wait_event(used[b])  # the step that read this buffer is done
            with torch.cuda.stream(cstream):
                xbuf[b].copy_(Xh, non_blocking=True)
            copied[b].record(cstream)

        barrier()
        torch.cuda.synchronize(dev)
        e0.record(stream)
        cstream.wait_event(e0)
        issue_copy(0)
        for i in range(args.steps):
            b = i % 2
            if i + 1 < args.steps:
                issue_copy(i + 1)
            stream.wait_event(copied[b])
            w.copy_(w_h, non_blocking=True)
            mu.copy_(mu_h, non_blocking=True)
            var.copy_(var_h, non_blocking=True)
            step(xbuf[b])
            used[b].record(stream)
            w_h.copy_(w, non_blocking=True)
            mu_h.copy_(mu, non_blocking=True)
            var_h.copy_(var, non_blocking=True)
            ll_h.copy_(ll, non_blocking=True)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1)) / args.steps
        h2d = (Xd.numel() * Xd.element_size() + pbytes) * world
        d2h = (pbytes + 8) * world
        pipeline = ("each step's X and parameters copied from pinned host memory on a second "
                    "stream, double-buffered, overlapping the previous step; parameters and LL "
                    "read back")

    ms = total_ms / args.steps
    # whole-job throughput in workload iterations: rows of all ranks per second / workload N
    value = (N_total / wl.N) * iters_per_step * 1e3 / ms
    nkd = float(N) * wl.K * wl.D * iters_per_step  # per timed step (and per fused launch)
    pk, pk_kind = peaks()
    sustained = total_ms >= 1000.0
    peak = pk["bf16_tflops_sustained" if sustained else "bf16_tflops"]
    fused_avg = statistics.mean(fused_ms)
    achieved = 8.0 * nkd / (fused_avg * 1e-3) / 1e12
    traffic = ncu_traffic(wl.name)
    cfg = workload_config(wl, N)
    cfg["em_iters_per_timed_step"] = iters_per_step
    if world > 1:
        cfg.update({"ranks": world, "rows_per_rank": N, "exchange": "NCCL all-gather of fp64 "
                    "statistics, M-step sums shards in rank order"})
    if iters_per_step > 1:
        dtype = "f32"
        precision = ("fp32 direct form on the CUDA cores, fp64 statistics exchanged over "
                     "distributed shared memory, M-step on chip")
        kernel = (f"small_fit_kernel: all {iters_per_step} iterations of gmm_fit in one launch "
                  "of one cluster, X resident in shared memory")
    elif plan["tensor_cores"]:
        dtype = "f16"
        precision = ("fp16 hi/lo split operands on the tensor cores (tcgen05 kind::f16), fp32 "
                     "accumulation in tensor memory, fp64 reductions and M-step")
        if plan["groups"] == 1:
            kernel = (f"tc_fused_kernel: one fused pass, {plan['cluster_ctas']}-CTA clusters "
                      "exchanging each row's (max, sum-exp) over DSMEM")
        else:
            kernel = (f"tc_fused_kernel, {plan['groups']} component groups of "
                      f"{plan['cluster_ctas']}-CTA clusters: per chunk of "
                      f"{plan['chunk_rows']} rows tc_convert_kernel (features to HBM), the "
                      "partial (max, sum-exp) pass and the statistics pass, features TMA-loaded")
    else:
        raise SystemExit(f"{wl.name}: no tensor-core plan for this shape")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": dtype, "precision": precision,
        "data": "synthetic", "config": cfg,
        "nkd_per_s": nkd * world * 1e3 / ms,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": kernel, "plan": plan,
                     "algorithmic": "8*N*K*D flop per fused pass (all its launches)",
                     "fused_ms_per_launch": fused_avg,
                     "tf32_tflops_measured": tf32,
                     "frac_vs_tf32_measured": achieved / tf32 if tf32 else None,
                     "mufu_exp_floor_ms": N * wl.K / MUFU_EXP_PER_S * 1e3,
                     "peak_source": f"{pk_kind} bf16 dense "
                                    f"{'sustained' if sustained else 'burst'} "
                                    "(fp16 runs at the bf16 rate)"},
        "e2e": {"value": (N_total / wl.N) * 1e3 / e2e_ms, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "pipeline": pipeline},
        "gpu_launches": launches,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle

        theta = tuple(t.double().cpu().numpy() for t in theta0)
        n = size_sample(wl, X_np, theta, args.cpu_seconds)
        t_cpu, ref = oracle_sample(wl, X_np, theta, n)
        line["cpu_baseline"] = {
            "value": 1.0 / (t_cpu * N / n), "unit": UNIT, "cores": oracle.num_threads(),
            "kind": "oracle",
            "sample": f"first {n} of {N} rows, one EM step from the bench's starting "
                      f"parameters ({t_cpu:.1f} s), time scaled by N/n"}
        # parity on the same sample, same starting parameters, same kernels
        from oracle import compare

        ws_s = G.workspace(G.problem_for(Xd[:n], wl.K, wl.var_floor), dev)
        tw, tmu, tvar = (t.clone() for t in theta0)
        lls = torch.zeros(1, dtype=torch.float64, device=dev)
        G.gmm_em_step(Xd[:n], tw, tmu, tvar, lls, wl.var_floor, ws=ws_s)
        got = (tw.double().cpu().numpy(), tmu.double().cpu().numpy(),
               tvar.double().cpu().numpy(), lls.item())
        rep = compare.compare_step(ref[:4], got, ref[4])
        line["parity"] = {"rows": n, **{k: rep[k] for k in ("ok", "w", "mu", "var", "ll")}}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier()
        dist.destroy_process_group()


def ivf_bench(args):
    """One GPU: the IVF list build on a seeded top-m assignment of the bf16stream size.

    A step is one gmm_ivf_build (counter reset, count pass, two scans, fill pass)
    over N points with m = 2 candidates each.  The inputs (N x m int32 + float32)
    exceed L2, so no flush is needed.  Algorithmic bytes per build: the
    assignment read once, the ids and offsets written once.
    """
    import torch

    from oracle import ivf as ivf_oracle
    from soft_clustering_em_b200 import gmm as G

    wl = synth.WORKLOADS["bf16stream"]
    N, K, m, tau = args.rows or wl.N, wl.K, wl.topm, args.ivf_tau
    dev = torch.device("cuda", 0)
    idx, resp = synth.topm_inputs(N, K, m, seed=wl.init_seed)
    idx_d, resp_d = torch.from_numpy(idx).to(dev), torch.from_numpy(resp).to(dev)
    ws = torch.zeros(G.gmm_ivf_workspace_size(N, K), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None)
    for _ in range(max(3, args.warmup)):
        offsets, ids = G.gmm_ivf_build(idx_d, resp_d, K, tau, ws=ws)
    torch.cuda.synchronize(dev)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    stops = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    launches0 = G.gmm_launch_count()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        starts[i].record(stream)
        offsets, ids = G.gmm_ivf_build(idx_d, resp_d, K, tau, ws=ws)
        stops[i].record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gmm_launch_count() - launches0
    clocks = sampler.stop()
    ms = [a.elapsed_time(b) for a, b in zip(starts, stops)]
    total_ms = sum(ms)
    rc, flags = G.gmm_device_status(ws)
    total = int(offsets[-1].item())
    algo_bytes = N * m * 8 + total * 8 + (K + 1) * 8
    pk, kind = peaks()
    achieved = algo_bytes / (total_ms / args.steps * 1e-3) / 1e9
    # oracle on a bounded sample of the same assignment, on the host
    n_s = min(N, 10_000_000)
    t0 = time.perf_counter()
    ivf_oracle.ivf_lists(idx[:n_s], resp[:n_s], K, tau)
    cpu_s = time.perf_counter() - t0
    line = {
        "metric": "IVF list build from a top-2 assignment, points/s on 1 B200",
        "value": N * args.steps / (total_ms * 1e-3), "unit": "points/s", "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": total_ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int64", "data": "synthetic",
        "config": {"workload": "ivf_build", "N": N, "K": K, "m": m, "tau": tau,
                   "entries": total, "list_inflation": total / N,
                   "l2": "inputs larger than L2 (no flush)"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / pk["hbm_gbs"], "traffic": None,
                     "peak_kind": kind, "algorithmic_bytes_per_build": algo_bytes},
        "cpu_baseline": {"value": n_s / cpu_s, "unit": "points/s", "cores": 1,
                         "kind": "oracle", "sample": f"first {n_s} points of the assignment"},
        "gpu_launches": launches, "device_status": rc, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def topm_bench(args):
    """One GPU: the top-m assignment (m = 2) of a workload's rows after a short fit.

    A step is one gmm_assign_topm: the E-step on the tensor cores (the groups'
    partial pass first where K spans several clusters), each (CTA, column half)'s
    best candidates, then the direct-form refinement of each row's candidates.
    The parameters come from the seeded init and 3 EM steps.  Algorithmic work:
    the E-step's 4*N*K*D flop.
    """
    import torch

    from soft_clustering_em_b200 import gmm as G

    wl = synth.WORKLOADS[args.workload]
    N = args.rows or wl.N
    dev = torch.device("cuda", 0)
    X_np, _ = synth.make_data(wl, N)
    Xd = torch.from_numpy(X_np.view(np.int16) if wl.dtype == "bf16" else X_np)
    if wl.dtype == "bf16":
        Xd = Xd.view(torch.bfloat16)
    Xd = Xd.to(dev)
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    p = G.problem_for(Xd, wl.K, wl.var_floor)
    ws = G.workspace(p, dev)
    w, mu, var = G.gmm_init(Xd, wl.init_seed, wl.K, mode, wl.var_floor, ws=ws)
    ll = torch.zeros(1, dtype=torch.float64, device=dev)
    for _ in range(3):
        G.gmm_em_step(Xd, w, mu, var, ll, wl.var_floor, ws=ws)
    m = 2
    stream = torch.cuda.current_stream(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None)
    for _ in range(max(3, args.warmup)):
        G.gmm_assign_topm(Xd, w, mu, var, m, wl.var_floor, ws=ws)
    torch.cuda.synchronize(dev)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = G.gmm_launch_count()
    start.record(stream)
    for _ in range(args.steps):
        G.gmm_assign_topm(Xd, w, mu, var, m, wl.var_floor, ws=ws)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gmm_launch_count() - launches0
    clocks = sampler.stop()
    ms = start.elapsed_time(stop) / args.steps
    rc, flags = G.gmm_device_status(ws)
    pk, kind = peaks()
    achieved = 4.0 * N * wl.K * wl.D / (ms * 1e-3) / 1e12
    line = {
        "metric": "top-2 assignment, points/s on 1 B200", "value": N / (ms * 1e-3),
        "unit": "points/s", "n_gpus": 1, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": dict(workload_config(wl, N), m=m, params="seeded init + 3 EM steps"),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": achieved / pk["bf16_tflops"], "traffic": None,
                     "algorithmic": "4*N*K*D flop (the E-step)", "peak_kind": kind},
        "gpu_launches": launches, "device_status": rc, "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def host_stream_bench(args):
    """One GPU: EM iterations with X in pinned host memory, streamed in chunks.

    A step is one gmm_em_step_host: every chunk of X crosses PCIe inside the
    step (copy stream) while the previous chunk's E-step runs, then one M-step;
    the step's LL is read back to pinned host memory.  Timed with CUDA events on
    the compute stream; the copy stream waits on the start event.
    """
    import torch

    from soft_clustering_em_b200 import gmm as G

    wl = synth.WORKLOADS[args.workload]
    N = args.rows or wl.N
    dev = torch.device("cuda", 0)
    X_np, _ = synth.make_data(wl, N)
    Xh = torch.from_numpy(X_np.view(np.int16) if wl.dtype == "bf16" else X_np)
    if wl.dtype == "bf16":
        Xh = Xh.view(torch.bfloat16)
    Xh = Xh.pin_memory()
    Xd = Xh.to(dev)
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    p = G.problem_for(Xh, wl.K, wl.var_floor)
    ws = G.workspace(p, dev)
    w, mu, var = G.gmm_init(Xd, wl.init_seed, wl.K, mode,
                            wl.var_floor, ws=ws)
    del Xd  # from here on X lives only in host memory
    torch.cuda.empty_cache()
    staging = torch.empty(G.gmm_host_staging_size(p, args.chunk_rows), dtype=torch.uint8,
                          device=dev)
    ll = torch.zeros(1, dtype=torch.float64, device=dev)
    ll_host = torch.zeros(args.steps, dtype=torch.float64).pin_memory()
    stream = torch.cuda.current_stream(dev)
    cs = G.copy_stream_for(dev)
    props = torch.cuda.get_device_properties(dev)
    sampler = ClockSampler(f"GPU-{props.uuid}" if getattr(props, "uuid", None) else None)
    for _ in range(max(3, args.warmup)):
        G.gmm_em_step_host(Xh, w, mu, var, ll, args.chunk_rows, wl.var_floor, staging=staging,
                           ws=ws)
    torch.cuda.synchronize(dev)
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = G.gmm_launch_count()
    start.record(stream)
    cs.wait_event(start)
    for i in range(args.steps):
        G.gmm_em_step_host(Xh, w, mu, var, ll, args.chunk_rows, wl.var_floor, staging=staging,
                           ws=ws)
        ll_host[i].copy_(ll[0], non_blocking=True)
    stop.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gmm_launch_count() - launches0
    clocks = sampler.stop()
    ms = start.elapsed_time(stop)
    rc, flags = G.gmm_device_status(ws)
    h2d = N * wl.D * (2 if wl.dtype == "bf16" else 4)
    line = {
        "metric": "EM iterations/s with X streamed from pinned host memory (gmm_em_step_host)",
        "value": args.steps / (ms * 1e-3), "unit": "EM iterations/s", "n_gpus": 1,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": dict(workload_config(wl, N), chunk_rows=args.chunk_rows,
                       l2="X crosses PCIe every step"),
        "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": 8,
        "h2d_gbs": h2d * args.steps / (ms * 1e-3) / 1e9,
        "gpu_launches": launches, "device_status": rc, "ll_last": float(ll_host[-1]),
        "clocks": clocks,
    }
    print(json.dumps(line), flush=True)


def all_workloads(args):
    """One line per workload, each from its own process (bench.py --workload W)."""
    rc = 0
    for name in sorted(synth.WORKLOADS):
        cmd = [sys.executable, os.path.abspath(__file__), "--workload", name,
               "--steps", str(args.steps), "--warmup", str(args.warmup)]
        if args.no_cpu_baseline:
            cmd.append("--no-cpu-baseline")
        r = subprocess.run(cmd, capture_output=True, text=True)
        lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
        if r.returncode != 0 or not lines:
            rc = r.returncode or 1
            print(json.dumps({"workload": name, "error": (r.stderr.strip().splitlines() or
                                                          ["no output"])[-1]}), flush=True)
        else:
            print(lines[-1], flush=True)
    return rc


def main():
    args = parse()
    if args.all:
        raise SystemExit(all_workloads(args))
    if args.impl == "reference":
        reference_arm(args)
        return
    if args.ivf:
        ivf_bench(args)
        return
    if args.host_stream:
        host_stream_bench(args)
        return
    if args.topm:
        topm_bench(args)
        return
    ours(args)


if __name__ == "__main__":
    main()
