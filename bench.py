#!/usr/bin/env python
"""Benchmark of the W4A16 group-wise GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload (one step): the decode projection K = N = 4096, G = 128, run at M = 1
and at M = 16 (two GEMM launches over the same weight shape). Inputs are seeded
synthetic data with the distributions of the workloads module, resident in HBM
before the timed region. Every launch reads a different one of R rotating
copies of (tiled weights, scales, activations) whose total exceeds twice the
L2 size, so no launch finds its weights in L2.

The timed region replays CUDA graphs of the steps, bracketed by a barrier and
torch.cuda.synchronize(); its time is the max over ranks (CUDA events). One
JSON line goes to stdout on rank 0. `value` is effective HBM GB/s: algorithmic
bytes (packed weights + scales + activations + output, each once) of all ranks'
steps divided by that time. With --gpus N > 1 the ranks are independent
replicas (the path has no exchange step).

`--impl reference` times the CPU oracle (fp64, OpenMP) on a bounded column
sample of the same step, on the host cores; under torchrun only rank 0 runs it.
"""
from __future__ import annotations

import argparse
import csv
import hashlib
import io
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "W4A16 GEMM TFLOPS and effective HBM GB/s vs roofline, M=1..2048 (1 B200)"
K_DIM, N_DIM, G_DIM = 4096, 4096, 128
M_STEP = (1, 16)
WORKLOAD = "decode projection: W4A16 GEMM at M=1 and at M=16, K=4096, N=4096, G=128 (one launch each per step)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
GRAPH_CHUNK = 500


def algorithmic_bytes(M, N, K, G):
    """Packed int4 weights + fp16 scales + fp16 activations + fp16 output, each moved once."""
    return (K * N) // 2 + (-(-K // G)) * N * 2 + M * K * 2 + M * N * 2


def algorithmic_bytes_w8(M, N, K, G):
    """8-bit codes + fp16 scales + fp16 activations + fp16 output, each moved once."""
    return K * N + (-(-K // G)) * N * 2 + M * K * 2 + M * N * 2


def flops(M, N, K):
    return 2 * M * N * K


def step_bytes():
    return sum(algorithmic_bytes(m, N_DIM, K_DIM, G_DIM) for m in M_STEP)


def step_flops():
    return sum(flops(m, N_DIM, K_DIM) for m in M_STEP)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    return dict(FALLBACK_PEAKS, source="fallback")


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi clock and throttle-reason samples taken while the timed region runs."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.out, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.25)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.15)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.out.close()
        rows = list(csv.reader(io.StringIO(open(self.path).read())))
        os.unlink(self.path)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except ValueError:
                continue
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ helpers

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def max_over_ranks(x: float, device=None) -> float:
    """The largest of one float per rank (every rank gets it); the identity without a process group."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, seconds_max: float) -> float:
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return world * units_per_rank / seconds_max


def replay_stats(graph, launches_per_replay, reps):
    """Per-launch device time of `reps` timed replays of a captured graph (CUDA events on
    the replaying stream, one pair per replay): median, p10, p90 and mean, microseconds."""
    import torch
    samples = []
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(reps):
        e0.record()
        graph.replay()
        e1.record()
        e1.synchronize()
        samples.append(e0.elapsed_time(e1) * 1e3 / launches_per_replay)
    samples.sort()
    q = lambda f: samples[min(len(samples) - 1, int(f * len(samples)))]
    return {"median": round(statistics.median(samples), 3), "p10": round(q(0.10), 3), "p90": round(q(0.90), 3),
            "mean": round(sum(samples) / len(samples), 3), "reps": reps, "launches_per_rep": launches_per_replay}


SKINNY_SOURCES = ("w4a16_skinny.cu", "dequant.cuh", "epilogue.cuh", "ptx.cuh")


def skinny_source_digest() -> str:
    """sha256 over the sources that make up the skinny kernel, in a fixed order."""
    h = hashlib.sha256()
    for name in SKINNY_SOURCES:
        with open(os.path.join(ROOT, "weight_only_int4_wise_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def traffic_from_profile():
    """DRAM bytes per launch from the committed ncu summary, if it was taken on the current kernel source."""
    path = os.path.join(ROOT, "profiles", "decode_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_source_sha256") != skinny_source_digest():
        return None
    return d.get("dram_bytes_per_launch")


def oracle_sample(o, case, cols):
    """Packed weights and scales of the first `cols` columns (setup, outside any timing)."""
    return o.pack(np.ascontiguousarray(case.q[:, :cols])), np.ascontiguousarray(case.S[:, :cols])


def oracle_decode_step(o, case, sample):
    """One decode step (M=1 and M=16) of the CPU oracle over a column sample."""
    wp, S = sample
    for m in M_STEP:
        o.gemm(case.A[:m], wp, S, K_DIM, G_DIM)


def sample_bytes(cols):
    return sum(algorithmic_bytes(m, cols, K_DIM, G_DIM) for m in M_STEP)


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(budget_s=12.0):
    """The oracle on the host cores: the full decode step on all cores (the value), and a
    column sample of it on one core (scaled to the step), each the median of a few runs."""
    import oracle
    o = oracle.load()
    case = workloads.dense(16, K_DIM, N_DIM, G_DIM, seed=1)
    wp = o.pack(case.q)

    def timed(step, budget, cap):
        times = []
        t_end = time.perf_counter() + budget
        while True:
            t0 = time.perf_counter()
            step()
            times.append(time.perf_counter() - t0)
            if time.perf_counter() > t_end or len(times) >= cap:
                break
        return statistics.median(times), len(times)

    def full_step():
        for m in M_STEP:
            o.gemm(case.A[:m], wp, case.S, K_DIM, G_DIM)
    t_all, n_all = timed(full_step, budget_s, 20)
    cols = 512
    wp1, S1 = oracle_sample(o, case, cols)

    def one_core_step():
        for m in M_STEP:
            o.gemm(case.A[:m], wp1, S1, K_DIM, G_DIM, threads=1)
    t_one, n_one = timed(one_core_step, budget_s / 2, 5)
    one_value = sample_bytes(cols) / t_one / 1e9
    return {"value": step_bytes() / t_all / 1e9, "unit": "GB/s", "cores": o.threads(), "kind": "oracle",
            "sample": f"full decode step (M=1 and M=16, K=N=4096, G=128), median of {n_all} runs, "
                      f"{t_all * 1e3:.1f} ms per step",
            "one_core": {"value": one_value, "unit": "GB/s", "cores": 1,
                         "sample": f"M=1 and M=16 over the first {cols} of {N_DIM} columns, median of {n_one} "
                                   f"runs, {t_one * 1e3:.1f} ms"},
            "affinity_cores": len(os.sched_getaffinity(0)), "cpu_model": cpu_model()}


# ------------------------------------------------------------------ our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    from weight_only_int4_wise_b200 import build as wbuild
    wbuild.build()
    import weight_only_int4_wise_b200 as w4

    dev = torch.device("cuda", local)
    case = workloads.dense(16, K_DIM, N_DIM, G_DIM, seed=1)
    q = torch.from_numpy(case.q).to(dev)
    _, wt0 = w4.prepare_weights(q)
    S0 = torch.from_numpy(case.S).to(dev)
    A0 = torch.from_numpy(case.A).to(dev)
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20)
    # Weights and scales rotate over copies that together exceed L2 twice, so every
    # launch streams its weights from HBM. The activations come from one buffer,
    # as a decoder layer's input comes from the kernel before it (still in L2);
    # --cold-activations rotates them with the weights instead.
    copy_bytes = wt0.numel() + S0.numel() * 2 + (A0.numel() * 2 if args.cold_activations else 0)
    R = max(3, math.ceil(2 * l2 / copy_bytes) + 1)
    wts = [wt0] + [wt0.clone() for _ in range(R - 1)]
    Ss = [S0] + [S0.clone() for _ in range(R - 1)]
    As = [A0] + [A0.clone() if args.cold_activations else A0 for _ in range(R - 1)]
    C1 = torch.empty((1, N_DIM), dtype=torch.float16, device=dev)
    C16 = torch.empty((16, N_DIM), dtype=torch.float16, device=dev)
    outs = {1: C1, 16: C16}

    def launch(m, r):
        rc = w4.w4a16_gemm(As[r], wts[r], Ss[r], outs[m], m, N_DIM, K_DIM, G_DIM)
        if rc:
            raise RuntimeError(w4.status_string(rc))

    # Weights and scales are prepared once, before any timing, and never written
    # again: declare them static so each GEMM may stream them before the previous
    # kernel on the stream finishes (activations and outputs still wait for it).
    torch.cuda.synchronize()
    w4.w4a16_set_static_weights(True)
    # warm the library's per-device setup outside any capture
    launch(1, 0)
    launch(16, 1)
    torch.cuda.synchronize()
    # Launch forms. By default the library's built-in heuristic, whose choices for
    # these two shapes were made for this alternating M=1 / M=16 sequence. With
    # --tune-headline the autotuner picks each shape's fastest form on its own
    # (back to back over the rotating copies); on B200 its M=16 choice (a deeper
    # ring, 92 KB of shared memory) is faster alone but no longer shares an SM
    # with the M=1 launch, and the alternating step got slower (17.8 against
    # 15.5 us), so it stays opt-in.
    w4.w4a16_clear_tactics()
    tuned = {}
    pinned = dict(tuple(int(x) for x in kv.split("=")) for kv in args.pin_tactics.split(",") if kv)
    for m in M_STEP:
        heur = w4.w4a16_gemm_launch_info(m, N_DIM, K_DIM, G_DIM)[1].as_dict()
        if not args.tune_headline and m not in pinned:
            tuned[f"M={m}"] = {"tactic": 0, "form": heur, "note": "built-in heuristic"}
            continue
        if m in pinned:
            rc = w4.w4a16_set_tactic(m, N_DIM, K_DIM, G_DIM, pinned[m])
            if rc:
                raise RuntimeError(f"tactic {pinned[m]}: {w4.status_string(rc)}")
            tuned[f"M={m}"] = {"tactic": pinned[m], "pinned": True, "heuristic_form": heur,
                               "form": w4.w4a16_gemm_launch_info(m, N_DIM, K_DIM, G_DIM)[1].as_dict()}
            continue
        rc, best, best_us = w4.w4a16_autotune(As[0], wts, Ss, outs[m], m, N_DIM, K_DIM, G_DIM, reps=20)
        if rc:
            raise RuntimeError(f"autotune: {w4.status_string(rc)}")
        tuned[f"M={m}"] = {"tactic": best, "tuner_us": round(best_us, 3), "heuristic_form": heur,
                           "form": w4.w4a16_gemm_launch_info(m, N_DIM, K_DIM, G_DIM)[1].as_dict()}
    launch(1, 0)
    launch(16, 1)
    torch.cuda.synchronize()

    def capture(nsteps, start):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(nsteps):
                launch(1, (2 * (start + i)) % R)
                launch(16, (2 * (start + i) + 1) % R)
        return g

    K, W = args.steps, args.warmup
    chunk = min(K, GRAPH_CHUNK)
    g_main = capture(chunk, 0)
    rem = K % chunk
    g_rem = capture(rem, 0) if rem else None
    for _ in range(max(1, math.ceil(W / chunk))):
        g_main.replay()
    torch.cuda.synchronize()

    sampler = ClockSampler(local)
    if rank == 0:
        sampler.start()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(K // chunk):
        g_main.replay()
    if g_rem is not None:
        g_rem.replay()
    e1.record()
    e1.synchronize()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = e0.elapsed_time(e1)
    clocks = sampler.stop() if rank == 0 else None
    ms_max = max_over_ranks(ms, dev)
    sec = ms_max / 1e3
    value = job_throughput(K * step_bytes(), world, sec) / 1e9
    tflops = job_throughput(K * step_flops(), world, sec) / 1e12

    # Distribution of the step time: 100 timed replays of a 20-step graph (after the timed region).
    g_stats = capture(20, 7)
    for _ in range(3):
        g_stats.replay()
    torch.cuda.synchronize()
    step_stats = replay_stats(g_stats, 20, 100)
    del g_stats

    status = w4.device_status(clear=True)
    if status != w4.OK:
        raise RuntimeError(f"device status after the timed region: {w4.status_string(status)}")

    # End to end through the public C entry point, as a server runs independent
    # batches: every step's activations (1 + 16 rows) come in from pinned host
    # memory and both results go back out to pinned host memory. The copies move
    # E2E_BATCH steps' inputs (or outputs) at a time, on one stream per direction
    # (the two copy engines work at once), into double batch buffers, so that a
    # batch's GEMMs overlap the next batch's copy-in and the previous batch's
    # copy-out. (A copy on another stream that a GEMM must wait for takes that
    # GEMM out of the programmatic-dependent-launch overlap with the kernel before
    # it; per-step copies cost about 4 us per step that way.) E2E_GRAPH_STEPS
    # steps, rotating weight copies as in the timed region, are recorded once
    # into a CUDA graph and replayed. Replays run one after another, so each
    # one starts with a batch copy-in that nothing overlaps and ends with a
    # copy-out: a long graph spreads those two over more steps.
    E2E_BATCH, E2E_GRAPH_STEPS = 8, 128
    rows_step = 1 + 16
    A_step = np.concatenate([case.A[:1], case.A], axis=0)
    A_h = torch.from_numpy(np.concatenate([A_step] * E2E_BATCH, axis=0)).pin_memory()
    C_h = torch.empty((E2E_BATCH * rows_step, N_DIM), dtype=torch.float16).pin_memory()
    A_db = [torch.empty((E2E_BATCH * rows_step, K_DIM), dtype=torch.float16, device=dev) for _ in range(2)]
    C_db = [torch.empty((E2E_BATCH * rows_step, N_DIM), dtype=torch.float16, device=dev) for _ in range(2)]
    K_e2e = min(K, 2048)
    cgemm = w4.load().w4a16_gemm
    wptr = [x.data_ptr() for x in wts]
    sptr = [x.data_ptr() for x in Ss]
    in_stream, out_stream = torch.cuda.Stream(dev), torch.cuda.Stream(dev)  # one copy engine per direction

    def e2e_steps(n):
        comp = torch.cuda.current_stream(dev)
        st = comp.cuda_stream
        nb = n // E2E_BATCH
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]
        ev_back = [torch.cuda.Event() for _ in range(nb)]
        in_stream.wait_stream(comp)
        out_stream.wait_stream(comp)

        def copy_in(j):
            with torch.cuda.stream(in_stream):
                if j >= 2:
                    in_stream.wait_event(ev_out[j - 2])  # batch j-2's GEMMs have read this buffer
                A_db[j % 2].copy_(A_h, non_blocking=True)
                ev_in[j].record(in_stream)

        copy_in(0)
        for j in range(nb):
            b = j % 2
            if j + 1 < nb:
                copy_in(j + 1)
            comp.wait_event(ev_in[j])
            if j >= 2:
                comp.wait_event(ev_back[j - 2])  # batch j-2's results have left this buffer
            for u in range(E2E_BATCH):
                i = j * E2E_BATCH + u
                a0 = A_db[b][u * rows_step:(u + 1) * rows_step]
                c0 = C_db[b][u * rows_step:(u + 1) * rows_step]
                r1, r2 = (2 * i) % R, (2 * i + 1) % R
                if cgemm(a0[:1].data_ptr(), wptr[r1], sptr[r1], c0[:1].data_ptr(), 1, N_DIM, K_DIM, G_DIM, st) or \
                        cgemm(a0[1:].data_ptr(), wptr[r2], sptr[r2], c0[1:].data_ptr(), 16, N_DIM, K_DIM, G_DIM,
                              st):
                    raise RuntimeError("a GEMM call failed in the end-to-end loop")
            ev_out[j].record(comp)
            with torch.cuda.stream(out_stream):
                out_stream.wait_event(ev_out[j])
                C_h.copy_(C_db[b], non_blocking=True)
                ev_back[j].record(out_stream)
        comp.wait_stream(in_stream)
        comp.wait_stream(out_stream)

    e2e_steps(E2E_GRAPH_STEPS)
    torch.cuda.synchronize()
    g_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_e2e):
        e2e_steps(E2E_GRAPH_STEPS)
    reps_e2e = max(1, K_e2e // E2E_GRAPH_STEPS)
    K_e2e = reps_e2e * E2E_GRAPH_STEPS
    for _ in range(3):
        g_e2e.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record()
    for _ in range(reps_e2e):
        g_e2e.replay()
    f1.record()
    f1.synchronize()
    e2e_sec = max_over_ranks(f0.elapsed_time(f1), dev) / 1e3
    e2e = {"value": job_throughput(K_e2e * step_bytes(), world, e2e_sec) / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": sum(m * K_DIM * 2 for m in M_STEP),
           "d2h_bytes_per_step": sum(m * N_DIM * 2 for m in M_STEP), "steps": K_e2e,
           "launch": f"CUDA graph of {E2E_GRAPH_STEPS} steps, replayed: every step's inputs copied in from "
                     f"pinned host memory and its outputs copied out, {E2E_BATCH} steps per copy, on one stream "
                     "per direction with double batch buffers overlapping the neighbouring batches' GEMMs; two "
                     "w4a16_gemm calls per step"}

    only = [x for x in args.configs.split(",") if x] if args.configs else None
    extra = per_config(w4, dev, tune=not args.no_tune, only=only) if (rank == 0 and not args.no_configs) else None
    tactics = tactic_report(w4, dev) if (rank == 0 and not args.no_configs and not only) else None
    peaks = load_peaks()
    achieved = K * step_bytes() / sec / 1e9  # per GPU: every launch in the step is the same kernel
    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": ms_max / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "M": list(M_STEP), "K": K_DIM, "N": N_DIM, "G": G_DIM,
                   "l2": (f"inputs larger than L2: {R} rotating copies of weights+scales+activations "
                          f"({R * copy_bytes / 2 ** 20:.0f} MiB vs {l2 / 2 ** 20:.0f} MiB L2)"
                          if args.cold_activations else
                          f"inputs larger than L2: {R} rotating copies of weights+scales "
                          f"({R * copy_bytes / 2 ** 20:.0f} MiB vs {l2 / 2 ** 20:.0f} MiB L2); the activations "
                          f"come from one buffer, as a layer's input comes from the kernel before it"),
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "static_weights": True,
                   "launch": "CUDA graphs, programmatic dependent launch" +
                             ("; launch forms from the library's autotuner at setup" if args.tune_headline
                              else "; built-in launch heuristic")},
        "tflops": round(tflops, 3),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic_from_profile(),
                     "peak_source": f"{peaks['source']} (copy bandwidth)",
                     "kernel": "w4a16_skinny_kernel (M <= 16: 8- or 16-row token tiles, K split over a cluster)"},
        "e2e": e2e,
        "step_us": dict(step_stats, note="device time per step (one M=1 and one M=16 launch), 100 CUDA-graph "
                                         "replays of 20 steps, after the timed region"),
        "gpu_launches": world * 2 * K,
        "launch": {k: v["form"] for k, v in tuned.items()},
        "tactics_at_setup": tuned,
        "clocks": clocks,
    }
    if rank == 0:
        line["cpu_baseline"] = None if args.no_cpu_baseline else cpu_baseline()
        if extra is not None:
            line["per_config"] = extra
        if tactics is not None:
            line["tactics"] = tactics
        print(json.dumps(line), flush=True)
    del g_main, g_rem
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


TACTIC_SHAPES = [(1, 4096, 4096), (16, 4096, 4096), (8, 4096, 14336), (8, 14336, 4096)]  # (M, K, N), G = 128


def tactic_report(w4, dev):
    """The tactic table on the decode launches and the MLP shapes: the autotuner
    times every valid form the way the headline runs (back-to-back launches in a
    CUDA graph over rotating weight copies larger than L2), then the heuristic's
    form and the tuned one are timed again by the same replay as per_config.
    The headline uses the heuristic; the table is emptied again afterwards."""
    import torch
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20)
    out = {}
    for (M, K, N) in TACTIC_SHAPES:
        G = G_DIM
        c = workloads.dense(M, K, N, G, seed=1)
        _, wt = w4.prepare_weights(torch.from_numpy(c.q).to(dev))
        S = torch.from_numpy(c.S).to(dev)
        A = torch.from_numpy(c.A).to(dev)
        C = torch.empty((M, N), dtype=torch.float16, device=dev)
        per = wt.numel() + S.numel() * 2
        R = max(2, math.ceil(2 * l2 / per) + 1)
        wts = [wt] + [wt.clone() for _ in range(R - 1)]
        Ss = [S] + [S.clone() for _ in range(R - 1)]
        w4.w4a16_clear_tactics()
        heur = w4.w4a16_gemm_launch_info(M, N, K, G)[1].as_dict()
        _, ids = w4.w4a16_get_valid_tactics(M, N, K, G)
        forms = {t: w4.w4a16_tactic_launch_info(M, N, K, G, t)[1].as_dict() for t in ids}
        heur_id = next((t for t in ids if forms[t] == heur), 0)
        rc, best, best_us, times = w4.w4a16_autotune(A, wts, Ss, C, M, N, K, G, reps=20, with_times=True)
        if rc:
            raise RuntimeError(f"autotune: {w4.status_string(rc)}")

        def graph_us():
            def launch(r):
                rc_ = w4.w4a16_gemm(A, wts[r], Ss[r], C, M, N, K, G)
                if rc_:
                    raise RuntimeError(w4.status_string(rc_))
            launch(0)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for i in range(20):
                    launch(i % R)
            for _ in range(3):
                g.replay()
            torch.cuda.synchronize()
            st = replay_stats(g, 20, 50)
            del g
            return st["median"]

        tuned_graph = graph_us()  # the tuned entry is in the table now
        w4.w4a16_clear_tactics()
        heur_graph = graph_us()
        out[f"M={M},K={K},N={N}"] = {
            "tactics": len(ids), "heuristic": heur_id, "heuristic_form": heur,
            "heuristic_tuner_us": round(times[heur_id - 1], 3) if heur_id else None,
            "tuned": best, "tuned_form": forms[best], "tuned_tuner_us": round(best_us, 3),
            "heuristic_graph_us": heur_graph, "tuned_graph_us": tuned_graph,
            "tuner_us_by_tactic": [round(x, 2) for x in times]}
    w4.w4a16_clear_tactics()
    return out


def per_config(w4, dev, tune=True, only=None):
    """Device time per launch for every workload family (context for the headline line).
    Dense W4A16 shapes run the autotuned launch form (unless tune is False)."""
    import torch
    peaks = load_peaks()
    l2 = getattr(torch.cuda.get_device_properties(dev), "L2_cache_size", 126 * 2 ** 20)
    out = {}
    for name, cfg in workloads.CONFIGS.items():
        if name == "tiny" or (only and name not in only):
            continue
        c = workloads.make(name)
        tactic = None
        if cfg["kind"] == "dense":
            _, wt = w4.prepare_weights(torch.from_numpy(c.q).to(dev))
            S = torch.from_numpy(c.S).to(dev)
            A = torch.from_numpy(c.A).to(dev)
            C = torch.empty((c.M, c.N), dtype=torch.float16, device=dev)
            # weights and scales rotate (from HBM); activations and output stay in one buffer
            per = wt.numel() + S.numel() * 2
            R = max(2, math.ceil(2 * l2 / per) + 1)
            bufs = [(wt, S, A, C)] + [(wt.clone(), S.clone(), A, C) for _ in range(R - 1)]
            M, N, K, G = c.M, c.N, c.K, c.G

            def launch(r, b=bufs, M=M, N=N, K=K, G=G):
                wt_, S_, A_, C_ = b[r]
                rc = w4.w4a16_gemm(A_, wt_, S_, C_, M, N, K, G)
                if rc:
                    raise RuntimeError(w4.status_string(rc))
            tactic = 0
            if tune:  # the library's autotuner over the same rotating copies, as a user tunes at setup
                rc, tactic, _ = w4.w4a16_autotune(A, [b[0] for b in bufs], [b[1] for b in bufs], C, M, N, K, G,
                                                  reps=20)
                if rc:
                    raise RuntimeError(f"autotune: {w4.status_string(rc)}")
            fl = flops(M, N, K)
            by = algorithmic_bytes(M, N, K, G)
        elif cfg["kind"] == "dense8":
            wt = w4.repack_w8(torch.from_numpy(c.q).to(dev))
            S = torch.from_numpy(c.S).to(dev)
            A = torch.from_numpy(c.A).to(dev)
            C = torch.empty((c.M, c.N), dtype=torch.float16, device=dev)
            # weights and scales rotate (from HBM); activations and output stay in one buffer
            per = wt.numel() + S.numel() * 2
            R = max(2, math.ceil(2 * l2 / per) + 1)
            bufs = [(wt, S, A, C)] + [(wt.clone(), S.clone(), A, C) for _ in range(R - 1)]
            M, N, K, G = c.M, c.N, c.K, c.G

            def launch(r, b=bufs, M=M, N=N, K=K, G=G):
                wt_, S_, A_, C_ = b[r]
                rc = w4.w8a16_gemm(A_, wt_, S_, C_, M, N, K, G)
                if rc:
                    raise RuntimeError(w4.status_string(rc))
            fl = flops(M, N, K)
            by = algorithmic_bytes_w8(M, N, K, G)
        elif cfg["kind"] == "moe":
            # The whole expert layer: route, dispatch, gather, up (GELU epilogue), down, combine.
            def expert_set(q, S):
                return ([w4.prepare_weights(torch.from_numpy(q[e]).to(dev))[1] for e in range(c.E)],
                        [torch.from_numpy(S[e]).to(dev) for e in range(c.E)])
            up, down = expert_set(c.q_up, c.S_up), expert_set(c.q_down, c.S_down)
            X = torch.from_numpy(c.X).to(dev)
            lg = torch.from_numpy(c.logits).to(dev)
            C = torch.empty((c.tokens, c.H), dtype=torch.float16, device=dev)
            ws = torch.empty(w4.w4a16_moe_workspace_size(c.tokens, c.E, c.top_k, c.H, c.I), dtype=torch.uint8,
                             device=dev)
            per = sum(x.numel() for x in up[0] + down[0]) + sum(x.numel() * 2 for x in up[1] + down[1])
            R = max(2, math.ceil(2 * l2 / per) + 1)
            sets = [(up, down)] + [(([x.clone() for x in up[0]], [x.clone() for x in up[1]]),
                                    ([x.clone() for x in down[0]], [x.clone() for x in down[1]]))
                                   for _ in range(R - 1)]

            def launch(r, sets=sets, X=X, lg=lg, C=C, ws=ws, c=c):
                (wu, su), (wd, sd) = sets[r]
                rc = w4.w4a16_moe_layer(X, lg, wu, su, wd, sd, C, c.tokens, c.E, c.top_k, c.H, c.I, c.G,
                                        w4.ACT_GELU_ERF, ws, ws.numel())
                if rc:
                    raise RuntimeError(w4.status_string(rc))
            rows = c.tokens * c.top_k
            fl = 2 * flops(rows, c.I, c.H)
            # experts that receive rows (the GPU's own routing of these logits)
            ids = torch.empty((c.tokens, c.top_k), dtype=torch.int32, device=dev)
            wts_r = torch.empty((c.tokens, c.top_k), dtype=torch.float32, device=dev)
            if w4.w4a16_moe_route(lg, ids, wts_r, c.tokens, c.E, c.top_k):
                raise RuntimeError("routing failed")
            active = int(torch.unique(ids).numel())
            # the active experts' weights and scales of both projections, activations in
            # and out of each, the gather and the combine
            by = active * (algorithmic_bytes(0, c.I, c.H, c.G) + algorithmic_bytes(0, c.H, c.I, c.G)) + \
                rows * (c.H + c.I) * 2 * 2 + (c.tokens * c.H * 2) * 2 + rows * c.H * 2 * 2
        else:
            wts = [w4.prepare_weights(torch.from_numpy(c.q[e]).to(dev))[1] for e in range(c.E)]
            Ss = [torch.from_numpy(c.S[e]).to(dev) for e in range(c.E)]
            A = torch.from_numpy(c.A).to(dev)
            off = torch.from_numpy(c.offsets).to(dev)
            C = torch.empty((c.total_rows, c.N), dtype=torch.float16, device=dev)
            per = sum(x.numel() for x in wts) + sum(x.numel() * 2 for x in Ss)
            R = max(2, math.ceil(2 * l2 / per) + 1)
            sets = [(wts, Ss)] + [([x.clone() for x in wts], [x.clone() for x in Ss]) for _ in range(R - 1)]

            def launch(r, sets=sets, A=A, off=off, C=C, c=c):
                wts_, Ss_ = sets[r]
                rc = w4.w4a16_grouped_gemm(A, wts_, Ss_, off, C, c.E, c.total_rows, c.N, c.K, c.G)
                if rc:
                    raise RuntimeError(w4.status_string(rc))
            fl = flops(c.total_rows, c.N, c.K)
            by = sum(algorithmic_bytes(int(c.offsets[e + 1] - c.offsets[e]), c.N, c.K, c.G) for e in range(c.E))
        launch(0)
        torch.cuda.synchronize()
        n = 20 if fl < 1e10 else 4
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for i in range(n):
                launch(i % R)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        st = replay_stats(g, n, 100)
        us = st["median"]
        gbs = by / (us * 1e-6) / 1e9
        tf = fl / (us * 1e-6) / 1e12
        t_roof = max(by / (peaks["hbm_gbs"] * 1e9), fl / (peaks["bf16_tflops"] * 1e12))
        out[name] = {"us_per_launch": round(us, 3), "us_p10": st["p10"], "us_p90": st["p90"],
                     "GB/s": round(gbs, 1), "TFLOP/s": round(tf, 2),
                     "roofline_frac": round(t_roof / (us * 1e-6), 4),
                     "bound": "hbm" if by / (peaks["hbm_gbs"] * 1e9) >= fl / (peaks["bf16_tflops"] * 1e12)
                     else "tensor", "rotating_copies": R, "timing": f"median of {st['reps']} CUDA-graph replays of "
                                                                  f"{n} launches each"}
        if tactic is not None:
            out[name]["tactic"] = tactic
        if cfg["kind"] == "moe":
            out[name]["active_experts"] = active
        del g
    if not only or "quantize" in only:
        out["quantize"] = quantize_timing(w4, dev, peaks, l2)
        out["quantize_w8"] = quantize_timing(w4, dev, peaks, l2, bits=8)
    status = w4.device_status(clear=True)
    if status != w4.OK:
        raise RuntimeError(f"device status after per-config timing: {w4.status_string(status)}")
    return out


def quantize_timing(w4, dev, peaks, l2, K=4096, N=14336, G=128, bits=4):
    """The export-time quantiser (setup, not on the GEMM path) on the MLP up projection's
    fp16 weights: W read once, codes (int4 packed, or 8-bit) and scales written once per launch."""
    import torch
    gen = torch.Generator(device=dev).manual_seed(5)
    per_w = K * N * 2
    code_bytes = ((K + 1) // 2) * N if bits == 4 else K * N
    by = per_w + code_bytes + ((K + G - 1) // G) * N * 2
    R = max(2, math.ceil(2 * l2 / per_w) + 1)
    sets = []
    for _ in range(R):
        W = (torch.randn((K, N), generator=gen, device=dev, dtype=torch.float32) * 0.02).half()
        codes = (torch.empty(((K + 1) // 2, N), dtype=torch.uint8, device=dev) if bits == 4
                 else torch.empty((K, N), dtype=torch.int8, device=dev))
        sets.append((W, codes, torch.empty(((K + G - 1) // G, N), dtype=torch.float16, device=dev)))

    def launch(r):
        W, wp, S = sets[r]
        rc = (w4.w4a16_quantize if bits == 4 else w4.w8a16_quantize)(W, wp, S, K, N, G)
        if rc:
            raise RuntimeError(w4.status_string(rc))
    launch(0)
    torch.cuda.synchronize()
    n = 4
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(n):
            launch(i % R)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    st = replay_stats(g, n, 100)
    us = st["median"]
    del g
    return {"us_per_launch": round(us, 3), "us_p10": st["p10"], "us_p90": st["p90"],
            "GB/s": round(by / (us * 1e-6) / 1e9, 1),
            "roofline_frac": round(by / (peaks["hbm_gbs"] * 1e9) / (us * 1e-6), 4), "bound": "hbm",
            "rotating_copies": R, "shape": {"K": K, "N": N, "G": G}}


# ------------------------------------------------------------------ reference arm

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return
    import oracle
    o = oracle.load()
    case = workloads.dense(16, K_DIM, N_DIM, G_DIM, seed=1)
    K, W = args.steps, args.warmup
    # Calibrate a column sample so that warm-up plus timed steps take about two minutes.
    probe = oracle_sample(o, case, 64)
    oracle_decode_step(o, case, probe)
    t0 = time.perf_counter()
    oracle_decode_step(o, case, probe)
    t64 = max(time.perf_counter() - t0, 1e-6)
    cols = int(64 * (120.0 / (K + W)) / t64)
    cols = max(8, min(N_DIM, cols - cols % 8))
    sample = oracle_sample(o, case, cols)
    for _ in range(W):
        oracle_decode_step(o, case, sample)
    t0 = time.perf_counter()
    for _ in range(K):
        oracle_decode_step(o, case, sample)
    sec = time.perf_counter() - t0
    value = K * sample_bytes(cols) / sec / 1e9
    line = {
        "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world, "steps": K, "warmup": W,
        "ms_per_step": sec * 1e3 / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": WORKLOAD, "M": list(M_STEP), "K": K_DIM, "N": N_DIM, "G": G_DIM,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": o.threads(), "kind": "oracle",
                         "sample": f"each step: M=1 and M=16 over the first {cols} of {N_DIM} columns "
                                   f"(K=4096, G=128), fp64 oracle"},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile(args):
    """A few plain launches of one workload family, for ncu (no timing, no rotation)."""
    import torch
    from weight_only_int4_wise_b200 import build as wbuild
    wbuild.build()
    import weight_only_int4_wise_b200 as w4
    dev = torch.device("cuda", 0)
    if args.profile == "quantize":
        K, N, G = 4096, 14336, 128
        gen = torch.Generator(device=dev).manual_seed(5)
        W = (torch.randn((K, N), generator=gen, device=dev, dtype=torch.float32) * 0.02).half()
        for _ in range(args.launches):
            w4.quantize(W, G)
        torch.cuda.synchronize()
        print(f"profiled quantize: {args.launches} launches")
        return
    c = workloads.make(args.profile)
    kind = workloads.CONFIGS[args.profile]["kind"]
    if kind == "dense8":
        wt = w4.repack_w8(torch.from_numpy(c.q).to(dev))
        A, S = torch.from_numpy(c.A).to(dev), torch.from_numpy(c.S).to(dev)
        C = torch.empty((c.M, c.N), dtype=torch.float16, device=dev)
        for _ in range(args.launches):
            w4.gemm_w8(A, wt, S, c.N, c.G, out=C)
    elif kind == "moe":
        up = [w4.prepare_weights(torch.from_numpy(c.q_up[e]).to(dev))[1] for e in range(c.E)]
        down = [w4.prepare_weights(torch.from_numpy(c.q_down[e]).to(dev))[1] for e in range(c.E)]
        su = [torch.from_numpy(x).to(dev) for x in c.S_up]
        sd = [torch.from_numpy(x).to(dev) for x in c.S_down]
        X, lg = torch.from_numpy(c.X).to(dev), torch.from_numpy(c.logits).to(dev)
        for _ in range(args.launches):
            w4.moe_layer(X, lg, up, su, down, sd, c.top_k, c.I, c.G, w4.ACT_GELU_ERF)
    elif isinstance(c, workloads.DenseCase):
        if args.tactic:
            rc = w4.w4a16_set_tactic(c.M, c.N, c.K, c.G, args.tactic)
            if rc:
                raise RuntimeError(f"tactic {args.tactic}: {w4.status_string(rc)}")
        _, wt = w4.prepare_weights(torch.from_numpy(c.q).to(dev))
        A, S = torch.from_numpy(c.A).to(dev), torch.from_numpy(c.S).to(dev)
        C = torch.empty((c.M, c.N), dtype=torch.float16, device=dev)
        for _ in range(args.launches):
            w4.gemm(A, wt, S, c.N, c.G, out=C)
    else:
        wts = [w4.prepare_weights(torch.from_numpy(c.q[e]).to(dev))[1] for e in range(c.E)]
        Ss = [torch.from_numpy(c.S[e]).to(dev) for e in range(c.E)]
        A, off = torch.from_numpy(c.A).to(dev), torch.from_numpy(c.offsets).to(dev)
        C = torch.empty((c.total_rows, c.N), dtype=torch.float16, device=dev)
        for _ in range(args.launches):
            w4.grouped_gemm(A, wts, Ss, off, c.N, c.G, out=C)
    torch.cuda.synchronize()
    status = w4.device_status(clear=True)
    if status != w4.OK:
        raise RuntimeError(w4.status_string(status))
    print(f"profiled {args.profile}: {args.launches} launches")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100000)
    ap.add_argument("--warmup", type=int, default=1000)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the per-config timings")
    ap.add_argument("--configs", default="", help="comma-separated subset of the per-config timings")
    ap.add_argument("--cold-activations", action="store_true",
                    help="rotate the activations with the weights (from HBM) instead of one L2-resident buffer")
    ap.add_argument("--no-tune", action="store_true",
                    help="per-config timings with the built-in heuristic instead of autotuned launch forms")
    ap.add_argument("--tune-headline", action="store_true",
                    help="autotune the two headline shapes at setup (each on its own) instead of the heuristic")
    ap.add_argument("--profile", choices=sorted(workloads.CONFIGS) + ["quantize"],
                    help="only launch this workload (for ncu)")
    ap.add_argument("--launches", type=int, default=4, help="launches in --profile mode")
    ap.add_argument("--tactic", type=int, default=0, help="--profile mode: pin this tactic id for the shape")
    ap.add_argument("--pin-tactics", default="",
                    help="headline mode: 'M=id,...' pins these tactics instead of autotuning (profiling runs)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
