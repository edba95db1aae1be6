#!/usr/bin/env python
"""Benchmark of the block-quantized W4A8 matmul (Q4_0 weights x Q8_0 activations) on B200.

Headline (one JSON line on rank 0): the decode GEMV, M=1, K=N=4096, x f32 ~N(0,1),
W ~N(0,0.02) packed to Q4_0; metric = weight GB/s (packed weight + scale bytes per call /
call time). One step = one w4a8_gemm call through the C ABI: Q8_0 activation
quantisation + the M-dispatched contraction (the GEMV at M=1). Weights are packed once,
outside the timed region. Packed weight copies are rotated so that the set read by the
timed loop (28 x 9.44 MB) is larger than twice the 126 MB L2.

The same line carries: the dominant kernel's roofline (the contraction kernel alone, timed
with CUDA events through w4a8_gemm_prepared), an end-to-end figure through the C ABI with
host buffers (pinned H2D of x and D2H of y inside the timed region), the CPU oracle timed
on the host cores, SM clocks sampled during the timed region, and -- unless --no-extra --
the other workloads (MiniLM 64x384x1536, prefill 1024x4096x4096, the MLP-shape sweep, the
affine gs64/gs128 workloads) with µs, TOP/s and roofline fractions. Every timed workload
is first checked against the oracle; a workload that fails parity is reported as failed
and not timed.

--impl reference times the CPU oracle (the only reference this method has) on the same
workload and metric. Under torchrun every rank runs the same workload (independent
replicas: the path has no exchange step); the time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extra", action="store_true", help="headline workload only")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ramp-seconds", type=float, default=1.0, help="untimed load before warm-up (clock ramp)")
    ap.add_argument("--sweep", choices=["some", "all", "none"], default="all")
    ap.add_argument("--replays", type=int, default=7, help="timed graph replays of the headline (median reported)")
    ap.add_argument("--probe", default=None,
                    help="profiling probe: run `--steps` calls of one workload (decode, minilm, prefill, affine64, "
                         "affine128, affine6_64, affine8_64, q4k, q4k_bwd, or MxKxN) through w4a8_gemm[_affine[_nbit]], then exit "
                         "without timing")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(FALLBACK_PEAKS)
    d["source"] = "fallback"
    return d


def traffic_table():
    """Per-launch DRAM bytes (read + write) from the committed ncu summaries, keyed by
    kernel and workload; lines of the form `traffic_bytes_per_launch <key> <bytes>`."""
    out = {}
    d = os.path.join(ROOT, "profiles")
    if not os.path.isdir(d):
        return out
    for f in sorted(os.listdir(d)):
        if not f.endswith((".md", ".txt")):
            continue
        with open(os.path.join(d, f)) as fh:
            for line in fh:
                parts = line.strip().strip("`").split()
                if len(parts) == 3 and parts[0] == "traffic_bytes_per_launch":
                    try:
                        out[parts[1]] = float(parts[2])
                    except ValueError:
                        pass
    return out


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms in the background; keeps host-timestamped rows."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, bus_id: str | None):
        self.bus_id = (bus_id or "").lower()
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 10:
                self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self, t0: float, t1: float):
        rows = [p for (t, p) in self.rows if self.bus_id == "" or self.bus_id.endswith(p[1].lower()[-12:])
                or p[1].lower().endswith(self.bus_id[-12:])]
        if not rows:
            rows = [p for (_, p) in self.rows]
        inwin = [p for (t, p) in self.rows if t0 - 0.25 <= t <= t1 + 0.25 and p in rows]
        use = inwin if inwin else rows[-5:]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        sm = sorted(float(p[2]) for p in use if p[2].replace(".", "").isdigit())
        smx = max((float(p[3]) for p in use if p[3].replace(".", "").isdigit()), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in use for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": sm[len(sm) // 2] if sm else None, "sm_max_mhz": smx, "reasons": reasons,
                "samples": len(use), "in_window": bool(inwin)}


# ------------------------------------------------------------------ helpers
def rank_info():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("LOCAL_RANK", "0"))


# Cross-rank steps of the benchmark. Every rank calls each of these at the same point (in
# the error paths too), so the collectives match; with dist None (one process) they are
# plain values. `device` is where the collective's tensor lives ("cuda" under NCCL).
def max_over_ranks(value: float, dist=None, device="cuda") -> float:
    """The largest `value` over all ranks (the job's time is its slowest rank's)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def all_ranks_ok(ok: bool, dist=None, device="cuda") -> bool:
    """True when `ok` holds on every rank."""
    if dist is None:
        return bool(ok)
    import torch
    t = torch.tensor([1 if ok else 0], dtype=torch.int32, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MIN)
    return bool(t.item())


def whole_job_rate(units_per_rank: float, world: int, ms: float) -> float:
    """Units processed by all ranks per second, over the max-over-ranks time `ms`."""
    return units_per_rank * world / (ms * 1e-3)


def check_parity_sampled(y_dev, ref_fn, M, N, count=400, seed=7):
    import numpy as np
    from block_quantized_w4a8_b200 import inputs
    ms, ns = inputs.sample_indices(M, N, count, seed)
    yref, T = ref_fn(ms, ns)
    y = y_dev.cpu().numpy()[ms, ns].astype(np.float64)
    return bool(np.all(np.abs(y - yref) <= 1e-5 * T))


def timed(step, steps, torch, dist=None, graph=False):
    """Time exactly `steps` calls of step(i) with CUDA events on the current stream,
    bracketed by a barrier and a device synchronize on both sides. Returns ms (max over ranks).
    With graph=True the `steps` calls are first captured into one CUDA graph (outside the
    timed region) and the timed region is one replay of it, so host launch overhead is
    not part of the measurement."""
    if graph:
        g = torch.cuda.CUDAGraph()
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            with torch.cuda.graph(g, stream=s):
                for i in range(steps):
                    step(i)
        torch.cuda.current_stream().wait_stream(s)
        g.replay()  # one untimed replay
        torch.cuda.synchronize()
        run = g.replay
    else:
        def run():
            for i in range(steps):
                step(i)
    stream = torch.cuda.current_stream()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    run()
    e1.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    return max_over_ranks(e0.elapsed_time(e1), dist, "cuda")


def timed_replays(step, steps, torch, replays, dist=None):
    """The headline's timing: the `steps` calls captured once into a CUDA graph, then
    `replays` replays each timed as in timed() (barrier + synchronize on both sides, max over
    ranks). Returns the list of ms per replay."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for i in range(steps):
                step(i)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()  # one untimed replay
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    out = []
    for _ in range(replays):
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        if dist is not None:
            dist.barrier()
        out.append(max_over_ranks(e0.elapsed_time(e1), dist, "cuda"))
    del g
    return out


def copies_for(bytes_per_copy: int) -> int:
    return max(2, math.ceil(2 * L2_BYTES / max(1, bytes_per_copy)))


# ------------------------------------------------------------------ oracle timing
def oracle_decode_seconds(budget_s: float, nthreads: int):
    """Time the oracle on the decode workload (quantise x, contract over all 4096 rows)."""
    import oracle
    from block_quantized_w4a8_b200 import inputs
    x, w = inputs.make(inputs.DECODE)
    qs, d = oracle.pack_q4_0(w.numpy())
    xn = x.numpy()
    reps, t0 = 0, time.perf_counter()
    while True:
        qx, dx, _ = oracle.quant_act_q8_0(xn)
        oracle.gemm_q4_0(qx, dx, qs, d, nthreads=nthreads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s and reps >= 1:
            return el / reps, reps


def weight_bytes(N, K):
    return N * K // 2 + N * (K // 32) * 2


def gemv_algorithmic_bytes(M, N, K):
    B = K // 32
    return weight_bytes(N, K) + M * K + M * B * 8 + M * N * 4


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank, world, _ = rank_info()
    if rank != 0:
        return 0
    nthreads = os.cpu_count() or 1
    per_step = []
    for i in range(args.warmup + args.steps):
        s, _ = oracle_decode_seconds(0.0, nthreads)
        if i >= args.warmup:
            per_step.append(s)
    sec = sum(per_step) / len(per_step)
    M, N, K = 1, 4096, 4096
    gbs = weight_bytes(N, K) / sec / 1e9
    line = {
        "impl": "reference", "metric": "W4A8 decode GEMV weight GB/s (M=1, K=N=4096)", "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": "decode_gemv_m1_4096x4096", "M": M, "N": N, "K": K},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": nthreads, "kind": "oracle",
                         "sample": f"{args.steps} full decode steps (Q8_0 quantisation of x + all 4096 outputs of "
                                   f"the 1x4096x4096 contraction), threads over output elements; one step per "
                                   f"timed step"},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
def run_ours(args):
    import numpy as np
    import torch
    import torch.distributed as dist_mod

    import block_quantized_w4a8_b200 as w4a8
    import oracle
    from block_quantized_w4a8_b200 import inputs

    rank, world, local_rank = rank_info()
    dist = None
    if world > 1:
        from datetime import timedelta
        torch.cuda.set_device(local_rank)
        dist_mod.init_process_group("nccl", timeout=timedelta(seconds=120))
        dist = dist_mod
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    w4a8.load_library()
    peaks = load_peaks()
    traffic = traffic_table()
    props = torch.cuda.get_device_properties(dev)
    bus = None
    try:
        bus = f"{props.pci_domain_id:04x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}"
    except Exception:
        pass
    launches = 0

    # ---------------- headline: decode GEMV
    wl = inputs.DECODE
    M, N, K = wl.M, wl.N, wl.K
    x, w = inputs.make(wl)
    xd, wd = x.to(dev), w.to(dev)
    qs0, d0 = w4a8.pack_q4_0(wd)
    R = copies_for(weight_bytes(N, K))
    qsl = [qs0.clone() for _ in range(R)]
    dl = [d0.clone() for _ in range(R)]
    ws = w4a8.workspace(M, N, K, 0, dev)
    y = torch.empty(M, N, device=dev)
    w4a8.w4a8_gemm(xd, qs0, d0, y, ws)
    torch.cuda.synchronize()
    rqx, rdx, _ = oracle.quant_act_q8_0(x.numpy())
    rqs, rd = oracle.pack_q4_0(w.numpy())
    yref, T = oracle.gemm_q4_0(rqx, rdx, rqs, rd, nthreads=os.cpu_count() or 1)
    parity = bool(np.array_equal(qs0.cpu().numpy(), rqs)) and bool(
        np.all(np.abs(y.cpu().numpy().astype(np.float64) - yref) <= 1e-5 * T))
    if not all_ranks_ok(parity, dist, "cuda"):  # every rank stops together
        if rank == 0:
            print(json.dumps({"metric": "W4A8 decode GEMV weight GB/s (M=1, K=N=4096)", "value": None,
                              "error": "parity check against the oracle failed; not timed"}), flush=True)
        if dist is not None:
            dist.destroy_process_group()
        return 1

    def step(i):
        w4a8.w4a8_gemm(xd, qsl[i % R], dl[i % R], y, ws)

    sampler = ClockSampler(bus)
    sampler.start()
    t_ramp = time.time()
    while time.time() - t_ramp < args.ramp_seconds:  # bring clocks up before warm-up
        for i in range(200):
            step(i)
        torch.cuda.synchronize()
    for i in range(args.warmup):
        step(i)
    t0 = time.time()
    reps_ms = timed_replays(step, args.steps, torch, max(1, args.replays), dist)
    t1 = time.time()
    ms = sorted(reps_ms)[len(reps_ms) // 2]  # the median replay
    ms_eager = timed(step, args.steps, torch, dist)
    # M*K = 4096 is small enough for the GEMV to quantise x itself: one launch per step
    launches += args.steps
    ms_step = ms / args.steps
    value = whole_job_rate(weight_bytes(N, K) * args.steps, world, ms) / 1e9
    k_us = ms_step * 1e3
    alg = weight_bytes(N, K) + M * K * 4 + M * N * 4   # packed weights + scales, f32 x, f32 y
    achieved = alg / (k_us * 1e-6) / 1e9
    tkey = "gemv_resident_m1_q4_0:decode_m1_4096x4096"

    # the split form (quantise once, then the contraction kernel alone), for reference
    w4a8.w4a8_prepare_act(xd, ws)
    for i in range(args.warmup):
        w4a8.w4a8_gemm_prepared(M, K, qsl[i % R], dl[i % R], y, ws)
    kms = timed(lambda i: w4a8.w4a8_gemm_prepared(M, K, qsl[i % R], dl[i % R], y, ws), args.steps, torch, dist,
                graph=True)
    prepared_us = kms / args.steps * 1e3

    # end to end through the C ABI with host buffers
    xh = x.pin_memory()
    yh = torch.empty(M, N, pin_memory=True)

    def step_e2e(i):
        xd.copy_(xh, non_blocking=True)
        w4a8.w4a8_gemm(xd, qsl[i % R], dl[i % R], y, ws)
        yh.copy_(y, non_blocking=True)

    for i in range(args.warmup):
        step_e2e(i)
    ems = timed(step_e2e, args.steps, torch, dist)
    e2e_value = whole_job_rate(weight_bytes(N, K) * args.steps, world, ems) / 1e9
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    line = {
        "metric": "W4A8 decode GEMV weight GB/s (M=1, K=N=4096)", "value": value, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": "decode_gemv_m1_4096x4096", "M": M, "N": N, "K": K,
                   "weights": "Q4_0 (32-blocks, fp16 scale)", "activations": "f32 -> Q8_0 in the call",
                   "l2": f"inputs larger than L2: {R} rotating packed weight copies "
                         f"({R * weight_bytes(N, K) / 1e6:.0f} MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "parity": "pass",
        "timing": f"CUDA graph of the {args.steps} timed steps captured outside the region; {len(reps_ms)} replays "
                  f"each timed with events; value = the median replay",
        "replays_ms_per_step": {"median": ms_step, "min": min(reps_ms) / args.steps,
                                "max": max(reps_ms) / args.steps, "n": len(reps_ms),
                                "spread_pct": 100.0 * (max(reps_ms) - min(reps_ms)) / ms},
        "ms_per_step_eager": ms_eager / args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "traffic": traffic.get(tkey),
                     "traffic_note": None if traffic.get(tkey) is not None else
                     "no ncu capture of the current kernel build (profiles/ holds an earlier build's counters)",
                     "kernel": "gemv_resident_kernel<1,0,true,XS> (Q4_0, M=1, weights resident in shared "
                               "memory, x quantised in-kernel; the whole step)",
                     "kernel_us": k_us, "prepared_contraction_us": prepared_us,
                     "algorithmic_bytes_per_launch": alg, "peak_source": peaks.get("source", "measured") +
                     " (MEASURED_PEAKS.json hbm_gbs, copy bandwidth)"},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": M * K * 4, "d2h_bytes_per_step": M * N * 4,
                "ms_per_step": ems / args.steps},
        "gpu_launches": launches,
        "clocks": clocks,
    }

    # ---------------- CPU baseline (rank 0, N=1)
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        nth = os.cpu_count() or 1
        sec, reps = oracle_decode_seconds(args.cpu_seconds, nth)
        line["cpu_baseline"] = {"value": weight_bytes(N, K) / sec / 1e9, "unit": "GB/s", "cores": nth,
                                "kind": "oracle", "ms_per_step": sec * 1e3,
                                "sample": f"{reps} full decode steps (Q8_0 quantisation of x + all 4096 outputs of "
                                          f"the 1x4096x4096 contraction), threads over output elements; as many "
                                          f"steps as fit in ~{args.cpu_seconds:.0f} s"}
        # the same oracle on one host thread (the scalar figure), a shorter bounded sample
        sec1, reps1 = oracle_decode_seconds(max(1.0, args.cpu_seconds / 4), 1)
        line["cpu_baseline"]["single_thread"] = {"value": weight_bytes(N, K) / sec1 / 1e9, "unit": "GB/s",
                                                 "cores": 1, "ms_per_step": sec1 * 1e3,
                                                 "sample": f"{reps1} full decode steps on one thread"}

    # ---------------- other workloads (rank 0 only, after the collective steps)
    if rank == 0 and not args.no_extra:
        line["configs"] = run_extra(args, torch, w4a8, oracle, inputs, peaks, traffic, dev)

    if dist is not None:
        dist.barrier()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


def run_extra(args, torch, w4a8, oracle, inputs, peaks, traffic, dev):
    import numpy as np
    # Dense INT8 peak: 2 x the measured dense bf16 rate. The factor is measured: a
    # tcgen05.mma rate loop issues kind::i8 at 16.2K and kind::f16 at 8.1K ops per clock per
    # SM on this part (ratio 2.00).
    int8_peak = 2.0 * peaks["bf16_tflops"]
    f16_peak = peaks["bf16_tflops"]             # the pair kernel runs kind::f16 (fp16 = bf16 rate)
    results = []
    wls = [inputs.MINILM, inputs.PREFILL]
    if args.sweep != "none":
        sweep = inputs.sweep_workloads()
        if args.sweep == "some":
            keep = {(1, 4096, 14336), (16, 4096, 14336), (64, 4096, 14336), (256, 14336, 4096),
                    (1024, 4096, 14336), (4096, 8192, 2048), (8, 8192, 2048)}
            sweep = [s for s in sweep if (s.M, s.K, s.N) in keep]
        wls += sweep
    wls += [inputs.AFFINE_GS64, inputs.AFFINE_GS128]
    steps = max(5, min(args.steps, 50))
    for wl in wls:
        M, N, K = wl.M, wl.N, wl.K
        x, w = inputs.make(wl)
        xd = x.to(dev)
        affine = wl.kind == "affine"
        if affine:
            q, s, b = w4a8.pack_affine(w.to(dev), wl.group)
            wbytes = N * K // 2 + 2 * N * (K // wl.group) * 2
        else:
            qs, d = w4a8.pack_q4_0(w.to(dev))
            wbytes = weight_bytes(N, K)
        R = copies_for(wbytes)
        ws = w4a8.workspace(M, N, K, wl.group if affine else 0, dev)
        y = torch.empty(M, N, device=dev)
        rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
        if affine:
            sets = [(q.clone(), s.clone(), b.clone()) for _ in range(R)]
            rq, rs, rb = oracle.pack_affine(w.numpy(), wl.group)
            w4a8.w4a8_gemm_affine(xd, q, s, b, y, ws, wl.group)
            ok = check_parity_sampled(y, lambda ms, ns: oracle.gemm_affine_sampled(rqx, rdx, rsx, rq, rs, rb, wl.group,
                                                                                   ms, ns), M, N)

            def step(i):
                qq, ss, bb = sets[i % R]
                w4a8.w4a8_gemm_affine(xd, qq, ss, bb, y, ws, wl.group)

            def kstep(i):
                qq, ss, bb = sets[i % R]
                w4a8.w4a8_gemm_affine_prepared(M, K, wl.group, qq, ss, bb, y, ws)
        else:
            sets = [(qs.clone(), d.clone()) for _ in range(R)]
            rqs, rd = oracle.pack_q4_0(w.numpy())
            w4a8.w4a8_gemm(xd, qs, d, y, ws)
            ok = check_parity_sampled(y, lambda ms, ns: oracle.gemm_q4_0_sampled(rqx, rdx, rqs, rd, ms, ns), M, N)

            def step(i):
                qq, dd = sets[i % R]
                w4a8.w4a8_gemm(xd, qq, dd, y, ws)

            def kstep(i):
                qq, dd = sets[i % R]
                w4a8.w4a8_gemm_prepared(M, K, qq, dd, y, ws)
        path = w4a8.w4a8_gemm_path(M, N, K, wl.group if affine else 0)
        hbm_bound = path in ("gemv", "gemm_i8")
        entry = {"workload": wl.name, "M": M, "N": N, "K": K, "path": path, "parity": "pass" if ok else "FAIL"}
        if ok:
            for i in range(3):
                step(i)
            ms = timed(step, steps, torch, graph=True)
            if affine:
                w4a8.w4a8_prepare_act(xd, ws, wl.group)
            else:
                w4a8.w4a8_prepare_act(xd, ws)
            for i in range(3):
                kstep(i)
            kms = timed(kstep, steps, torch, graph=True)
            us, kus = ms / steps * 1e3, kms / steps * 1e3
            ops = 2.0 * M * N * K
            entry.update({"us_per_call": us, "kernel_us": kus, "tops_call": ops / (us * 1e-6) / 1e12,
                          "tops_kernel": ops / (kus * 1e-6) / 1e12,
                          "weight_gbs_call": wbytes / (us * 1e-6) / 1e9})
            if hbm_bound:
                # weights + quantised activation + f32 output, over the contraction alone
                alg = wbytes + M * K + M * (K // 32) * 8 + M * N * 4
                entry["roofline"] = {"bound": "hbm", "achieved": alg / (kus * 1e-6) / 1e9, "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "algorithmic_bytes": alg,
                                     "frac_int8": entry["tops_kernel"] / int8_peak}
                entry["roofline"]["frac"] = entry["roofline"]["achieved"] / peaks["hbm_gbs"]
            else:
                tk = entry["tops_kernel"]
                # The tensor path runs each 32-wide block dot as fp16 MMAs on exact operands:
                # Q4_0 twice (the weight scale split into two exactly representable parts),
                # affine once plus one K=16 MMA per block for the group bias term (CTA-pair
                # kernel), so the tensor pipe executes `parts` x the useful operations.
                parts = 1.5 if affine else 2
                entry["roofline"] = {"bound": "tensor", "achieved": tk, "unit": "TOP/s",
                                     "peak_int8": int8_peak, "frac_int8": tk / int8_peak,
                                     "mma_f16_tflops_executed": parts * tk, "peak_f16_mma": f16_peak,
                                     "frac_f16_mma": parts * tk / f16_peak}
            entry["l2"] = f"{R} rotating weight copies"
        results.append(entry)
        del sets
        torch.cuda.empty_cache()
    results += run_epilogue(args, torch, w4a8, oracle, inputs, steps, dev)
    results += run_wide(args, torch, w4a8, oracle, inputs, steps, dev, int8_peak)
    results += run_q4k(args, torch, w4a8, oracle, inputs, steps, dev, peaks)
    return results


def run_epilogue(args, torch, w4a8, oracle, inputs, steps, dev):
    """The output epilogue (per-column f32 bias, bf16 output) on the decode GEMV and the
    prefill GEMM, through w4a8_gemm_epi, timed beside the plain call on the same inputs."""
    import numpy as np
    out = []
    for wl in (inputs.DECODE, inputs.PREFILL):
        M, N, K = wl.M, wl.N, wl.K
        x, w = inputs.make(wl)
        xd = x.to(dev)
        bias = inputs.randn((N,), seed=5, std=1.0)
        bd = bias.to(dev)
        qs, d = w4a8.pack_q4_0(w.to(dev))
        R = copies_for(weight_bytes(N, K))
        sets = [(qs.clone(), d.clone()) for _ in range(R)]
        ws = w4a8.workspace(M, N, K, 0, dev)
        y = torch.empty(M, N, device=dev, dtype=torch.bfloat16)
        yp = torch.empty(M, N, device=dev)
        w4a8.w4a8_gemm_epi(xd, qs, d, y, ws, bias=bd)
        torch.cuda.synchronize()
        rqx, rdx, _ = oracle.quant_act_q8_0(x.float().numpy())
        rqs, rd = oracle.pack_q4_0(w.numpy())
        ms, ns = (np.asarray(t) for t in inputs.sample_indices(M, N, 400, 7))
        yref, T = oracle.gemm_q4_0_sampled(rqx, rdx, rqs, rd, ms, ns)
        ref = oracle.bf16_to_f32(oracle.epilogue(yref.astype(np.float32)[None, :], bias.numpy()[ns],
                                                 out_bf16=True)[0]).astype(np.float64)
        got = y.float().cpu().numpy()[ms, ns].astype(np.float64)
        ok = bool(np.all(np.abs(got - ref) <= 1e-5 * T + np.abs(ref) * 2.0 ** -7))
        entry = {"workload": wl.name + "_bias_bf16out", "M": M, "N": N, "K": K,
                 "path": w4a8.w4a8_gemm_path(M, N, K), "epilogue": "f32 bias per column, bf16 output",
                 "parity": "pass" if ok else "FAIL"}
        if ok:
            def step(i):
                qq, dd = sets[i % R]
                w4a8.w4a8_gemm_epi(xd, qq, dd, y, ws, bias=bd)

            def plain(i):
                qq, dd = sets[i % R]
                w4a8.w4a8_gemm(xd, qq, dd, yp, ws)
            for i in range(3):
                step(i)
                plain(i)
            us = timed(step, steps, torch, graph=True) / steps * 1e3
            us_plain = timed(plain, steps, torch, graph=True) / steps * 1e3
            entry.update({"us_per_call": us, "us_per_call_plain": us_plain,
                          "tops_call": 2.0 * M * N * K / (us * 1e-6) / 1e12, "l2": f"{R} rotating weight copies"})
        out.append(entry)
        del sets
        torch.cuda.empty_cache()
    return out


def run_wide(args, torch, w4a8, oracle, inputs, steps, dev, int8_peak):
    """Affine weights with 6- and 8-bit codes (w4a8_gemm_affine_nbit) on the MLX page's
    setup (M=1024, K=N=4096, bf16 x, normal weights; groups of 64 and 128) and a decode
    GEMV line, each parity-checked on sampled outputs before it is timed. Per call,
    including the activation quantisation."""
    import numpy as np
    out = []
    cases = [(1024, 6, 64), (1024, 8, 64), (1024, 8, 128), (1, 8, 64)]
    for M, bits, group in cases:
        N = K = 4096
        wl = inputs.Workload(f"affine{bits}_m{M}_{K}x{N}_gs{group}", M=M, K=K, N=N, x_dtype="bf16", w_std=1.0,
                             kind="affine", group=group)
        x, w = inputs.make(wl)
        xd = x.to(dev)
        q, s, b = w4a8.pack_affine_nbit(w.to(dev), group, bits)
        wbytes = N * K * bits // 8 + 2 * N * (K // group) * 2
        R = copies_for(wbytes)
        sets = [(q.clone(), s.clone(), b.clone()) for _ in range(R)]
        ws = w4a8.workspace(M, N, K, group, dev)
        y = torch.empty(M, N, device=dev)
        w4a8.w4a8_gemm_affine_nbit(xd, q, s, b, y, ws, group, bits)
        torch.cuda.synchronize()
        rqx, rdx, rsx = oracle.quant_act_q8_0(x.float().numpy())
        rq, rs, rb = oracle.pack_affine(w.numpy(), group, bits=bits)
        ok = check_parity_sampled(y, lambda ms, ns: oracle.gemm_affine_sampled(
            rqx, rdx, rsx, rq, rs, rb, group, np.asarray(ms), np.asarray(ns), bits=bits), M, N)
        entry = {"workload": wl.name, "M": M, "N": N, "K": K, "bits": bits, "group": group,
                 "path": "gemv" if M <= 8 else "gemm_pair", "parity": "pass" if ok else "FAIL"}
        if ok:
            def step(i):
                qq, ss, bb = sets[i % R]
                w4a8.w4a8_gemm_affine_nbit(xd, qq, ss, bb, y, ws, group, bits)
            for i in range(3):
                step(i)
            us = timed(step, steps, torch, graph=True) / steps * 1e3
            tops = 2.0 * M * N * K / (us * 1e-6) / 1e12
            entry.update({"us_per_call": us, "tops_call": tops, "weight_gbs_call": wbytes / (us * 1e-6) / 1e9,
                          "l2": f"{R} rotating weight copies"})
            if M > 8:
                entry["frac_int8_call"] = tops / int8_peak
        out.append(entry)
        del sets
        torch.cuda.empty_cache()
    return out


def run_q4k(args, torch, w4a8, oracle, inputs, steps, dev, peaks):
    """Q4_K GEMV (y = x W^T) and its input gradient (dX = dY W) with FP32 activations at
    decode size (M=1, K=N=4096), each checked against the oracle on all outputs before it
    is timed; weight GB/s against the measured HBM copy bandwidth."""
    import numpy as np
    out = []
    M, N, K = 1, 4096, 4096
    W = inputs.make_q4_k(N, K, seed=21)
    wbytes = N * K // 256 * 144
    R = copies_for(wbytes)
    sets = [W.to(dev) for _ in range(R)]
    x = inputs.randn((M, K), seed=22)
    dy = inputs.randn((M, N), seed=23)
    xd, dyd = x.to(dev), dy.to(dev)
    y = torch.empty(M, N, device=dev)
    dx = torch.empty(M, K, device=dev)
    ws = torch.empty(max(16, w4a8.w4a8_q4_k_backward_workspace_bytes(M, N, K)), dtype=torch.uint8, device=dev)
    w4a8.w4a8_gemv_q4_k(xd, sets[0], y)
    w4a8.w4a8_gemv_q4_k_backward(dyd, sets[0], dx, ws)
    torch.cuda.synchronize()
    yref, Ty = oracle.gemv_q4_k(x.numpy(), W.numpy(), N, nthreads=8)
    dxref, Tx = oracle.gemv_q4_k_backward(dy.numpy(), W.numpy(), K, nthreads=8)
    # the same tolerance as every other output: 1e-5 of the sum of |terms|
    ok_f = bool(np.all(np.abs(y.cpu().numpy().astype(np.float64) - yref) <= 1e-5 * Ty))
    ok_b = bool(np.all(np.abs(dx.cpu().numpy().astype(np.float64) - dxref) <= 1e-5 * Tx))
    for name, ok, fn in [("q4_k_gemv_m1_4096x4096", ok_f, lambda i: w4a8.w4a8_gemv_q4_k(xd, sets[i % R], y)),
                         ("q4_k_backward_m1_4096x4096", ok_b,
                          lambda i: w4a8.w4a8_gemv_q4_k_backward(dyd, sets[i % R], dx, ws))]:
        entry = {"workload": name, "M": M, "N": N, "K": K, "parity": "pass" if ok else "FAIL"}
        if ok:
            for i in range(3):
                fn(i)
            us = timed(fn, steps, torch, graph=True) / steps * 1e3
            gbs = wbytes / (us * 1e-6) / 1e9
            entry.update({"us_per_call": us, "weight_gbs_call": gbs,
                          "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                       "frac": gbs / peaks["hbm_gbs"]},
                          "l2": f"{R} rotating weight copies"})
        out.append(entry)
    del sets
    torch.cuda.empty_cache()
    return out


def run_probe(args):
    """A short, fixed sequence of launches for ncu: `--steps` calls of w4a8_gemm (or
    w4a8_gemm_affine) through the C ABI on the workload named by --probe."""
    import torch
    import block_quantized_w4a8_b200 as w4a8
    from block_quantized_w4a8_b200 import inputs
    named = {"decode": inputs.DECODE, "minilm": inputs.MINILM, "prefill": inputs.PREFILL,
             "affine64": inputs.AFFINE_GS64, "affine128": inputs.AFFINE_GS128}
    wide = {"affine6_64": (6, 64), "affine8_64": (8, 64)}  # 6/8-bit codes, M=1024, K=N=4096
    bits = 4
    if args.probe in ("q4k", "q4k_bwd"):  # Q4_K forward / input gradient, M=1, K=N=4096
        torch.cuda.set_device(0)
        w4a8.load_library()
        W = inputs.make_q4_k(4096, 4096, seed=21).cuda()
        x = inputs.randn((1, 4096), seed=22).cuda()
        out = torch.empty(1, 4096, device="cuda")
        ws = torch.empty(max(16, w4a8.w4a8_q4_k_backward_workspace_bytes(1, 4096, 4096)), dtype=torch.uint8,
                         device="cuda")
        for _ in range(args.steps):
            if args.probe == "q4k":
                w4a8.w4a8_gemv_q4_k(x, W, out)
            else:
                w4a8.w4a8_gemv_q4_k_backward(x, W, out, ws)
        torch.cuda.synchronize()
        print(f"probe {args.probe}: {args.steps} steps ok")
        return 0
    if args.probe in wide:
        bits, group = wide[args.probe]
        wl = inputs.Workload(f"affine{bits}_m1024_4096x4096_gs{group}", M=1024, K=4096, N=4096, x_dtype="bf16",
                             w_std=1.0, kind="affine", group=group)
    elif args.probe in named:
        wl = named[args.probe]
    else:
        M, K, N = (int(v) for v in args.probe.split("x"))
        wl = inputs.Workload(f"probe_{args.probe}", M=M, K=K, N=N)
    torch.cuda.set_device(0)
    w4a8.load_library()
    x, w = inputs.make(wl)
    xd, wd = x.cuda(), w.cuda()
    g = wl.group if wl.kind == "affine" else 0
    ws = w4a8.workspace(wl.M, wl.N, wl.K, g)
    y = torch.empty(wl.M, wl.N, device="cuda")
    if bits != 4:
        q, s, b = w4a8.pack_affine_nbit(wd, g, bits)
    elif g:
        q, s, b = w4a8.pack_affine(wd, g)
    else:
        qs, d = w4a8.pack_q4_0(wd)
    torch.cuda.synchronize()
    for _ in range(args.steps):  # the public call one benchmark step makes
        if bits != 4:
            w4a8.w4a8_gemm_affine_nbit(xd, q, s, b, y, ws, g, bits)
        elif g:
            w4a8.w4a8_gemm_affine(xd, q, s, b, y, ws, g)
        else:
            w4a8.w4a8_gemm(xd, qs, d, y, ws)
    torch.cuda.synchronize()
    assert w4a8.w4a8_last_device_error() == 0
    print(f"probe {wl.name}: {args.steps} steps ok")
    return 0


def main():
    args = parse_args()
    if args.probe:
        return run_probe(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
