#!/usr/bin/env python3
"""Benchmark of the block-wise mixed-precision weight-only linear layer.

One step = one mpq_linear call (activation reorder + mixed-precision GEMV +
inverse output reorder) on one seeded synthetic layer: by default the
Llama-2-7B attention projection 4096x4096 at M=1 with 2.1 average bits.  Each
step uses the next of R replicas of the packed layer, whose total size is more
than 4x the L2 cache, so no step finds its weights in L2.

Prints ONE JSON line (rank 0).  value = algorithmic HBM bytes / time
(GB/s, summed over ranks, time = max over ranks).  Multi-GPU runs are
independent replicas (the path has no exchange step).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mpq|reference]
                  [--extra]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "mpq_linear HBM GB/s (M=1) & TFLOP/s (M≥512), as fraction of B200 roofline"
HEADLINE_CFG = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
# helpers usable without a GPU
# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return dict(FALLBACK_PEAKS), "fallback"


def algorithmic_bytes(N, K, M, codes_bytes, n_sz, T, has_rp, has_cp):
    """Bytes a layer call must move: codes, fp16 scale+zero, the block table,
    the permutations, bf16 x and fp32 y."""
    return (codes_bytes + 4 * n_sz + 16 * T + 4 * (N if has_rp else 0) +
            4 * (K if has_cp else 0) + 2 * M * K + 4 * M * N)


def source_hash():
    h = hashlib.sha1()
    d = os.path.join(ROOT, "block_wise_mixed_b200", "csrc")
    for name in sorted(os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != source_hash():
        return None
    return e.get("dram_bytes_per_launch")


def reduce_max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a float over ranks (the device time of a multi-GPU step)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum_over_ranks(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled in the background."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            f = [v.strip() for v in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": float(max(mx)),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle as it stands
# ---------------------------------------------------------------------------
def oracle_baseline(layer, x, min_seconds=10.0, rows=None, threads=None):
    """The oracle's linear timed on the host: all cores (threads=None) or a
    given number of OpenMP threads."""
    from oracle import oracle
    R = oracle.pack(layer.W, layer.bits, layer.row_perm, layer.col_perm)
    prev = oracle.set_threads(threads) if threads else None
    if rows is None:
        rows = np.arange(layer.N, dtype=np.int32)
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle.linear_rows(R, x, rows)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    if prev is not None:
        oracle.set_threads(prev)
    frac = len(rows) / layer.N
    T = (layer.N // 64) * (layer.K // 128)
    nbytes = algorithmic_bytes(layer.N, layer.K, x.shape[0], R.codes.size * frac,
                               R.scales.size * frac, T * frac, layer.row_perm is not None,
                               layer.col_perm is not None)
    cores = threads or int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": nbytes * n / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "%d calls of the fp64 oracle's linear on %d of %d output rows "
                      "(dequant + dot), %.1f s" % (n, len(rows), layer.N, el),
            "seconds_per_call": el / n}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def build_replicas(mpq, P, R):
    """R deep copies of a packed layer (distinct device addresses)."""
    import torch
    from block_wise_mixed_b200 import _lib
    reps = []
    for _ in range(R):
        c = {k: (getattr(P, k).clone() if getattr(P, k) is not None else None)
             for k in ("codes", "table", "sched", "scales", "zeros", "row_perm", "col_perm")}
        layer = _lib.Layer(P.c.N, P.c.K, P.c.n_units, 0, c["codes"].data_ptr(),
                           c["table"].data_ptr(), c["sched"].data_ptr(), c["scales"].data_ptr(),
                           c["zeros"].data_ptr(),
                           c["row_perm"].data_ptr() if c["row_perm"] is not None else None,
                           c["col_perm"].data_ptr() if c["col_perm"] is not None else None)
        reps.append(_lib.PackedLayer(P.layout, c["codes"], c["table"], c["sched"], c["scales"],
                                     c["zeros"], c["row_perm"], c["col_perm"], layer))
    torch.cuda.synchronize()
    return reps


def launches_per_call(lay, M, has_row_perm):
    """Kernels one mpq_linear call launches (the library's dispatch rule):
    M <= 16 -- the activation prologue unless M == 1 on a layer whose runs
    hold at most two blocks on average (the decode kernel then builds its own
    activation records), plus one decode launch per 8 tokens; M > 16 -- the
    prologue, the tensor-core kernel and, when the rows are reordered, the
    reordering kernel (split-K partials too)."""
    if M <= 16:
        fused = M == 1 and lay.NB * lay.KB <= 2 * lay.n_units
        return (0 if fused else 1) + (M + 7) // 8
    return 2 + (1 if has_row_perm else 0)


def time_layer(mpq, layer_spec, M, steps, warmup, world, device, soak_s=1.0, sampler=None,
               quick=False):
    """Times `steps` mpq_linear calls over L2-busting replicas of one layer.
    Returns a dict of measurements."""
    import torch
    from block_wise_mixed_b200 import synth
    L = layer_spec
    W = torch.from_numpy(L.W.view(np.int16)).to(device)
    P = mpq.pack(W, L.bits, L.row_perm, L.col_perm)
    del W
    lay = P.layout
    T = lay.NB * lay.KB
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    per_rep = lay.codes_bytes + 4 * lay.n_sz + 16 * T + 4 * (lay.N + lay.K)
    R = int(max(2, min(512, np.ceil(4 * l2 / max(per_rep, 1)))))
    reps = build_replicas(mpq, P, R)
    x_bits = synth.make_x(synth.seed_of(99, 0), M, L.K)
    x = torch.from_numpy(x_bits.view(np.int16)).to(device)
    y = torch.empty((M, L.N), dtype=torch.float32, device=device)
    ws = torch.zeros(mpq.linear_workspace_size(P, M), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for i in range(max(warmup, 3)):
        mpq.linear(reps[i % R], x, y, ws)
    torch.cuda.synchronize(device)
    # soak: keep the GPU under the same load for ~soak_s so the clock record
    # covers a sustained state, then the timed region
    if sampler:
        sampler.start()
    t_end = time.perf_counter() + soak_s
    i = 0
    while time.perf_counter() < t_end:
        for _ in range(50):
            mpq.linear(reps[i % R], x, y, ws)
            i += 1
        torch.cuda.synchronize(device)
    # the timed steps run as one CUDA graph (launch overhead of the host
    # binding is not part of the device time, as in graph-launched decoding)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for s_ in range(steps):
            mpq.linear(reps[s_ % R], x, y, ws)
    graph.replay()
    torch.cuda.synchronize(device)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    torch.cuda.synchronize(device)
    clocks = sampler.stop() if sampler else None
    ms_total = e0.elapsed_time(e1)
    ms_step = reduce_max_over_ranks(ms_total, world, device) / steps
    nbytes = algorithmic_bytes(L.N, L.K, M, lay.codes_bytes, lay.n_sz, T,
                               L.row_perm is not None, L.col_perm is not None)
    del graph
    if quick:
        return dict(N=L.N, K=L.K, M=M, bytes=nbytes, ms_step=ms_step, replicas=R)

    # main-kernel time alone: events recorded by the library around it.  A
    # spin kernel first holds the GPU while the host enqueues every call, so
    # the calls run back to back and the events see device time only.
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for a, b in evs:        # torch creates the CUDA events on first record
        a.record(stream)
        b.record(stream)
    torch.cuda.synchronize(device)
    torch.cuda._sleep(int(2e6 + 4e4 * steps))   # ~1 ms + 20 us per enqueued call
    for s_ in range(steps):
        mpq.linear_timed(reps[s_ % R], x, y, ws, evs[s_][0], evs[s_][1])
    torch.cuda.synchronize(device)
    k_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))

    # end to end through the host entry point (pinned host x and y)
    xh = torch.from_numpy(x_bits.view(np.int16)).pin_memory()
    yh = torch.empty((M, L.N), dtype=torch.float32).pin_memory()
    wsh = torch.zeros(mpq.linear_host_workspace_size(P, M), dtype=torch.uint8, device=device)
    for i in range(3):
        mpq.linear_host(reps[i % R], xh, yh, wsh)
    torch.cuda.synchronize(device)
    h0 = torch.cuda.Event(enable_timing=True)
    h1 = torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    for s in range(steps):
        mpq.linear_host(reps[s % R], xh, yh, wsh)
    h1.record(stream)
    torch.cuda.synchronize(device)
    e2e_ms = reduce_max_over_ranks(h0.elapsed_time(h1), world, device) / steps

    # one cold call: L2 flushed by writing a buffer twice its size, then a
    # single mpq_linear between events (launch latency included)
    flush = torch.empty(2 * l2, dtype=torch.uint8, device=device)
    cold = []
    for i in range(3):
        flush.fill_(i + 1)
        c0 = torch.cuda.Event(enable_timing=True)
        c1 = torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        mpq.linear(reps[i % R], x, y, ws)
        c1.record(stream)
        torch.cuda.synchronize(device)
        cold.append(c0.elapsed_time(c1))
    del flush
    cold_ms = float(np.median(cold))

    kbytes = (lay.codes_bytes + 4 * lay.n_sz + 16 * T + 4 * (L.N if L.row_perm is not None else 0)
              + 2 * M * L.K + 4 * M * L.N)
    out = dict(N=L.N, K=L.K, M=M, avg_bits=float(L.bits.mean()), f0=float((L.bits == 0).mean()),
               replicas=R, l2_bytes=int(l2), bytes=nbytes, kernel_bytes=kbytes,
               ms_step=ms_step, kernel_ms=k_ms, e2e_ms=e2e_ms, cold_ms=cold_ms, clocks=clocks,
               launches_per_step=launches_per_call(lay, M, L.row_perm is not None), n_units=lay.n_units,
               h2d=M * L.K * 2, d2h=M * L.N * 4)
    del reps
    torch.cuda.empty_cache()
    return out


def run_gpu(args):
    import torch
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    from block_wise_mixed_b200 import build
    if rank == 0:
        build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    import block_wise_mixed_b200 as mpq
    from block_wise_mixed_b200 import synth

    peaks, peak_src = load_peaks()
    if args.quick:
        layer = synth.config_layer(args.cfg, args.proj)
        M = args.M
        # the timed loop only (for profiler captures of the same command)
        r = time_layer(mpq, layer, M, args.steps, args.warmup, world, device, soak_s=0.0,
                       quick=True)
        if rank == 0:
            print(json.dumps({"quick": True, "cfg": args.cfg, "proj": args.proj, "M": M,
                              "N": layer.N, "K": layer.K, "us_per_step": r["ms_step"] * 1e3,
                              "GBps": r["bytes"] / (r["ms_step"] * 1e-3) / 1e9}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    layer = synth.config_layer(HEADLINE_CFG, 0)
    M = 1
    sampler = ClockSampler(local)
    r = time_layer(mpq, layer, M, args.steps, args.warmup, world, device, sampler=sampler)

    total_bytes = reduce_sum_over_ranks(float(r["bytes"]), world, device)
    value = total_bytes / (r["ms_step"] * 1e-3) / 1e9
    e2e_value = total_bytes / (r["e2e_ms"] * 1e-3) / 1e9
    achieved = r["kernel_bytes"] / (r["kernel_ms"] * 1e-3) / 1e9
    traffic = load_traffic("k_decode", "attn4096_m1")
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "fp16", "data": "synthetic",
        "config": {"workload": "Llama-2-7B attention projection N=K=4096, M=1, avg %.2f bits "
                               "(f0=%.3f), saliency-ordered, mpq_linear" % (r["avg_bits"], r["f0"]),
                   "N": r["N"], "K": r["K"], "M": M, "replicas": r["replicas"],
                   "l2": "inputs larger than L2: %d packed replicas cycled (%.0f MB > 4x L2)"
                         % (r["replicas"], r["replicas"] * r["bytes"] / 1e6),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "kernel": "k_decode", "peak_source": peak_src,
                     "kernel_us": round(r["kernel_ms"] * 1e3, 3),
                     "kernel_bytes": r["kernel_bytes"]},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"]},
        "clocks": r["clocks"],
        "gpu_launches": args.steps * r["launches_per_step"],
        # one call after an L2 flush, launch latency included (not the headline)
        "cold": {"us": round(r["cold_ms"] * 1e3, 2),
                 "GBps": round(r["bytes"] / (r["cold_ms"] * 1e-3) / 1e9, 1)},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        xb = synth.make_x(synth.seed_of(99, 0), M, layer.K)
        res["cpu_baseline"] = oracle_baseline(layer, xb, min_seconds=args.cpu_seconds)
        one = oracle_baseline(layer, xb, min_seconds=args.cpu_seconds, threads=1)
        res["cpu_baseline"]["single_thread"] = {"value": one["value"], "cores": 1,
                                                "sample": one["sample"]}
    if args.extra and rank == 0:
        res["extra"] = run_extra(mpq, args, device, peaks)
        res["extra"]["tensor_core_llama3_8b_layer"] = run_tensor_core(mpq, args, device, peaks)
        # q, k, v of Llama-2-7B (three seeded 4096x4096 layers) in one call
        qkv = [synth.config_layer(2, 0, replica=r) for r in range(3)]
        res["extra"]["group_llama2_7b_qkv_M1"] = time_group(mpq, qkv, min(args.steps, 200), device)
        res["extra"]["pack_llama3_8b_layer"] = run_pack(mpq, device, peaks)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def time_prefill(mpq, L, M, steps, device):
    """Tensor-core path: kernel time (events around the main kernel) and the
    whole mpq_linear step for one layer at M tokens."""
    import torch
    from block_wise_mixed_b200 import synth
    W = torch.from_numpy(L.W.view(np.int16)).to(device)
    P = mpq.pack(W, L.bits, L.row_perm, L.col_perm)
    del W
    lay = P.layout
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    per_rep = lay.codes_bytes + 4 * lay.n_sz
    R = int(max(2, min(64, np.ceil(4 * l2 / max(per_rep, 1)))))
    reps = build_replicas(mpq, P, R)
    x = torch.from_numpy(synth.make_x(synth.seed_of(98, 0), M, L.K).view(np.int16)).to(device)
    y = torch.empty((M, L.N), dtype=torch.float32, device=device)
    ws = torch.zeros(mpq.linear_workspace_size(P, M), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    for i in range(3):
        mpq.linear(reps[i % R], x, y, ws)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for a, b in evs:
        a.record(stream); b.record(stream)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
    torch.cuda._sleep(int(2e6 + 4e4 * steps))   # the host enqueues ahead of the GPU
    e0.record(stream)
    for s_ in range(steps):
        mpq.linear_timed(reps[s_ % R], x, y, ws, evs[s_][0], evs[s_][1])
    e1.record(stream)
    torch.cuda.synchronize(device)
    k_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    step_ms = e0.elapsed_time(e1) / steps
    f0 = float((L.bits == 0).mean())
    flops = 2.0 * M * L.N * L.K * (1.0 - f0)
    del reps
    torch.cuda.empty_cache()
    return dict(name=L.name, N=L.N, K=L.K, M=M, f0=f0, kernel_us=k_ms * 1e3, step_us=step_ms * 1e3,
                flops=flops, dense_flops=2.0 * M * L.N * L.K)


def time_pack(mpq, L, device, reps=3):
    """mpq_pack of one layer: the quantize kernel's time with events (the host
    planning and table uploads happen before the first event and are in the
    wall time only)."""
    import torch
    W = torch.from_numpy(L.W.view(np.int16)).to(device)
    mpq.pack(W, L.bits, L.row_perm, L.col_perm)      # warm-up
    torch.cuda.synchronize(device)
    stream = torch.cuda.current_stream(device)
    ts, walls = [], []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True); b = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        P = mpq.pack(W, L.bits, L.row_perm, L.col_perm, check=False, ev_begin=a, ev_end=b)
        torch.cuda.synchronize(device)
        walls.append(time.perf_counter() - t0)
        ts.append(a.elapsed_time(b))
    lay = P.layout
    nbytes = 2 * L.N * L.K + lay.codes_bytes + 4 * lay.n_sz
    return dict(name=L.name, gpu_us=float(np.median(ts)) * 1e3, wall_ms=float(np.median(walls)) * 1e3,
                bytes=nbytes)


def run_tensor_core(mpq, args, device, peaks, which=None):
    """Llama-3-8B layer at M = 512 and 2048 on the tensor-core path."""
    from block_wise_mixed_b200 import synth
    projs = range(7) if which is None else which
    out = {}
    for M in (512, 2048):
        tot_flops = tot_us = 0.0
        per = {}
        for proj in projs:
            L = synth.config_layer(5, proj)
            r = time_prefill(mpq, L, M, 10, device)
            tot_flops += r["flops"]
            tot_us += r["kernel_us"]
            per[L.name] = {"kernel_us": round(r["kernel_us"], 1), "step_us": round(r["step_us"], 1),
                           "TFLOPs": round(r["flops"] / (r["kernel_us"] * 1e-6) / 1e12, 1)}
        tf = tot_flops / (tot_us * 1e-6) / 1e12
        out["M%d" % M] = {"layer_kernel_us": round(tot_us, 1), "TFLOPs": round(tf, 1),
                          "frac_burst": round(tf / peaks["bf16_tflops"], 4),
                          "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
                          "projections": per}
    return out


def run_pack(mpq, device, peaks):
    from block_wise_mixed_b200 import synth
    tot_us = tot_bytes = 0.0
    per = {}
    for proj in range(7):
        L = synth.config_layer(5, proj)
        r = time_pack(mpq, L, device)
        tot_us += r["gpu_us"]
        tot_bytes += r["bytes"]
        per[L.name] = {"gpu_us": round(r["gpu_us"], 1), "wall_ms": round(r["wall_ms"], 2)}
    gbs = tot_bytes / (tot_us * 1e-6) / 1e9
    return {"layer_gpu_us": round(tot_us, 1), "GBps": round(gbs, 1),
            "frac": round(gbs / peaks["hbm_gbs"], 4), "projections": per}


def time_group(mpq, specs, steps, device):
    """Layers that share x at M=1: mpq_linear_group (one launch when every
    layer's decode builds its own activation records) against one mpq_linear
    per layer, each as a CUDA graph over L2-busting replicas."""
    import torch
    from block_wise_mixed_b200 import synth
    Ps = []
    for L in specs:
        W = torch.from_numpy(L.W.view(np.int16)).to(device)
        Ps.append(mpq.pack(W, L.bits, L.row_perm, L.col_perm))
        del W
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    per = sum(P.layout.codes_bytes + 4 * P.layout.n_sz for P in Ps)
    R = int(max(2, min(256, np.ceil(4 * l2 / max(per, 1)))))
    reps = [build_replicas(mpq, P, R) for P in Ps]
    x = torch.from_numpy(synth.make_x(synth.seed_of(97, 0), 1, specs[0].K).view(np.int16)).to(device)
    ys = [torch.empty((1, L.N), dtype=torch.float32, device=device) for L in specs]
    wsg = torch.zeros(mpq.linear_group_workspace_size(Ps, 1), dtype=torch.uint8, device=device)
    wss = torch.zeros(max(mpq.linear_workspace_size(P, 1) for P in Ps), dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def run(grouped, r):
        layers = [rp[r % R] for rp in reps]
        if grouped:
            mpq.linear_group(layers, x, ys, wsg)
        else:
            for P, y in zip(layers, ys):
                mpq.linear(P, x, y, wss)

    out = {}
    for grouped in (True, False):
        for r in range(5):
            run(grouped, r)
        torch.cuda.synchronize(device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for r in range(steps):
                run(grouped, r)
        graph.replay()
        torch.cuda.synchronize(device)
        e0 = torch.cuda.Event(enable_timing=True); e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream); graph.replay(); e1.record(stream)
        torch.cuda.synchronize(device)
        out["grouped_us" if grouped else "separate_us"] = round(e0.elapsed_time(e1) * 1e3 / steps, 2)
        del graph
    nbytes = sum(algorithmic_bytes(L.N, L.K, 1, P.layout.codes_bytes, P.layout.n_sz,
                                   P.layout.NB * P.layout.KB, L.row_perm is not None,
                                   L.col_perm is not None) for L, P in zip(specs, Ps))
    out["GBps_grouped"] = round(nbytes / (out["grouped_us"] * 1e-6) / 1e9, 1)
    del reps
    torch.cuda.empty_cache()
    return out


def run_extra(mpq, args, device, peaks):
    """Other workloads (context, not the headline): cfg 3 and 4 at M=1."""
    from block_wise_mixed_b200 import synth
    out = {}
    for cfg, proj in [(3, 0), (3, 2), (4, 4), (4, 0)]:
        L = synth.config_layer(cfg, proj)
        for M in synth.CONFIGS[cfg]["M"]:
            r = time_layer(mpq, L, M, min(args.steps, 100), 5, 1, device, soak_s=0.2)
            gbs = r["bytes"] / (r["ms_step"] * 1e-3) / 1e9
            kgbs = r["kernel_bytes"] / (r["kernel_ms"] * 1e-3) / 1e9
            out["cfg%d_%s_M%d" % (cfg, L.name, M)] = {
                "N": L.N, "K": L.K, "avg_bits": round(r["avg_bits"], 3), "us": round(r["ms_step"] * 1e3, 2),
                "GBps": round(gbs, 1), "kernel_us": round(r["kernel_ms"] * 1e3, 2),
                "kernel_GBps": round(kgbs, 1), "frac": round(kgbs / peaks["hbm_gbs"], 3)}
    return out


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle as it stands
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_wise_mixed_b200 import synth
    from oracle import oracle
    layer = synth.config_layer(HEADLINE_CFG, 0)
    M = 1
    x = synth.make_x(synth.seed_of(99, 0), M, layer.K)
    R = oracle.pack(layer.W, layer.bits, layer.row_perm, layer.col_perm)
    rows = np.arange(0, layer.N, 16, dtype=np.int32)   # 1/16 of the outputs per step
    for _ in range(max(args.warmup, 3)):
        oracle.linear_rows(R, x, rows)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.linear_rows(R, x, rows)
    el = time.perf_counter() - t0
    frac = len(rows) / layer.N
    T = (layer.N // 64) * (layer.K // 128)
    nbytes = algorithmic_bytes(layer.N, layer.K, M, R.codes.size * frac, R.scales.size * frac,
                               T * frac, True, True)
    value = nbytes * args.steps / el / 1e9
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = "each step: fp64 oracle linear on %d of %d output rows of the 4096x4096 M=1 layer" % (
        len(rows), layer.N)
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
           "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": "Llama-2-7B attention projection N=K=4096, M=1, avg %.2f bits, "
                                  "fp64 CPU oracle" % layer.bits.mean(), "N": layer.N, "K": layer.K,
                      "M": M},
           "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="mpq", choices=["mpq", "reference"])
    ap.add_argument("--extra", action="store_true", help="also time the other workloads")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--quick", action="store_true",
                    help="timed loop only, no soak/e2e/CPU baseline (for ncu)")
    ap.add_argument("--cfg", type=int, default=HEADLINE_CFG, help="workload for --quick")
    ap.add_argument("--proj", type=int, default=0, help="projection for --quick")
    ap.add_argument("--M", type=int, default=1, help="tokens for --quick")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
