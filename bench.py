#!/usr/bin/env python3
"""Benchmark of the block-wise mixed-precision weight-only linear layer.

Headline step: one Llama-3-70B decoder layer at M=1 (one decode token) --
its seven projections q, k, v, o, gate, up, down (8192 hidden, 28672 MLP,
2.1 average bits, channel orders on all but q and k), each an activation
reorder + mixed-precision GEMV + inverse output reorder; k and v, which
share x, go through one mpq_linear_group call (one launch).  The
steps cycle through replicas of the packed layer whose total size is more
than 4x the L2 cache, and L2 is flushed (a buffer of twice its size is
written) right before the timed replay, so every timed step streams its
weights from HBM whatever the step count.

value = algorithmic HBM bytes of the seven projections / device time of a step
(GB/s, summed over ranks, time = max over ranks).  The same line carries the
tensor-core path on the Llama-3-8B layer at M = 512 and 2048 (TFLOP/s), the
full-layer mpq_pack time and the 4096x4096 (Llama-2-7B attention) layer at
M=1.  Multi-GPU runs are independent replicas (the path has no exchange
step).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mpq|reference]
                  [--extra] [--quick --cfg C --proj P --M M]
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
HEADLINE_CFG = 4          # Llama-3-70B decoder layer, 7 projections, M=1
HEADLINE_M = 1
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


def kernel_bytes(N, K, M, codes_bytes, n_sz, T, has_rp):
    """Algorithmic bytes of the main GEMM kernel of a call: the same without
    the column order (read by the activation prologue)."""
    return codes_bytes + 4 * n_sz + 16 * T + 4 * (N if has_rp else 0) + 2 * M * K + 4 * M * N


def source_hash(names=None):
    """Hash of the kernel sources (all of csrc/, or the listed files)."""
    h = hashlib.sha1()
    d = os.path.join(ROOT, "block_wise_mixed_b200", "csrc")
    for name in sorted(names if names else os.listdir(d)):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_traffic(kernel: str, workload: str):
    """DRAM bytes per step from a committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("source_hash") != source_hash(e.get("sources")):
        return None
    return e.get("dram_bytes_per_step", e.get("dram_bytes_per_launch"))


def launches_per_call(lay, M, has_row_perm, has_16bit=False):
    """Kernels one mpq_linear call launches (the library's dispatch rule):
    M <= 8 -- the activation prologue unless M == 1 on a layer whose runs
    hold at most two blocks on average (the decode kernel then builds its own
    activation records), plus one decode launch; 9..16 tokens on a layer of
    at least 100 tiles of 128 rows without 16-bit blocks -- the record
    prologue and the integer tensor-core kernel; otherwise the prologue, the
    tensor-core kernel and, when the rows are reordered (or k is split), the
    reordering kernel."""
    if M <= 8:
        fused = M == 1 and lay.NB * lay.KB <= 2 * lay.n_units
        return (0 if fused else 1) + (M + 7) // 8
    if M <= 16 and (lay.NB + 1) // 2 >= 100 and not has_16bit:
        return 2
    return 2 + (1 if has_row_perm else 0)


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
        self.proc = None
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
def oracle_packs(layers):
    from oracle import oracle
    return [oracle.pack(L.W, L.bits, L.row_perm, L.col_perm) for L in layers]


def oracle_step_sample(layers, packs, xs, row_stride):
    """One sampled step of the oracle: its linear (dequant + dot, fp64) on
    every row_stride-th output row of each layer.  Returns the algorithmic
    bytes of the sampled part."""
    from oracle import oracle
    nbytes = 0.0
    for L, R, x in zip(layers, packs, xs):
        rows = np.arange(0, L.N, row_stride, dtype=np.int32)
        oracle.linear_rows(R, x, rows)
        frac = len(rows) / L.N
        T = (L.N // 64) * (L.K // 128)
        nbytes += algorithmic_bytes(L.N, L.K, x.shape[0], R.codes.size * frac, R.scales.size * frac,
                                    T * frac, L.row_perm is not None, L.col_perm is not None)
    return nbytes


def oracle_baseline(layers, packs, xs, row_stride, min_seconds=10.0, threads=None):
    """The oracle's sampled step timed on the host: all cores (threads=None)
    or a given number of OpenMP threads."""
    from oracle import oracle
    prev = oracle.set_threads(threads) if threads else None
    n, nbytes = 0, 0.0
    t0 = time.perf_counter()
    while True:
        nbytes += oracle_step_sample(layers, packs, xs, row_stride)
        n += 1
        el = time.perf_counter() - t0
        if el >= min_seconds:
            break
    if prev is not None:
        oracle.set_threads(prev)
    cores = threads or int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    return {"value": nbytes / el / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": "%d passes of the fp64 oracle's linear (dequant + dot) on every %dth output "
                      "row of each of the %d projections, %.1f s" % (n, row_stride, len(layers), el)}


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def clone_layer(P):
    """A deep copy of a packed layer (distinct device addresses)."""
    from block_wise_mixed_b200 import _lib
    c = {k: (getattr(P, k).clone() if getattr(P, k) is not None else None)
         for k in ("codes", "table", "sched", "scales", "zeros", "row_perm", "col_perm")}
    layer = _lib.Layer(P.c.N, P.c.K, P.c.n_units, P.c.flags, c["codes"].data_ptr(),
                       c["table"].data_ptr(), c["sched"].data_ptr(), c["scales"].data_ptr(),
                       c["zeros"].data_ptr(),
                       c["row_perm"].data_ptr() if c["row_perm"] is not None else None,
                       c["col_perm"].data_ptr() if c["col_perm"] is not None else None)
    return _lib.PackedLayer(P.layout, c["codes"], c["table"], c["sched"], c["scales"],
                            c["zeros"], c["row_perm"], c["col_perm"], layer)


def packed_bytes(P):
    lay = P.layout
    return lay.codes_bytes + 4 * lay.n_sz + 16 * lay.NB * lay.KB + 4 * (lay.N + lay.K)


# The decoder layer's calls: q, then k and v as one mpq_linear_group call
# (they share x; at M=1 both take the one-token path, so the group is one
# launch), o, gate, up, down.  x sources as in the model: q, k, v read the
# normed hidden state, o the attention output, gate and up the normed hidden
# state of the MLP, down the MLP activation.
DECODER_GROUPS = [[0], [1, 2], [3], [4], [5], [6]]
DECODER_X_SRC = [0, 0, 0, 1, 2, 2, 3]


def headline_desc(layers):
    """The headline workload, as both arms name it in `config`."""
    avg_bits = float(np.mean(np.concatenate([L.bits for L in layers])))
    f0 = float(np.mean(np.concatenate([L.bits == 0 for L in layers])))
    return ("Llama-3-70B decoder layer at M=1: q 8192x8192, k,v 1024x8192, "
            "o 8192x8192, gate,up 28672x8192, down 8192x28672 (856 M weights), "
            "avg %.2f bits (f0=%.3f), saliency channel orders (identity for q,k); "
            "one step = q, k+v (one mpq_linear_group call), o, gate, up, down; "
            "q, k, v share x, gate and up share x" % (avg_bits, f0))


class Workload:
    """A step of mpq_linear calls at M tokens -- one per layer, or one
    mpq_linear_group call per entry of `groups` -- over replicas of the
    packed layers whose total size is at least 4x L2.  x_src[i] names the
    activation that layer i reads (layers with the same source share it)."""

    def __init__(self, mpq, layers, M, device, seed=99, max_replicas=64, groups=None, x_src=None):
        import torch
        from block_wise_mixed_b200 import synth
        self.mpq, self.layers, self.M, self.device = mpq, layers, M, device
        self.packs = []
        for L in layers:
            W = torch.from_numpy(L.W.view(np.int16)).to(device)
            self.packs.append(mpq.pack(W, L.bits, L.row_perm, L.col_perm))
            del W
        self.l2 = torch.cuda.get_device_properties(device).L2_cache_size
        per_step = sum(packed_bytes(P) for P in self.packs)
        self.R = int(max(2, min(max_replicas, np.ceil(4 * self.l2 / max(per_step, 1)))))
        self.reps = [self.packs] + [[clone_layer(P) for P in self.packs] for _ in range(self.R - 1)]
        self.groups = groups if groups is not None else [[i] for i in range(len(layers))]
        x_src = x_src if x_src is not None else list(range(len(layers)))
        srcs = {}
        for i, L in enumerate(layers):
            if x_src[i] not in srcs:
                srcs[x_src[i]] = synth.make_x(synth.seed_of(seed, x_src[i]), M, L.K)
        self.x_bits = [srcs[x_src[i]] for i in range(len(layers))]
        xdev = {k: torch.from_numpy(v.view(np.int16)).to(device) for k, v in srcs.items()}
        self.x = [xdev[x_src[i]] for i in range(len(layers))]
        self.y = [torch.empty((M, L.N), dtype=torch.float32, device=device) for L in layers]
        self.ws = torch.zeros(max(mpq.linear_workspace_size(P, M) for P in self.packs),
                              dtype=torch.uint8, device=device)
        self.gws = {tuple(g): torch.zeros(mpq.linear_group_workspace_size([self.packs[i] for i in g], M),
                                          dtype=torch.uint8, device=device)
                    for g in self.groups if len(g) > 1}
        self.flush = torch.empty(2 * self.l2, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(device)
        lays = [P.layout for P in self.packs]
        self.bytes = sum(algorithmic_bytes(L.N, L.K, M, l.codes_bytes, l.n_sz, l.NB * l.KB,
                                           L.row_perm is not None, L.col_perm is not None)
                         for L, l in zip(layers, lays))
        self.kbytes = sum(kernel_bytes(L.N, L.K, M, l.codes_bytes, l.n_sz, l.NB * l.KB,
                                       L.row_perm is not None) for L, l in zip(layers, lays))
        self.flops = sum(2.0 * M * L.N * L.K * (1.0 - float((L.bits == 0).mean())) for L in layers)
        self.dense_flops = sum(2.0 * M * L.N * L.K for L in layers)
        self.launches = 0
        for g in self.groups:
            per = [launches_per_call(lays[i], M, layers[i].row_perm is not None,
                                     bool((layers[i].bits == 16).any())) for i in g]
            one_launch = len(g) > 1 and M == 1 and all(
                lays[i].NB * lays[i].KB <= 2 * lays[i].n_units for i in g)
            self.launches += 1 if one_launch else sum(per)
        self.footprint = self.R * per_step

    def step(self, r):
        rep = self.reps[r % self.R]
        for g in self.groups:
            if len(g) == 1:
                i = g[0]
                self.mpq.linear(rep[i], self.x[i], self.y[i], self.ws)
            else:
                self.mpq.linear_group([rep[i] for i in g], self.x[g[0]], [self.y[i] for i in g],
                                      self.gws[tuple(g)])

    def flush_l2(self):
        self.flush.fill_(1)

    def time_steps(self, steps, warmup, world, sampler=None, soak_s=1.0):
        """Device time per step: `steps` steps captured as one CUDA graph,
        replayed once after an L2 flush, between CUDA events."""
        import torch
        dev, stream = self.device, torch.cuda.current_stream(self.device)
        for i in range(max(warmup, 3)):
            self.step(i)
        torch.cuda.synchronize(dev)
        if sampler:
            sampler.start()
        t_end = time.perf_counter() + soak_s
        i = 0
        while time.perf_counter() < t_end:
            for _ in range(20):
                self.step(i)
                i += 1
            torch.cuda.synchronize(dev)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for s in range(steps):
                self.step(s)
        graph.replay()
        self.flush_l2()
        torch.cuda.synchronize(dev)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        torch.cuda.synchronize(dev)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
        clocks = sampler.stop() if sampler else None
        del graph
        return reduce_max_over_ranks(e0.elapsed_time(e1), world, dev) / steps, clocks

    def time_kernels(self, steps):
        """Device time of the main GEMM kernels alone per step: events that
        the library records around them (mpq_linear_timed), the calls queued
        behind a spin kernel so the events see device time only, L2 flushed
        first.  Returns (ms per step, [ms per call of each layer])."""
        import torch
        dev, stream = self.device, torch.cuda.current_stream(self.device)
        n = len(self.layers)
        evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                for _ in range(n)] for _ in range(steps)]
        for row in evs:          # torch creates the CUDA events on first record
            for a, b in row:
                a.record(stream)
                b.record(stream)
        self.flush_l2()
        torch.cuda.synchronize(dev)
        torch.cuda._sleep(int(2e6 + 4e4 * steps * n))   # ~1 ms + 20 us per enqueued call
        for s in range(steps):
            for i, (P, x, y) in enumerate(zip(self.reps[s % self.R], self.x, self.y)):
                self.mpq.linear_timed(P, x, y, self.ws, evs[s][i][0], evs[s][i][1])
        torch.cuda.synchronize(dev)
        per = np.array([[a.elapsed_time(b) for a, b in row] for row in evs])
        return float(per.sum(axis=1).mean()), per.mean(axis=0).tolist()

    def time_e2e(self, steps, world):
        """The same step through mpq_linear_host: pinned host x in, host y
        out, copies inside the timed region."""
        import torch
        dev, stream = self.device, torch.cuda.current_stream(self.device)
        xh = [torch.from_numpy(xb.view(np.int16)).pin_memory() for xb in self.x_bits]
        yh = [torch.empty((self.M, L.N), dtype=torch.float32).pin_memory() for L in self.layers]
        wsh = torch.zeros(max(self.mpq.linear_host_workspace_size(P, self.M) for P in self.packs),
                          dtype=torch.uint8, device=dev)

        def run(r):
            for P, a, b in zip(self.reps[r % self.R], xh, yh):
                self.mpq.linear_host(P, a, b, wsh)

        for i in range(3):
            run(i)
        self.flush_l2()
        torch.cuda.synchronize(dev)
        h0 = torch.cuda.Event(enable_timing=True)
        h1 = torch.cuda.Event(enable_timing=True)
        h0.record(stream)
        for s in range(steps):
            run(s)
        h1.record(stream)
        torch.cuda.synchronize(dev)
        ms = reduce_max_over_ranks(h0.elapsed_time(h1), world, dev) / steps
        h2d = sum(self.M * L.K * 2 for L in self.layers)
        d2h = sum(self.M * L.N * 4 for L in self.layers)
        return ms, h2d, d2h

    def release(self):
        import torch
        self.reps = self.packs = self.flush = self.ws = None
        torch.cuda.empty_cache()


def time_pack(mpq, L, device, reps=3):
    """mpq_pack of one layer: the quantize kernel's time with events (the host
    planning and table uploads happen before the first event and are in the
    wall time only)."""
    import torch
    W = torch.from_numpy(L.W.view(np.int16)).to(device)
    mpq.pack(W, L.bits, L.row_perm, L.col_perm)      # warm-up
    torch.cuda.synchronize(device)
    ts, walls = [], []
    for _ in range(reps):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        P = mpq.pack(W, L.bits, L.row_perm, L.col_perm, check=False, ev_begin=a, ev_end=b)
        torch.cuda.synchronize(device)
        walls.append(time.perf_counter() - t0)
        ts.append(a.elapsed_time(b))
    lay = P.layout
    nbytes = 2 * L.N * L.K + lay.codes_bytes + 4 * lay.n_sz
    del W, P
    return dict(name=L.name, gpu_us=float(np.median(ts)) * 1e3, wall_ms=float(np.median(walls)) * 1e3,
                bytes=nbytes)


def run_pack(mpq, layers, device, peaks):
    tot_us = tot_bytes = 0.0
    per = {}
    for L in layers:
        r = time_pack(mpq, L, device)
        tot_us += r["gpu_us"]
        tot_bytes += r["bytes"]
        per[L.name] = {"gpu_us": round(r["gpu_us"], 1), "wall_ms": round(r["wall_ms"], 2)}
    gbs = tot_bytes / (tot_us * 1e-6) / 1e9
    return {"workload": "mpq_pack of the Llama-3-8B layer (7 projections, 218 M weights, avg 4.0 "
                        "bits): quantize kernel between CUDA events",
            "layer_gpu_us": round(tot_us, 1), "GBps": round(gbs, 1),
            "frac": round(gbs / peaks["hbm_gbs"], 4), "bytes": int(tot_bytes), "projections": per}


def run_tensor_core(mpq, layers, device, peaks, steps):
    """Llama-3-8B layer at M = 512 and 2048 on the tensor-core path."""
    out = {}
    for M in (512, 2048):
        wl = Workload(mpq, layers, M, device, seed=98)
        ms, _ = wl.time_steps(steps, 3, 1, soak_s=0.0)
        k_ms, per = wl.time_kernels(steps)
        tf = wl.flops / (k_ms * 1e-3) / 1e12
        out["M%d" % M] = {
            "step_us": round(ms * 1e3, 1), "kernel_us": round(k_ms * 1e3, 1),
            "TFLOPs": round(tf, 1), "TFLOPs_step": round(wl.flops / (ms * 1e-3) / 1e12, 1),
            "dense_equiv_TFLOPs": round(wl.dense_flops / (k_ms * 1e-3) / 1e12, 1),
            "frac_burst": round(tf / peaks["bf16_tflops"], 4),
            "frac_sustained": round(tf / peaks["bf16_tflops_sustained"], 4),
            "projections_kernel_us": {L.name: round(t * 1e3, 1) for L, t in zip(layers, per)},
            "replicas": wl.R}
        wl.release()
    return out


def run_mid_batch(mpq, device, peaks, steps):
    """Mid-size batches on the 8B MLP gate (14336x4096, 3.0 bits) and the
    70B gate (28672x8192, 2.1 bits) at 16 tokens (the integer tensor-core
    kernel) and 32 (the fp16 one): HBM GB/s of one call, replicas cycled,
    L2 flushed before the timed replay.  A failure is reported in the line
    instead of ending the run."""
    from block_wise_mixed_b200 import synth
    out = {}
    for cfg, proj, name in ((3, 0, "llama3_8b_gate"), (4, 4, "llama3_70b_gate")):
        try:
            L = synth.config_layer(cfg, proj)
            for M in (16, 32):
                wl = Workload(mpq, [L], M, device)
                ms, _ = wl.time_steps(steps, 3, 1, soak_s=0.0)
                gbs = wl.bytes / (ms * 1e-3) / 1e9
                out["%s_M%d" % (name, M)] = {"us": round(ms * 1e3, 1), "GBps": round(gbs, 1),
                                             "frac": round(gbs / peaks["hbm_gbs"], 4), "replicas": wl.R}
                wl.release()
                del wl
            del L
        except Exception as ex:   # keep the rest of the line
            out[name] = {"error": repr(ex)[:200]}
    return out


def run_allocation(mpq, device, peaks):
    """Budgeted bit allocation (mpq_allocate_bits) over the block count of the
    Llama-3-70B decoder layer: device time with CUDA events, search
    iterations, and the oracle's time for the same search on the host."""
    import torch
    from block_wise_mixed_b200 import synth
    from oracle import alloc
    T = sum((N // 64) * (K // 128) for _, N, K in synth.LLAMA3_70B)
    rng = np.random.default_rng(2024)
    loss = alloc.synthetic_loss(rng.lognormal(0.0, 2.0, T))
    budget = int(round(2.1 * T))
    ld = torch.from_numpy(loss).to(device)
    mpq.allocate_bits(ld, (0, 1, 2, 3, 4, 5, 6, 8), budget)      # warm-up
    ts = []
    for _ in range(5):
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record()
        bits, it, tot = mpq.allocate_bits(ld, (0, 1, 2, 3, 4, 5, 6, 8), budget)
        b.record()
        torch.cuda.synchronize(device)
        ts.append(a.elapsed_time(b))
    t0 = time.perf_counter()
    w, it_o, _ = alloc.allocate(loss, (0, 1, 2, 3, 4, 5, 6, 8), budget)
    t_o = time.perf_counter() - t0
    return {"workload": "bit allocation over the %d blocks of the Llama-3-70B decoder layer, "
                        "avg 2.1 bits, synthetic sensitivity surrogates" % T,
            "blocks": T, "budget_bits": budget, "total_bits": tot, "iterations": it,
            "us": round(float(np.median(ts)) * 1e3, 1),
            "matches_oracle": bool(np.array_equal(bits.cpu().numpy(), w) and it == it_o),
            "oracle_numpy_s": round(t_o, 3)}


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
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
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
        # the timed loop only (for profiler captures of the same command)
        cfg = HEADLINE_CFG if args.cfg is None else args.cfg
        layer = synth.config_layer(cfg, args.proj)
        wl = Workload(mpq, [layer], args.M, device)
        ms, _ = wl.time_steps(args.steps, args.warmup, world, soak_s=0.0)
        if rank == 0:
            print(json.dumps({"quick": True, "cfg": cfg, "proj": args.proj, "M": args.M,
                              "N": layer.N, "K": layer.K, "us_per_step": ms * 1e3,
                              "GBps": wl.bytes / (ms * 1e-3) / 1e9}), flush=True)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if args.layer_quick:
        # the headline step's timed loop only (for the launch list)
        layers = [synth.config_layer(HEADLINE_CFG, p) for p in range(7)]
        wl = Workload(mpq, layers, HEADLINE_M, device, groups=DECODER_GROUPS, x_src=DECODER_X_SRC)
        ms, _ = wl.time_steps(args.steps, args.warmup, world, soak_s=0.0)
        if rank == 0:
            print(json.dumps({"layer_quick": True, "us_per_step": ms * 1e3,
                              "GBps": wl.bytes / (ms * 1e-3) / 1e9}), flush=True)
        return

    layers = [synth.config_layer(HEADLINE_CFG, p) for p in range(7)]
    wl = Workload(mpq, layers, HEADLINE_M, device, groups=DECODER_GROUPS, x_src=DECODER_X_SRC)
    sampler = ClockSampler(local)
    ms_step, clocks = wl.time_steps(args.steps, args.warmup, world, sampler=sampler)
    k_ms, k_per = wl.time_kernels(args.steps)
    e2e_ms, h2d, d2h = wl.time_e2e(args.steps, world)
    total_bytes = reduce_sum_over_ranks(float(wl.bytes), world, device)
    value = total_bytes / (ms_step * 1e-3) / 1e9
    e2e_value = total_bytes / (e2e_ms * 1e-3) / 1e9
    # the dominant kernel's rate, from the step itself: the decode launches
    # are >= 90 % of a step (the profile's launch list), and their events
    # taken one call at a time (k_ms) lose the launch overlap, so the step
    # time is the conservative denominator and can never exceed the step
    achieved = wl.kbytes / (ms_step * 1e-3) / 1e9
    traffic = load_traffic("k_decode", "llama70b_layer_m1")
    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "int8", "data": "synthetic",
        "config": {"workload": headline_desc(layers),
                   "M": HEADLINE_M, "layer_bytes": int(wl.bytes), "replicas": wl.R,
                   "l2": "inputs larger than L2: %d replicas of the packed layer cycled (%.0f MB, "
                         "L2 %.0f MB), L2 flushed before the timed replay"
                         % (wl.R, wl.footprint / 1e6, wl.l2 / 1e6),
                   "parallelism": "replicas" if world > 1 else "single"},
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": traffic,
                     "kernel": "k_decode, k_decode_group (the 6 decode launches of a step)",
                     "peak_source": peak_src,
                     "kernel_us_per_step": round(ms_step * 1e3, 2),
                     "kernel_bytes_per_step": int(wl.kbytes),
                     "frac_of_8TBps_nominal": round(achieved / 8000.0, 4),
                     "isolated_kernel_us_per_step": round(k_ms * 1e3, 2),
                     "isolated_projections_kernel_us": {L.name: round(t * 1e3, 2)
                                                        for L, t in zip(layers, k_per)}},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "clocks": clocks,
        "gpu_launches": args.steps * wl.launches,
    }
    x_bits = wl.x_bits
    wl.release()
    del wl
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        packs = oracle_packs(layers)
        res["cpu_baseline"] = oracle_baseline(layers, packs, x_bits, 64, args.cpu_seconds)
        one = oracle_baseline(layers, packs, x_bits, 512, args.cpu_seconds / 2, threads=1)
        res["cpu_baseline"]["single_thread"] = {"value": one["value"], "cores": 1,
                                                "sample": one["sample"]}
        del packs
    del layers
    if rank == 0 and world == 1 and not args.headline_only:
        # the other metric half and the other workloads, on the same box
        l8b = [synth.config_layer(5, p) for p in range(7)]
        res["tensor_core_llama3_8b_layer"] = run_tensor_core(mpq, l8b, device, peaks,
                                                             min(args.steps, 20))
        res["pack_llama3_8b_layer"] = run_pack(mpq, l8b, device, peaks)
        res["bit_allocation"] = run_allocation(mpq, device, peaks)
        del l8b
        attn = Workload(mpq, [synth.config_layer(2, 0)], 1, device)
        ms, _ = attn.time_steps(max(args.steps, 64), 3, 1, soak_s=0.0)
        res["llama2_7b_attn_4096_M1"] = {"us": round(ms * 1e3, 2),
                                         "GBps": round(attn.bytes / (ms * 1e-3) / 1e9, 1),
                                         "frac": round(attn.bytes / (ms * 1e-3) / 1e9 /
                                                       peaks["hbm_gbs"], 4)}
        attn.release()
        res["mid_batch"] = run_mid_batch(mpq, device, peaks, max(min(args.steps, 50), 16))
    if args.extra and rank == 0:
        res["extra"] = run_extra(mpq, args, device, peaks)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(res), flush=True)


def run_extra(mpq, args, device, peaks):
    """Other workloads (context): every projection of cfg 3 and 4 at each M."""
    from block_wise_mixed_b200 import synth
    out = {}
    for cfg in (3, 4):
        for proj in range(len(synth.CONFIGS[cfg]["layers"])):
            L = synth.config_layer(cfg, proj)
            for M in synth.CONFIGS[cfg]["M"]:
                wl = Workload(mpq, [L], M, device)
                ms, _ = wl.time_steps(min(args.steps, 50), 3, 1, soak_s=0.0)
                k_ms, _ = wl.time_kernels(min(args.steps, 50))
                out["cfg%d_%s_M%d" % (cfg, L.name, M)] = {
                    "N": L.N, "K": L.K, "avg_bits": round(float(L.bits.mean()), 3),
                    "us": round(ms * 1e3, 2), "GBps": round(wl.bytes / (ms * 1e-3) / 1e9, 1),
                    "kernel_us": round(k_ms * 1e3, 2),
                    "frac": round(wl.kbytes / (k_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
                wl.release()
    return out


# ---------------------------------------------------------------------------
# reference arm: the fp64 CPU oracle as it stands
# ---------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from block_wise_mixed_b200 import synth
    cfg = HEADLINE_CFG if args.cfg is None else args.cfg     # --cfg: another workload's layers
    layers = [synth.config_layer(cfg, p) for p in range(len(synth.CONFIGS[cfg]["layers"]))]
    if cfg == HEADLINE_CFG:   # the same activations as the GPU arm's step
        src = {j: synth.make_x(synth.seed_of(99, j), HEADLINE_M, layers[DECODER_X_SRC.index(j)].K)
               for j in sorted(set(DECODER_X_SRC))}
        xs = [src[DECODER_X_SRC[i]] for i in range(len(layers))]
    else:
        xs = [synth.make_x(synth.seed_of(99, i), HEADLINE_M, L.K) for i, L in enumerate(layers)]
    packs = oracle_packs(layers)
    stride = 64      # each step: 1/64 of the output rows of every projection
    for _ in range(max(args.warmup, 3)):
        oracle_step_sample(layers, packs, xs, stride)
    t0 = time.perf_counter()
    nbytes = 0.0
    for _ in range(args.steps):
        nbytes += oracle_step_sample(layers, packs, xs, stride)
    el = time.perf_counter() - t0
    value = nbytes / el / 1e9
    cores = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    sample = ("each step: the fp64 oracle's linear on every %dth output row of the %d projections "
              "of workload %d at M=1" % (stride, len(layers), cfg))
    res = {"impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "GB/s",
           "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": (headline_desc(layers) if cfg == HEADLINE_CFG else
                                   "%s at M=1" % synth.CONFIGS[cfg]["desc"]),
                      "M": HEADLINE_M,
                      "oracle_sample": "fp64 CPU oracle on 1/%d of the output rows" % stride},
           "cpu_baseline": {"value": round(value, 6), "unit": "GB/s", "cores": cores,
                            "kind": "oracle", "sample": sample},
           "e2e": {"value": round(value, 6), "unit": "GB/s", "h2d_bytes_per_step": 0,
                   "d2h_bytes_per_step": 0}}
    print(json.dumps(res), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="mpq", choices=["mpq", "reference"])
    ap.add_argument("--extra", action="store_true", help="also time every cfg 3/4 projection")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--headline-only", action="store_true",
                    help="skip the tensor-core, pack and 4096x4096 fields")
    ap.add_argument("--quick", action="store_true",
                    help="timed loop of one layer only, no soak/e2e/CPU baseline (for ncu)")
    ap.add_argument("--layer-quick", action="store_true",
                    help="timed loop of the headline step only (for the ncu launch list)")
    ap.add_argument("--cfg", type=int, default=None,
                    help="workload for --quick (default the 70B layer) and the reference arm")
    ap.add_argument("--proj", type=int, default=4, help="projection for --quick")
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
