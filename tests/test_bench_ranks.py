"""bench.py's multi-rank plumbing on the CPU: the max / sum reductions over
ranks (gloo, world size 2) and the reference arm under a 2-rank launch
(rank 0 prints the only line, every rank exits 0).  No GPU is used."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _reduce_worker(rank, world, port, out):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method="tcp://127.0.0.1:%d" % port, rank=rank,
                            world_size=world)
    try:
        out[rank] = (bench.reduce_max_over_ranks(1.5 + rank, world),
                     bench.reduce_sum_over_ranks(10.0 * (rank + 1), world))
    finally:
        dist.destroy_process_group()


def test_reduce_over_ranks_gloo():
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    with mp.Manager() as man:
        out = man.dict()
        mp.start_processes(_reduce_worker, args=(world, port, out), nprocs=world,
                           start_method="spawn", join=True)
        got = dict(out)
    # every rank sees the slowest rank's time and the job's total bytes
    assert got == {0: (2.5, 30.0), 1: (2.5, 30.0)}


def test_reduce_single_rank_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks(3.25, 1) == 3.25
    assert bench.reduce_sum_over_ranks(7.0, 1) == 7.0


def _json_lines(text):
    return [json.loads(l) for l in text.splitlines() if l.startswith("{")]


def test_reference_arm_line():
    # the 4096x4096 workload's layer keeps the CPU suite short; the arm's
    # default is the 70B decoder layer
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "2",
                        "--warmup", "3", "--cfg", "2"], cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1
    d = lines[0]
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}


def test_reference_arm_two_ranks():
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py", "--impl",
           "reference", "--gpus", "2", "--steps", "2", "--warmup", "3", "--cfg", "2"]
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = _json_lines(r.stdout)
    assert len(lines) == 1 and lines[0]["impl"] == "reference"
    assert lines[0]["n_gpus"] == 2
