"""Builds libmpq.so (the C-ABI library) in-tree for sm_100a with nvcc."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB = os.path.join(PKG, "libmpq.so")
# The wait-test library: every bounded device wait gives up after 2 ms and
# the producers issue no copies, so calls end with MPQ_ERR_TIMEOUT; used only
# by the timeout test (tests/test_gpu_timeout.py), never by the package.
WAIT_TEST_LIB = os.path.join(PKG, "libmpq_waittest.so")
SOURCES = [os.path.join(PKG, "csrc", "mpq_api.cu")]
NVCC_FLAGS = ["-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
              "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-Xptxas", "-v"]


def _deps():
    return (glob.glob(os.path.join(PKG, "csrc", "*")) +
            [os.path.join(ROOT, "include", "mpq.h")])


def _compile(out: str, extra, verbose: bool) -> None:
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    tmp = out + ".tmp%d" % os.getpid()
    cmd = [nvcc, *NVCC_FLAGS, *extra, "-o", tmp, *SOURCES]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        sys.stderr.write(r.stdout + r.stderr)
        raise RuntimeError("nvcc failed building %s" % os.path.basename(out))
    if verbose:
        sys.stderr.write(r.stderr)
    os.replace(tmp, out)


def _stale(path: str) -> bool:
    return (not os.path.exists(path)
            or os.path.getmtime(path) < max(os.path.getmtime(d) for d in _deps()))


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libmpq.so if missing or older than its sources; returns its path."""
    if force or _stale(LIB):
        _compile(LIB, [], verbose)
    return LIB


def build_wait_test(force: bool = False) -> str:
    """Compile the wait-test library (see WAIT_TEST_LIB); returns its path."""
    if force or _stale(WAIT_TEST_LIB):
        _compile(WAIT_TEST_LIB, ["-DMPQ_WAIT_TEST"], False)
    return WAIT_TEST_LIB


if __name__ == "__main__":
    build(force=True, verbose=True)
    print(LIB)
