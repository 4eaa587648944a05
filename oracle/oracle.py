"""Python access to the fp64 CPU oracle (``mpq_oracle.c``).

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``.  It shares nothing with the CUDA
library and the library never imports it.

``build()`` compiles ``mpq_oracle.c`` with gcc (``-O2``, OpenMP, no fast-math)
into ``oracle/liboracle.so``; the other functions marshal numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mpq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# status codes of the oracle (same meaning as the library's, defined apart)
OK, ERR_ARG, ERR_SHAPE, ERR_BITS, ERR_PERM, ERR_NONFINITE, ERR_RANGE = range(7)
STATUS_NAMES = {0: "OK", 1: "ARG", 2: "SHAPE", 3: "BITS", 4: "PERM",
                5: "NONFINITE", 6: "RANGE"}


def build(force: bool = False) -> str:
    """Compile the oracle shared library if it is missing or stale."""
    hdr = os.path.join(_HERE, "mpq_oracle.h")
    if (not force and os.path.exists(_LIB)
            and os.path.getmtime(_LIB) >= max(os.path.getmtime(_SRC),
                                               os.path.getmtime(hdr))):
        return _LIB
    tmp = _LIB + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-Wall", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


class _Layout(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("NB", ctypes.c_int32), ("KB", ctypes.c_int32),
                ("codes_bytes", ctypes.c_uint64), ("n_sz", ctypes.c_uint64),
                ("bit_total", ctypes.c_uint64),
                ("seg_off", ctypes.c_uint64 * 17),
                ("seg_bytes", ctypes.c_uint64 * 17)]


class _Packed(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("table", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("row_perm", ctypes.c_void_p), ("col_perm", ctypes.c_void_p)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        _lib.mpqo_set_threads.argtypes = [ctypes.c_int]
        _lib.mpqo_plan.argtypes = [i32, i32, P, ctypes.POINTER(_Layout), P]
        _lib.mpqo_quantize_group.argtypes = [P, ctypes.c_int, ctypes.c_int, P, P, P]
        _lib.mpqo_pack.argtypes = [i32, i32, P, P, P, P, P, P, P, P]
        _lib.mpqo_dequant.argtypes = [ctypes.POINTER(_Packed), P]
        _lib.mpqo_dequant.restype = None
        _lib.mpqo_linear_dense.argtypes = [i32, i32, i32, P, P, P, P]
        _lib.mpqo_linear_dense.restype = None
        _lib.mpqo_linear_rows.argtypes = [ctypes.POINTER(_Packed), i32, P, P, i32, P, P]
        _lib.mpqo_linear_rows.restype = None
        _lib.mpqo_f16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.mpqo_f16_to_f64.restype = ctypes.c_double
        _lib.mpqo_bf16_to_f64.argtypes = [ctypes.c_uint16]
        _lib.mpqo_bf16_to_f64.restype = ctypes.c_double
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


class OracleError(RuntimeError):
    def __init__(self, status: int):
        super().__init__("oracle status %s" % STATUS_NAMES.get(status, status))
        self.status = status


@dataclass
class Layout:
    N: int
    K: int
    NB: int
    KB: int
    codes_bytes: int
    n_sz: int
    bit_total: int
    seg_off: list
    seg_bytes: list


@dataclass
class Packed:
    """Packed layer (format v1) in host memory."""
    N: int
    K: int
    codes: np.ndarray      # uint8 [codes_bytes]
    table: np.ndarray      # uint32 [T, 4] = code_off, sz_off, bits, bit_prefix
    scales: np.ndarray     # uint16 (fp16 bits) [n_sz]
    zeros: np.ndarray      # uint16 (fp16 bits) [n_sz]
    row_perm: np.ndarray | None
    col_perm: np.ndarray | None

    def _struct(self):
        return _Packed(self.N, self.K, _ptr(self.codes), _ptr(self.table),
                       _ptr(self.scales), _ptr(self.zeros),
                       _ptr(self.row_perm), _ptr(self.col_perm))


def plan(N: int, K: int, bits: np.ndarray):
    """Block table and segment layout for a bit map (uint8, NB*KB, row-major)."""
    bits = _c(bits, np.uint8).reshape(-1)
    L = _Layout()
    T = max(0, (N // 64) * (K // 128))
    table = np.zeros((max(T, 1), 4), dtype=np.uint32)
    st = lib().mpqo_plan(N, K, _ptr(bits), ctypes.byref(L), _ptr(table))
    if st != OK:
        raise OracleError(st)
    lay = Layout(L.N, L.K, L.NB, L.KB, L.codes_bytes, L.n_sz, L.bit_total,
                 list(L.seg_off), list(L.seg_bytes))
    return lay, table[:T]


def quantize_group(w: np.ndarray, b: int):
    """RTN of one group (float64 values): returns (s_bits, z_bits, q uint8)."""
    w = _c(w, np.float64)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    q = np.zeros(len(w), np.uint8)
    st = lib().mpqo_quantize_group(_ptr(w), len(w), b, _ptr(s), _ptr(z), _ptr(q))
    if st != OK:
        raise OracleError(st)
    return int(s[0]), int(z[0]), q


def pack(W_bf16: np.ndarray, bits: np.ndarray, row_perm=None, col_perm=None) -> Packed:
    """Quantize and pack W (uint16 bf16 bits, N x K, original order)."""
    W = _c(W_bf16, np.uint16)
    N, K = W.shape
    bits = _c(bits, np.uint8).reshape(-1)
    rp = _c(row_perm, np.int32)
    cp = _c(col_perm, np.int32)
    lay, _ = plan(N, K, bits)
    codes = np.zeros(max(lay.codes_bytes, 1), np.uint8)
    table = np.zeros((lay.NB * lay.KB, 4), np.uint32)
    scales = np.zeros(max(lay.n_sz, 1), np.uint16)
    zeros = np.zeros(max(lay.n_sz, 1), np.uint16)
    st = lib().mpqo_pack(N, K, _ptr(W), _ptr(bits), _ptr(rp), _ptr(cp),
                         _ptr(codes), _ptr(table), _ptr(scales), _ptr(zeros))
    if st != OK:
        raise OracleError(st)
    return Packed(N, K, codes[:lay.codes_bytes], table, scales[:lay.n_sz],
                  zeros[:lay.n_sz], rp, cp)


def dequant(P: Packed) -> np.ndarray:
    """Dequantized weights, original order, float64 N x K."""
    out = np.zeros((P.N, P.K), np.float64)
    s = P._struct()
    lib().mpqo_dequant(ctypes.byref(s), _ptr(out))
    return out


def linear_dense(x_bf16: np.ndarray, What: np.ndarray):
    """y = x @ What.T and bound = |x| @ |What|.T in float64 (plain loops)."""
    x = _c(x_bf16, np.uint16)
    What = _c(What, np.float64)
    M, K = x.shape
    N = What.shape[0]
    y = np.zeros((M, N), np.float64)
    bnd = np.zeros((M, N), np.float64)
    lib().mpqo_linear_dense(M, N, K, _ptr(x), _ptr(What), _ptr(y), _ptr(bnd))
    return y, bnd


def linear(P: Packed, x_bf16: np.ndarray):
    """The layer's output for x (bf16 bits, M x K): (y, bound), float64 M x N."""
    return linear_dense(x_bf16, dequant(P))


def set_threads(n: int) -> int:
    """OpenMP threads of the oracle's loops (for timing); returns the previous count."""
    return lib().mpqo_set_threads(int(n))


def linear_rows(P: Packed, x_bf16: np.ndarray, rows: np.ndarray):
    """(y, bound) for the chosen original output rows only: M x len(rows)."""
    x = _c(x_bf16, np.uint16)
    rows = _c(rows, np.int32)
    M = x.shape[0]
    y = np.zeros((M, len(rows)), np.float64)
    bnd = np.zeros((M, len(rows)), np.float64)
    s = P._struct()
    lib().mpqo_linear_rows(ctypes.byref(s), M, _ptr(x), _ptr(rows), len(rows),
                           _ptr(y), _ptr(bnd))
    return y, bnd


def f16_to_f64(h: int) -> float:
    return lib().mpqo_f16_to_f64(h)
