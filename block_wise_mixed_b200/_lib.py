"""ctypes binding of libmpq.so (C ABI in include/mpq.h).

Argument marshalling only: every step of the computation runs in the CUDA
library.  PyTorch supplies device memory and the current stream.  There is no
fallback: if libmpq.so is missing the calls raise.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import numpy as np

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmpq.so")
HEADER = os.path.join(os.path.dirname(PKG), "include", "mpq.h")

STATUS = {0: "MPQ_OK", 1: "MPQ_ERR_ARG", 2: "MPQ_ERR_SHAPE", 3: "MPQ_ERR_BITS",
          4: "MPQ_ERR_PERM", 5: "MPQ_ERR_NONFINITE", 6: "MPQ_ERR_RANGE",
          7: "MPQ_ERR_WORKSPACE", 8: "MPQ_ERR_CUDA", 9: "MPQ_ERR_TIMEOUT"}


class MpqError(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        super().__init__("%s%s" % (STATUS.get(status, status), (" in " + where) if where else ""))
        self.status = status
        self.name = STATUS.get(status, str(status))


class Block(ctypes.Structure):
    _fields_ = [("code_off", ctypes.c_uint32), ("sz_off", ctypes.c_uint32),
                ("bits", ctypes.c_uint32), ("bit_prefix", ctypes.c_uint32)]


class Layout(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("NB", ctypes.c_int32),
                ("KB", ctypes.c_int32), ("n_units", ctypes.c_int32),
                ("sched_words", ctypes.c_int32), ("codes_bytes", ctypes.c_uint64),
                ("n_sz", ctypes.c_uint64), ("bit_total", ctypes.c_uint64),
                ("seg_off", ctypes.c_uint64 * 17), ("seg_bytes", ctypes.c_uint64 * 17)]


class Layer(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int32), ("K", ctypes.c_int32), ("n_units", ctypes.c_int32),
                ("flags", ctypes.c_int32), ("codes", ctypes.c_void_p),
                ("table", ctypes.c_void_p), ("sched", ctypes.c_void_p),
                ("scales", ctypes.c_void_p), ("zeros", ctypes.c_void_p),
                ("row_perm", ctypes.c_void_p), ("col_perm", ctypes.c_void_p)]


_lib = None


def header_functions() -> list[str]:
    """Names of the functions declared in include/mpq.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return re.findall(r"\b(mpq_[a-z_]+)\s*\(", txt)


def lib():
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libmpq.so not found at %s: build it with "
                               "block_wise_mixed_b200.build.build()" % LIB_PATH)
        _lib = load(LIB_PATH)
    return _lib


def load(path: str):
    """A ctypes handle on a build of the library at `path`, with the C ABI's
    argument and result types declared."""
    L = ctypes.CDLL(path)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    class _Decl:
        """Declares argument/result types of exported functions; a build
        that lacks one (an older library loaded for comparison) keeps the
        rest usable, and the missing call fails when used."""
        def __init__(self, lib):
            self.lib = lib

        def __getattr__(self, name):
            f = getattr(self.lib, name, None)
            return f if f is not None else _Missing()

    class _Missing:
        def __setattr__(self, k, v):
            pass

    D = _Decl(L)
    D.mpq_plan.argtypes = [i32, i32, P, ctypes.POINTER(Layout)]
    D.mpq_plan_schedule.argtypes = [ctypes.POINTER(Layout), P, P]
    D.mpq_pack_workspace_size.argtypes = [ctypes.POINTER(Layout)]
    D.mpq_pack_workspace_size.restype = sz
    D.mpq_pack.argtypes = [ctypes.POINTER(Layout), P, P, P, P, ctypes.POINTER(Layer), P, sz, P]
    D.mpq_pack_timed.argtypes = [ctypes.POINTER(Layout), P, P, P, P, ctypes.POINTER(Layer), P, sz, P,
                                 P, P]
    D.mpq_linear_workspace_size.argtypes = [ctypes.POINTER(Layer), i32]
    D.mpq_linear_workspace_size.restype = sz
    D.mpq_linear.argtypes = [ctypes.POINTER(Layer), P, i32, P, P, sz, P]
    D.mpq_linear_timed.argtypes = [ctypes.POINTER(Layer), P, i32, P, P, sz, P, P, P]
    D.mpq_linear_typed_workspace_size.argtypes = [ctypes.POINTER(Layer), i32, ctypes.c_int]
    D.mpq_linear_typed_workspace_size.restype = sz
    D.mpq_linear_typed.argtypes = [ctypes.POINTER(Layer), P, i32, P, ctypes.c_int, P, sz, P]
    D.mpq_linear_group_workspace_size.argtypes = [ctypes.POINTER(Layer), i32, i32]
    D.mpq_linear_group_workspace_size.restype = sz
    D.mpq_linear_group.argtypes = [ctypes.POINTER(Layer), i32, P, i32, P, P, sz, P]
    D.mpq_linear_host_workspace_size.argtypes = [ctypes.POINTER(Layer), i32]
    D.mpq_linear_host_workspace_size.restype = sz
    D.mpq_linear_host.argtypes = [ctypes.POINTER(Layer), P, i32, P, P, sz, P]
    D.mpq_linear_noalloc.argtypes = [ctypes.POINTER(Layer), P, i32, P, P]
    D.mpq_linear_noalloc.restype = ctypes.c_int
    D.mpq_noalloc_check.argtypes = [P]
    D.mpq_noalloc_check.restype = ctypes.c_int
    D.mpq_allocate_bits_workspace_size.argtypes = [ctypes.c_int64]
    D.mpq_allocate_bits_workspace_size.restype = sz
    D.mpq_allocate_bits.argtypes = [ctypes.c_int64, P, ctypes.c_uint32, ctypes.c_uint64, P, P, P, sz, P]
    D.mpq_allocate_bits.restype = ctypes.c_int
    D.mpq_fold_orders.argtypes = [i32, P, P, P]
    D.mpq_fold_orders.restype = ctypes.c_int
    D.mpq_check.argtypes = [P, P]
    D.mpq_status_string.argtypes = [ctypes.c_int]
    D.mpq_status_string.restype = ctypes.c_char_p
    for f in ("mpq_plan", "mpq_pack", "mpq_pack_timed", "mpq_linear", "mpq_linear_typed",
              "mpq_linear_group", "mpq_linear_timed", "mpq_linear_host",
              "mpq_check"):
        getattr(D, f).restype = ctypes.c_int
    return L


def _np_ptr(a):
    return None if a is None else a.ctypes.data


def _t_ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _raise(st, where):
    if st != 0:
        raise MpqError(st, where)


def plan(N: int, K: int, bits: np.ndarray) -> Layout:
    """mpq_plan: layout of a packed layer (host only)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8).reshape(-1)
    L = Layout()
    _raise(lib().mpq_plan(N, K, _np_ptr(bits), ctypes.byref(L)), "mpq_plan")
    return L


def plan_schedule(L: Layout, bits: np.ndarray) -> np.ndarray:
    """mpq_plan_schedule: the decode schedule mpq_pack stores (host only)."""
    bits = np.ascontiguousarray(bits, dtype=np.uint8).reshape(-1)
    out = np.zeros(L.sched_words, np.uint32)
    _raise(lib().mpq_plan_schedule(ctypes.byref(L), _np_ptr(bits), _np_ptr(out)), "mpq_plan_schedule")
    return out


@dataclass
class PackedLayer:
    """A packed layer in device memory (torch tensors) plus its C view."""
    layout: Layout
    codes: object
    table: object
    sched: object
    scales: object
    zeros: object
    row_perm: object
    col_perm: object
    c: Layer

    @property
    def N(self):
        return self.layout.N

    @property
    def K(self):
        return self.layout.K


def alloc_layer(L: Layout, device, has_row_perm: bool, has_col_perm: bool) -> PackedLayer:
    import torch
    u8 = torch.uint8

    def buf(n, dtype=u8):
        return torch.empty(max(int(n), 16), dtype=dtype, device=device)

    T = L.NB * L.KB
    codes = buf(L.codes_bytes)
    table = buf(T * 16)
    sched = buf(L.sched_words * 4)
    scales = buf(2 * L.n_sz)
    zeros = buf(2 * L.n_sz)
    rp = torch.empty(L.N, dtype=torch.int32, device=device) if has_row_perm else None
    cp = torch.empty(L.K, dtype=torch.int32, device=device) if has_col_perm else None
    c = Layer(L.N, L.K, L.n_units, LAYER_16BIT if L.seg_bytes[16] else 0, codes.data_ptr(),
              table.data_ptr(), sched.data_ptr(),
              scales.data_ptr(), zeros.data_ptr(),
              rp.data_ptr() if rp is not None else None,
              cp.data_ptr() if cp is not None else None)
    return PackedLayer(L, codes, table, sched, scales, zeros, rp, cp, c)


def pack(W, bits: np.ndarray, row_perm=None, col_perm=None, ws=None, check=True,
         stream=None, ev_begin=None, ev_end=None) -> PackedLayer:
    """mpq_pack (mpq_pack_timed when torch.cuda.Event objects are given: they
    bracket the quantize kernel alone).  W: torch bf16 (or int16/uint16 bit
    patterns) N x K on cuda."""
    import torch
    N, K = W.shape
    bits = np.ascontiguousarray(bits, dtype=np.uint8).reshape(-1)
    rp = None if row_perm is None else np.ascontiguousarray(row_perm, dtype=np.int32)
    cp = None if col_perm is None else np.ascontiguousarray(col_perm, dtype=np.int32)
    L = plan(N, K, bits)
    P = alloc_layer(L, W.device, rp is not None, cp is not None)
    if ws is None:
        ws = torch.empty(lib().mpq_pack_workspace_size(ctypes.byref(L)), dtype=torch.uint8,
                         device=W.device)
    Wc = W.contiguous()
    if ev_begin is None and ev_end is None:
        st = lib().mpq_pack(ctypes.byref(L), Wc.data_ptr(), _np_ptr(bits), _np_ptr(rp), _np_ptr(cp),
                            ctypes.byref(P.c), ws.data_ptr(), ws.numel(), _stream(stream))
    else:
        st = lib().mpq_pack_timed(ctypes.byref(L), Wc.data_ptr(), _np_ptr(bits), _np_ptr(rp),
                                  _np_ptr(cp), ctypes.byref(P.c), ws.data_ptr(), ws.numel(),
                                  _stream(stream), _event(ev_begin), _event(ev_end))
    _raise(st, "mpq_pack")
    if check:
        _raise(lib().mpq_check(ws.data_ptr(), _stream(stream)), "mpq_pack (device)")
    return P


def linear_workspace_size(layer: PackedLayer, M: int) -> int:
    return lib().mpq_linear_workspace_size(ctypes.byref(layer.c), M)


Y_F32, Y_BF16 = 0, 1   # mpq_ydtype
LAYER_16BIT = 1        # mpq_layer.flags: the layer has 16-bit blocks


def linear_typed_workspace_size(layer: PackedLayer, M: int, ydtype: int = Y_F32) -> int:
    return lib().mpq_linear_typed_workspace_size(ctypes.byref(layer.c), M, ydtype)


def linear(layer: PackedLayer, x, out=None, ws=None, stream=None, ydtype: int = Y_F32):
    """mpq_linear: y (M x N) = x (bf16, M x K, cuda) * dequant(W)^T; y fp32, or
    bf16 (mpq_linear_typed, MPQ_Y_BF16) with ydtype=Y_BF16."""
    import torch
    M, K = x.shape
    if out is None:
        dt = torch.bfloat16 if ydtype == Y_BF16 else torch.float32
        out = torch.empty((M, layer.N), dtype=dt, device=x.device)
    if ws is None:
        ws = torch.zeros(max(linear_typed_workspace_size(layer, M, ydtype), 256), dtype=torch.uint8,
                         device=x.device)
    if ydtype == Y_F32:
        st = lib().mpq_linear(ctypes.byref(layer.c), x.data_ptr(), M, out.data_ptr(),
                              ws.data_ptr(), ws.numel(), _stream(stream))
    else:
        st = lib().mpq_linear_typed(ctypes.byref(layer.c), x.data_ptr(), M, out.data_ptr(), ydtype,
                                    ws.data_ptr(), ws.numel(), _stream(stream))
    _raise(st, "mpq_linear")
    return out


GROUP_MAX = 8   # MPQ_GROUP_MAX


def _layer_array(layers):
    arr = (Layer * len(layers))()
    for i, P in enumerate(layers):
        arr[i] = P.c
    return arr


def linear_group_workspace_size(layers, M: int) -> int:
    return lib().mpq_linear_group_workspace_size(_layer_array(layers), len(layers), M)


def linear_group(layers, x, outs=None, ws=None, stream=None):
    """mpq_linear_group: y_i (fp32, M x N_i) = x (bf16, M x K, cuda) * dequant(W_i)^T
    for layers that share K; one launch for the group when M == 1 on short-run
    layers.  Returns the list of outputs."""
    import torch
    M, K = x.shape
    if outs is None:
        outs = [torch.empty((M, P.N), dtype=torch.float32, device=x.device) for P in layers]
    arr = _layer_array(layers)
    if ws is None:
        ws = torch.zeros(max(lib().mpq_linear_group_workspace_size(arr, len(layers), M), 256),
                         dtype=torch.uint8, device=x.device)
    ptrs = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    st = lib().mpq_linear_group(arr, len(layers), x.data_ptr(), M, ptrs, ws.data_ptr(), ws.numel(),
                                _stream(stream))
    _raise(st, "mpq_linear_group")
    return outs


def _event(ev):
    """The cudaEvent_t handle of a torch.cuda.Event (or None)."""
    if ev is None:
        return None
    if ev.cuda_event == 0:   # torch creates the CUDA event on first record
        ev.record()
    return ctypes.c_void_p(ev.cuda_event)


def linear_timed(layer: PackedLayer, x, out, ws, ev_begin, ev_end, stream=None):
    """mpq_linear_timed: as linear(), recording torch.cuda.Event objects around
    the main GEMM kernel."""
    M = x.shape[0]
    for ev in (ev_begin, ev_end):
        if ev.cuda_event == 0:   # torch creates the CUDA event on first record
            ev.record()
    st = lib().mpq_linear_timed(ctypes.byref(layer.c), x.data_ptr(), M, out.data_ptr(),
                                ws.data_ptr(), ws.numel(), _stream(stream),
                                ctypes.c_void_p(ev_begin.cuda_event), ctypes.c_void_p(ev_end.cuda_event))
    _raise(st, "mpq_linear_timed")
    return out


def linear_host(layer: PackedLayer, x_host, y_host, ws, stream=None):
    """mpq_linear_host: host (ideally pinned) x -> host y, enqueued on the stream."""
    M = x_host.shape[0]
    st = lib().mpq_linear_host(ctypes.byref(layer.c), x_host.data_ptr(), M, y_host.data_ptr(),
                               ws.data_ptr(), ws.numel(), _stream(stream))
    _raise(st, "mpq_linear_host")
    return y_host


def linear_host_workspace_size(layer: PackedLayer, M: int) -> int:
    return lib().mpq_linear_host_workspace_size(ctypes.byref(layer.c), M)


def allocate_bits(loss, allowed, budget: int, stream=None):
    """mpq_allocate_bits: per-block widths (uint8 tensor) under a total-bits
    budget from a device float32 loss table [n][8] (widths 0..6, 8).  Returns
    (bits, iterations, total_bits)."""
    import torch
    n = loss.shape[0]
    mask = 0
    for b in allowed:
        mask |= 1 << int(b)
    bits = torch.empty(n, dtype=torch.uint8, device=loss.device)
    info = torch.zeros(4, dtype=torch.int32, device=loss.device)
    ws = torch.empty(max(lib().mpq_allocate_bits_workspace_size(n), 256), dtype=torch.uint8,
                     device=loss.device)
    lc = loss.contiguous()
    _raise(lib().mpq_allocate_bits(n, lc.data_ptr(), mask, int(budget), bits.data_ptr(),
                                   info.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           "mpq_allocate_bits")
    inf = info.cpu().numpy().view(np.uint32)
    _raise(int(inf[3]), "mpq_allocate_bits (device)")
    return bits, int(inf[0]), int(inf[1]) | (int(inf[2]) << 32)


def fold_orders(row_perm_a, col_perm_b, n: int) -> np.ndarray:
    """mpq_fold_orders: the column order that lets layer B read layer A's
    output in A's packed row order (A then runs with row_perm NULL)."""
    a = None if row_perm_a is None else np.ascontiguousarray(row_perm_a, dtype=np.int32)
    b = None if col_perm_b is None else np.ascontiguousarray(col_perm_b, dtype=np.int32)
    out = np.zeros(n, np.int32)
    _raise(lib().mpq_fold_orders(n, _np_ptr(a), _np_ptr(b), _np_ptr(out)), "mpq_fold_orders")
    return out


def with_orders(P: PackedLayer, row_perm=None, col_perm=None, keep_rows=True, keep_cols=True):
    """A view of a packed layer for inference with other activation / output
    orders (device int32 tensors or None): the packed buffers are shared."""
    rp = P.row_perm if keep_rows else row_perm
    cp = P.col_perm if keep_cols else col_perm
    c = Layer(P.c.N, P.c.K, P.c.n_units, P.c.flags, P.c.codes, P.c.table, P.c.sched, P.c.scales, P.c.zeros,
              rp.data_ptr() if rp is not None else None, cp.data_ptr() if cp is not None else None)
    return PackedLayer(P.layout, P.codes, P.table, P.sched, P.scales, P.zeros, rp, cp, c)


def check(ws, stream=None):
    """mpq_check: synchronize and raise on a device-side error word."""
    _raise(lib().mpq_check(ws.data_ptr(), _stream(stream)), "device")


def table_numpy(P: PackedLayer) -> np.ndarray:
    return P.table.cpu().numpy().view(np.uint32).reshape(-1, 4)
