"""The bounded device waits and their error report (MPQ_ERR_TIMEOUT), made to
run out without faulting anything: the wait-test build of the library
(build.build_wait_test: -DMPQ_WAIT_TEST, never the default build) gives every
wait a 2 ms limit and has the producers arm their barriers without issuing a
single copy, so the first wait of every consumer runs out while nothing is
in flight.  Each kernel must return, report MPQ_ERR_TIMEOUT through
mpq_check (or mpq_noalloc_check for the static scratch), and leave the
context usable: the default library then computes the same layer within the
parity bounds."""
import ctypes
import time

import numpy as np
import pytest

from block_wise_mixed_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def libs():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_wise_mixed_b200 import _lib, build
    build.build()
    wt = _lib.load(build.build_wait_test())
    import block_wise_mixed_b200 as m
    return m, _lib, wt


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


# fused one-token decode, decode + prologue, fp16 tensor core, and the
# integer tensor-core kernel (9..16 tokens on a layer of >= 100 row tiles)
@pytest.mark.parametrize("M,shape", [(1, None), (3, None), (40, None), (12, (64 * 201, 1024))])
def test_linear_wait_runs_out(libs, oracle, M, shape):
    import torch
    mpq, _lib, wt = libs
    L = synth.config_layer(1, 0) if shape is None else synth.make_layer("wt", shape[0], shape[1], 3.0, 77, "random")
    P = mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), L.bits, L.row_perm, L.col_perm)
    x = torch.from_numpy(synth.make_x(11, M, L.K).view(np.int16)).cuda()
    y = torch.empty((M, L.N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(mpq.linear_workspace_size(P, M), dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    st = wt.mpq_linear(ctypes.byref(P.c), ctypes.c_void_p(x.data_ptr()), M, ctypes.c_void_p(y.data_ptr()),
                       ctypes.c_void_p(ws.data_ptr()), ws.numel(), _stream())
    assert st == 0
    assert _lib.STATUS[wt.mpq_check(ctypes.c_void_p(ws.data_ptr()), _stream())] == "MPQ_ERR_TIMEOUT"
    assert time.perf_counter() - t0 < 30.0
    # reported once, then cleared
    assert wt.mpq_check(ctypes.c_void_p(ws.data_ptr()), _stream()) == 0
    # the context still works: the default library on the same layer
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    y2 = mpq.linear(P, x).cpu().numpy().astype(np.float64)
    y_ref, bnd = oracle.linear(R, synth.make_x(11, M, L.K))
    assert np.all(np.abs(y2 - y_ref) <= 1e-3 * bnd)


def test_group_wait_runs_out(libs):
    import torch
    mpq, _lib, wt = libs
    Ls = [synth.make_layer("g%d" % i, 256, 512, 2.5, 60 + i, "random") for i in range(3)]
    Ps = [mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), L.bits, L.row_perm, L.col_perm) for L in Ls]
    x = torch.from_numpy(synth.make_x(12, 1, 512).view(np.int16)).cuda()
    ys = [torch.empty((1, 256), dtype=torch.float32, device="cuda") for _ in Ps]
    arr = _lib._layer_array(Ps)
    size = wt.mpq_linear_group_workspace_size(arr, 3, 1)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    ptrs = (ctypes.c_void_p * 3)(*[y.data_ptr() for y in ys])
    st = wt.mpq_linear_group(arr, 3, ctypes.c_void_p(x.data_ptr()), 1, ptrs, ctypes.c_void_p(ws.data_ptr()),
                             size, _stream())
    assert st == 0
    assert _lib.STATUS[wt.mpq_check(ctypes.c_void_p(ws.data_ptr()), _stream())] == "MPQ_ERR_TIMEOUT"


def test_noalloc_wait_runs_out(libs):
    """The static scratch's error word: reported by mpq_noalloc_check, which
    then zero-fills the array (the next check reports nothing)."""
    import torch
    mpq, _lib, wt = libs
    L = synth.config_layer(1, 0)
    P = mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), L.bits, L.row_perm, L.col_perm)
    x = torch.from_numpy(synth.make_x(13, 2, L.K).view(np.int16)).cuda()
    y = torch.empty((2, L.N), dtype=torch.float32, device="cuda")
    st = wt.mpq_linear_noalloc(ctypes.byref(P.c), ctypes.c_void_p(x.data_ptr()), 2,
                               ctypes.c_void_p(y.data_ptr()), _stream())
    assert st == 0
    assert _lib.STATUS[wt.mpq_noalloc_check(_stream())] == "MPQ_ERR_TIMEOUT"
    assert wt.mpq_noalloc_check(_stream()) == 0
