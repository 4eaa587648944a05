"""mpq_linear_noalloc: the entry point for callers that cannot allocate device
memory (for example an engine plugin whose memory is fixed at initialization)
and therefore cannot pass a workspace.  It uses a static scratch array inside
the library.  Checked through the C ABI against the workspace entry point
mpq_linear and the fp64 oracle, on two calls in a row.  Kept in its own file
so that it is collected after every other test."""
import ctypes

import numpy as np
import pytest

from block_wise_mixed_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def mpq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_wise_mixed_b200 import build
    build.build()
    import block_wise_mixed_b200 as m
    return m


def _noalloc(lib, P, x, y):
    import torch
    return lib.mpq_linear_noalloc(ctypes.byref(P.c), ctypes.c_void_p(x.data_ptr()), x.shape[0],
                                  ctypes.c_void_p(y.data_ptr()),
                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _layer(spec):
    if spec[0] == "cfg":
        return synth.config_layer(spec[1], 0)
    _, N, K = spec      # a tensor-core shape whose k blocks are split across CTAs
    return synth.make_layer("tc", N, K, 3.0, 4000 + N + K, "random")


# Decode kernel (M <= 8), integer tensor-core kernel (9..16, its activation
# records in the static array) and the fp16 tensor-core kernel (M > 16): the
# latter carves its split-K partial sums out of the static array (N=512,
# K=128*11 at M=40 splits the k blocks in two) and reorders rows with a
# second kernel.
@pytest.mark.parametrize("spec,M", [(("cfg", 1), 1), (("cfg", 1), 5), (("cfg", 2), 1),
                                    (("cfg", 2), 8), (("tc", 64 * 201, 1024), 12), (("cfg", 1), 33),
                                    (("tc", 512, 128 * 11), 40)])
def test_noalloc_matches_workspace_entry_point(mpq, oracle, spec, M):
    import torch
    from block_wise_mixed_b200 import _lib
    lib = _lib.lib()
    L = _layer(spec)
    cfg = spec[1] if spec[0] == "cfg" else 0
    P = mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), L.bits, L.row_perm, L.col_perm)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    for call in range(2):
        xb = synth.make_x(synth.seed_of(cfg, 0) + call, M, L.K)
        x = torch.from_numpy(xb.view(np.int16)).cuda()
        y_ref_dev = mpq.linear(P, x)
        y = torch.full((M, L.N), float("nan"), dtype=torch.float32, device="cuda")
        st = _noalloc(lib, P, x, y)
        assert st == 0, _lib.STATUS.get(st, st)
        torch.cuda.synchronize()
        got = y.cpu().numpy().astype(np.float64)
        ref = y_ref_dev.cpu().numpy().astype(np.float64)
        y_or, bnd = oracle.linear(R, xb)
        # the same tolerance as the parity tests, against both references
        assert np.all(np.abs(got - y_or) <= 1e-3 * bnd)
        assert np.linalg.norm(got - y_or) <= 5e-4 * np.linalg.norm(y_or)
        assert np.all(np.abs(got - ref) <= 1e-3 * bnd)
    # no device error was recorded in the static array
    assert lib.mpq_noalloc_check(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0


def test_noalloc_rejects_oversize(mpq):
    import torch
    from block_wise_mixed_b200 import _lib
    lib = _lib.lib()
    L = synth.make_layer("big", 64, 128, 2.0, 5, "identity")
    P = mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), L.bits)
    M = 40000                       # x' alone would need M*K*2 > the static scratch
    x = torch.zeros((1, 1), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, 1), dtype=torch.float32, device="cuda")
    st = lib.mpq_linear_noalloc(ctypes.byref(P.c), ctypes.c_void_p(x.data_ptr()), M,
                                ctypes.c_void_p(y.data_ptr()), None)
    assert _lib.STATUS[st] == "MPQ_ERR_WORKSPACE"
