"""C-ABI checks that need no GPU: the library loads, exports every function
that include/mpq.h declares, and its host-side plan and argument validation
agree with the oracle.  No compute call is made here."""
import ctypes

import numpy as np
import pytest

from block_wise_mixed_b200 import _lib as B
from block_wise_mixed_b200 import build, synth


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.lib()


def test_exports_every_declared_symbol(lib):
    names = B.header_functions()
    assert {"mpq_plan", "mpq_pack", "mpq_linear", "mpq_check", "mpq_status_string",
            "mpq_pack_workspace_size", "mpq_linear_workspace_size", "mpq_linear_host",
            "mpq_linear_host_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n


def test_status_strings(lib):
    for code, name in B.STATUS.items():
        assert lib.mpq_status_string(code).decode() == name


def test_struct_sizes():
    assert ctypes.sizeof(B.Block) == 16
    assert ctypes.sizeof(B.Layout) == 4 * 6 + 8 * 3 + 8 * 34     # seg_off, seg_bytes: index = width 0..16
    assert ctypes.sizeof(B.Layer) == 16 + 7 * 8


@pytest.mark.parametrize("cfg", [1, 2])
def test_plan_matches_oracle(lib, oracle, cfg):
    L = synth.config_layer(cfg, 0)
    got = B.plan(L.N, L.K, L.bits)
    ref, _ = oracle.plan(L.N, L.K, L.bits)
    assert (got.N, got.K, got.NB, got.KB) == (ref.N, ref.K, ref.NB, ref.KB)
    assert got.codes_bytes == ref.codes_bytes and got.n_sz == ref.n_sz
    assert got.bit_total == ref.bit_total
    assert list(got.seg_off) == ref.seg_off and list(got.seg_bytes) == ref.seg_bytes
    assert 1 <= got.n_units <= 148 * 16


@pytest.mark.parametrize("N,K,bits,err", [
    (63, 128, [1], "MPQ_ERR_SHAPE"), (64, 100, [1], "MPQ_ERR_SHAPE"),
    (0, 128, [1], "MPQ_ERR_SHAPE"), (64, 128, [7], "MPQ_ERR_BITS"),
    (64, 256, [1, 9], "MPQ_ERR_BITS")])
def test_plan_errors(lib, N, K, bits, err):
    with pytest.raises(B.MpqError) as ei:
        B.plan(N, K, np.array(bits, np.uint8))
    assert ei.value.name == err


def _fake_layer(L, rp=False, cp=False):
    # non-null placeholders: these calls must fail validation before any
    # device access, so the pointers are never dereferenced
    return B.Layer(L.N, L.K, L.n_units, 0, 16, 16, 16, 16, 16, 16 if rp else None,
                   16 if cp else None)


def test_pack_host_validation(lib):
    N, K = 128, 256
    bits = np.array([1, 2, 3, 4], np.uint8)
    L = B.plan(N, K, bits)
    out = _fake_layer(L, rp=True, cp=True)
    rp = np.arange(N, dtype=np.int32)
    cp = np.arange(K, dtype=np.int32)
    bad = rp.copy()
    bad[3] = bad[4]
    P = ctypes.c_void_p

    def call(bits_=bits, rp_=rp, cp_=cp, out_=out, ws=256, L_=L):
        return lib.mpq_pack(ctypes.byref(L_), P(16), bits_.ctypes.data,
                            None if rp_ is None else rp_.ctypes.data,
                            None if cp_ is None else cp_.ctypes.data,
                            ctypes.byref(out_), P(256 if ws else 0), ws, None)
    assert B.STATUS[call(rp_=bad)] == "MPQ_ERR_PERM"
    bad_c = cp.copy()
    bad_c[0] = K
    assert B.STATUS[call(cp_=bad_c)] == "MPQ_ERR_PERM"
    assert B.STATUS[call(bits_=np.array([1, 2, 7, 4], np.uint8))] == "MPQ_ERR_BITS"
    # a permutation given on the host needs a device buffer for its copy
    assert B.STATUS[call(out_=_fake_layer(L))] == "MPQ_ERR_ARG"
    assert B.STATUS[call(ws=0)] == "MPQ_ERR_WORKSPACE"
    assert B.STATUS[call(ws=16)] == "MPQ_ERR_WORKSPACE"
    # layout that does not belong to these bits
    L2 = B.plan(N, K, np.array([2, 2, 3, 4], np.uint8))
    assert B.STATUS[call(L_=L2)] == "MPQ_ERR_ARG"


def test_linear_host_validation(lib):
    L = B.plan(128, 256, np.array([1, 2, 3, 4], np.uint8))
    layer = _fake_layer(L)
    P = ctypes.c_void_p
    need = lib.mpq_linear_workspace_size(ctypes.byref(layer), 4)
    assert need > 0
    # M == 0 is an empty batch: nothing to do
    assert lib.mpq_linear(ctypes.byref(layer), P(16), 0, P(16), P(256), need, None) == 0
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(16), -1, P(16), P(256), need, None)] == "MPQ_ERR_SHAPE"
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(16), 4, P(16), P(256), need - 1, None)] == "MPQ_ERR_WORKSPACE"
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(16), 4, P(16), P(8), need, None)] == "MPQ_ERR_WORKSPACE"
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), None, 4, P(16), P(256), need, None)] == "MPQ_ERR_ARG"
    bad = B.Layer(100, 256, L.n_units, 0, 16, 16, 16, 16, 16, None, None)
    assert B.STATUS[lib.mpq_linear(ctypes.byref(bad), P(16), 4, P(16), P(256), need, None)] == "MPQ_ERR_SHAPE"


def test_linear_typed_host_validation(lib):
    """mpq_linear_typed: the bf16 workspace holds the fp32 product on top of
    mpq_linear's; host-side checks return before any launch."""
    L = B.plan(128, 256, np.array([1, 2, 3, 4], np.uint8))
    layer = _fake_layer(L)
    P = ctypes.c_void_p
    M = 4
    f32 = lib.mpq_linear_typed_workspace_size(ctypes.byref(layer), M, B.Y_F32)
    b16 = lib.mpq_linear_typed_workspace_size(ctypes.byref(layer), M, B.Y_BF16)
    plain = lib.mpq_linear_workspace_size(ctypes.byref(layer), M)
    assert f32 >= plain and f32 % 256 == 0 and f32 - plain < 256
    assert b16 == f32 + M * L.N * 4
    typed = lib.mpq_linear_typed
    assert B.STATUS[typed(ctypes.byref(layer), P(16), M, P(16), 2, P(256), b16, None)] == "MPQ_ERR_ARG"
    assert B.STATUS[typed(ctypes.byref(layer), P(16), M, P(16), B.Y_BF16, P(256), b16 - 1,
                          None)] == "MPQ_ERR_WORKSPACE"
    assert B.STATUS[typed(ctypes.byref(layer), P(16), M, None, B.Y_BF16, P(256), b16,
                          None)] == "MPQ_ERR_ARG"
    assert typed(ctypes.byref(layer), P(16), 0, P(16), B.Y_BF16, P(256), b16, None) == 0


def test_linear_group_host_validation(lib):
    """mpq_linear_group: sizes add up layer by layer; bad groups are refused
    before any launch."""
    La = B.plan(128, 256, np.array([1, 2, 3, 4], np.uint8))
    Lb = B.plan(64, 256, np.array([2, 0], np.uint8))
    Lc = B.plan(64, 512, np.array([2, 0, 1, 1], np.uint8))
    a, b, c = _fake_layer(La), _fake_layer(Lb), _fake_layer(Lc)
    P = ctypes.c_void_p
    M = 1
    arr = (B.Layer * 2)(a, b)
    need = lib.mpq_linear_group_workspace_size(arr, 2, M)
    each = [lib.mpq_linear_workspace_size(ctypes.byref(l), M) for l in (a, b)]
    assert need == sum((e + 255) // 256 * 256 for e in each)
    ys = (ctypes.c_void_p * 2)(16, 16)
    grp = lib.mpq_linear_group
    assert B.STATUS[grp(arr, 0, P(16), M, ys, P(256), need, None)] == "MPQ_ERR_ARG"
    assert B.STATUS[grp(arr, 9, P(16), M, ys, P(256), need, None)] == "MPQ_ERR_ARG"
    assert B.STATUS[grp(arr, 2, P(16), M, ys, P(256), need - 1, None)] == "MPQ_ERR_WORKSPACE"
    assert B.STATUS[grp(arr, 2, None, M, ys, P(256), need, None)] == "MPQ_ERR_ARG"
    assert B.STATUS[grp(arr, 2, P(16), M, (ctypes.c_void_p * 2)(16, None), P(256), need,
                        None)] == "MPQ_ERR_ARG"
    mixed = (B.Layer * 2)(a, c)   # K 256 and 512
    assert B.STATUS[grp(mixed, 2, P(16), M, ys, P(256), 1 << 20, None)] == "MPQ_ERR_SHAPE"
    assert grp(arr, 2, P(16), 0, ys, P(256), need, None) == 0
    assert lib.mpq_linear_group_workspace_size(arr, 9, M) == 0


@pytest.mark.parametrize("field", ["codes", "table", "sched", "scales", "zeros", "row_perm", "col_perm"])
def test_misaligned_layer_pointers_refused(lib, field):
    """Every buffer the kernels read with vector loads or bulk copies must be
    16-byte aligned; a misaligned one is refused before any launch."""
    L = B.plan(128, 256, np.array([1, 2, 3, 4], np.uint8))
    layer = _fake_layer(L, rp=True, cp=True)
    P = ctypes.c_void_p
    need = lib.mpq_linear_workspace_size(ctypes.byref(layer), 4)
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(16), 0, P(16), P(256), need, None)] == "MPQ_OK"
    setattr(layer, field, 24)
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(16), 4, P(16), P(256), need, None)] == "MPQ_ERR_ARG"


def test_misaligned_x_and_w_refused(lib):
    L = B.plan(128, 256, np.array([1, 2, 3, 4], np.uint8))
    layer = _fake_layer(L)
    P = ctypes.c_void_p
    need = lib.mpq_linear_workspace_size(ctypes.byref(layer), 4)
    assert B.STATUS[lib.mpq_linear(ctypes.byref(layer), P(18), 4, P(16), P(256), need, None)] == "MPQ_ERR_ARG"
    bits = np.array([1, 2, 3, 4], np.uint8)
    out = _fake_layer(L)
    ws_need = lib.mpq_pack_workspace_size(ctypes.byref(L))
    st = lib.mpq_pack(ctypes.byref(L), P(8), bits.ctypes.data_as(P), None, None, ctypes.byref(out),
                      P(256), ws_need, None)
    assert B.STATUS[st] == "MPQ_ERR_ARG"


def test_fold_orders_host():
    """mpq_fold_orders composes the inverse of layer A's row order with layer
    B's column order; reading A's packed-order output through it gives B the
    values its own order would gather."""
    from block_wise_mixed_b200 import _lib
    rng = np.random.default_rng(11)
    n = 384
    a = rng.permutation(n).astype(np.int32)
    b = rng.permutation(n).astype(np.int32)
    q = _lib.fold_orders(a, b, n)
    y = rng.standard_normal((2, n))
    assert np.array_equal(y[:, a][:, q], y[:, b])
    # identities: NULL for either order
    assert np.array_equal(_lib.fold_orders(None, b, n), b)
    assert np.array_equal(_lib.fold_orders(a, None, n)[a], np.arange(n))
    assert np.array_equal(_lib.fold_orders(None, None, n), np.arange(n))
    # errors
    bad = a.copy()
    bad[0] = bad[1]
    with pytest.raises(_lib.MpqError) as ei:
        _lib.fold_orders(bad, b, n)
    assert ei.value.name == "MPQ_ERR_PERM"
    lib = _lib.lib()
    assert _lib.STATUS[lib.mpq_fold_orders(0, None, None, None)] == "MPQ_ERR_ARG"
