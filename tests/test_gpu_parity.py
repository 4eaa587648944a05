"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Bars: packed codes, table, scales and zeros bit-exact; y within
|y - y_ref| <= 1e-3 * sum_k |x_k * w_hat_k| per output and relative Frobenius
error <= 5e-4 (y is fp32).  Inputs are seeded synthetic layers with the
pages' Llama-2/3 shapes (see block_wise_mixed_b200/synth.py).
"""
import numpy as np
import pytest

from block_wise_mixed_b200 import synth

pytestmark = pytest.mark.gpu

PER_OUT = 1e-3
FROB = 5e-4


@pytest.fixture(scope="module")
def mpq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_wise_mixed_b200 import build
    build.build()
    import block_wise_mixed_b200 as m
    return m


def dev(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def pack_gpu(mpq, L):
    return mpq.pack(dev(L.W), L.bits, L.row_perm, L.col_perm)


def assert_pack_equal(P, R):
    import torch
    torch.cuda.synchronize()
    T = R.table.shape[0]
    got_table = P.table.cpu().numpy().view(np.uint32).reshape(-1, 4)[:T]
    assert np.array_equal(got_table, R.table)
    assert np.array_equal(P.codes.cpu().numpy()[:R.codes.size], R.codes)
    assert np.array_equal(P.scales.cpu().numpy().view(np.uint16)[:R.scales.size], R.scales)
    assert np.array_equal(P.zeros.cpu().numpy().view(np.uint16)[:R.zeros.size], R.zeros)


def check_sched(P, bits):
    """The device copy of the decode schedule is the host plan's, word for word."""
    from block_wise_mixed_b200 import _lib
    n = P.layout.sched_words
    got = P.sched.cpu().numpy().view(np.uint32)[:n]
    assert np.array_equal(got, _lib.plan_schedule(P.layout, bits))


def assert_y_close(y, y_ref, bnd):
    err = np.abs(y.astype(np.float64) - y_ref)
    bad = err > PER_OUT * bnd
    assert not bad.any(), "per-output bound violated at %d outputs, worst ratio %g" % (
        bad.sum(), float(np.max(err / np.maximum(bnd, 1e-300))))
    nrm = np.linalg.norm(y_ref)
    if nrm > 0:
        assert np.linalg.norm(y - y_ref) / nrm <= FROB
    else:
        assert np.all(y == 0)


def run_linear(mpq, P, x_bits):
    import torch
    y = mpq.linear(P, dev(x_bits))
    torch.cuda.synchronize()
    return y.cpu().numpy()


@pytest.mark.parametrize("cfg", [1, 2])
def test_pack_bit_exact_configs(mpq, oracle, cfg):
    L = synth.config_layer(cfg, 0)
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    check_sched(P, L.bits)


@pytest.mark.parametrize("cfg,M", [(1, 1), (1, 2), (1, 3), (1, 7), (1, 8), (1, 9), (1, 16),
                                   (1, 17), (1, 31), (1, 32), (1, 33), (1, 63), (1, 64),
                                   (1, 65), (2, 1), (2, 4), (2, 8), (2, 16)])
def test_linear_configs(mpq, oracle, cfg, M):
    L = synth.config_layer(cfg, 0)
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    x = synth.make_x(synth.seed_of(cfg, 0), M, L.K)
    y_ref, bnd = oracle.linear(R, x)
    assert_y_close(run_linear(mpq, P, x), y_ref, bnd)


@pytest.mark.parametrize("b", [1, 2, 3, 4, 5, 6, 8, 16])
def test_single_block_each_width(mpq, oracle, b):
    L = synth.make_layer("blk", 64, 128, float(b), 900 + b, "random", allowed=(b,))
    assert np.all(L.bits == b)
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    for M in (1, 5):
        x = synth.make_x(900 + b, M, L.K)
        y_ref, bnd = oracle.linear(R, x)
        assert_y_close(run_linear(mpq, P, x), y_ref, bnd)


@pytest.mark.parametrize("kind", ["all0", "all8", "one_nonzero", "identity", "uniform2"])
def test_edge_layers(mpq, oracle, kind):
    N, K = 384, 1024
    L = synth.make_layer("edge", N, K, 2.5, 777, "random")
    if kind == "all0":
        L.bits[:] = 0
    elif kind == "all8":
        L.bits[:] = 8
    elif kind == "one_nonzero":
        L.bits[:] = 0
        L.bits[len(L.bits) // 3] = 3
    elif kind == "identity":
        L.row_perm = None
        L.col_perm = None
    elif kind == "uniform2":
        L.bits[:] = 2
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    check_sched(P, L.bits)
    for M in (1, 3, 8):
        x = synth.make_x(777, M, K)
        y_ref, bnd = oracle.linear(R, x)
        y = run_linear(mpq, P, x)
        assert_y_close(y, y_ref, bnd)
        if kind == "all0":
            assert np.all(y == 0)


def test_zero_rows_and_zero_x(mpq, oracle):
    """An all-zero activation gives exactly 0; so do rows of W that are zero."""
    L = synth.make_layer("z", 256, 512, 3.0, 31, "random")
    W = L.W.copy()
    W[L.row_perm[:64]] = 0          # one whole block row of W' is zero
    P = mpq.pack(dev(W), L.bits, L.row_perm, L.col_perm)
    R = oracle.pack(W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    x = synth.make_x(31, 2, L.K)
    y = run_linear(mpq, P, x)
    y_ref, bnd = oracle.linear(R, x)
    assert_y_close(y, y_ref, bnd)
    assert np.all(y[:, L.row_perm[:64]] == 0)
    y0 = run_linear(mpq, P, np.zeros_like(x))
    assert np.all(y0 == 0)


def test_extreme_activation_scale(mpq, oracle):
    """Per-token power-of-two scaling keeps huge and tiny bf16 tokens exact in fp16."""
    L = synth.make_layer("s", 128, 256, 4.0, 41, "random")
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    xf = synth.bf16_bits_to_f32(synth.make_x(41, 3, L.K))
    xf = xf * np.array([[3e4], [1e-30], [1e30]], np.float32)
    x = synth.f32_to_bf16_bits(xf)
    y_ref, bnd = oracle.linear(R, x)
    assert_y_close(run_linear(mpq, P, x), y_ref, bnd)


def test_device_errors(mpq):
    import torch
    from block_wise_mixed_b200 import MpqError
    L = synth.make_layer("e", 128, 256, 2.0, 51, "random")
    W = L.W.copy()
    W[L.row_perm[5], L.col_perm[7]] = 0x7FC0         # NaN in block (0, 0)
    bits = np.full_like(L.bits, 2)
    with pytest.raises(MpqError) as ei:
        mpq.pack(dev(W), bits, L.row_perm, L.col_perm)
    assert ei.value.name == "MPQ_ERR_NONFINITE"
    W = L.W.copy()
    W[0, 0] = synth.f32_to_bf16_bits(np.array([1e30], np.float32))[0]
    with pytest.raises(MpqError) as ei:
        mpq.pack(dev(W), bits)
    assert ei.value.name == "MPQ_ERR_RANGE"
    # the context is still usable afterwards
    P = mpq.pack(dev(L.W), bits)
    torch.cuda.synchronize()


def test_deterministic(mpq):
    L = synth.config_layer(2, 0)
    P = pack_gpu(mpq, L)
    x = dev(synth.make_x(synth.seed_of(2, 0), 4, L.K))
    y1 = mpq.linear(P, x).cpu().numpy()
    y2 = mpq.linear(P, x).cpu().numpy()
    assert np.array_equal(y1, y2)


def test_linear_host_entry_point(mpq, oracle):
    import torch
    L = synth.config_layer(1, 0)
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    x = synth.make_x(synth.seed_of(1, 0), 3, L.K)
    xh = torch.from_numpy(x.view(np.int16)).pin_memory()
    yh = torch.empty((3, L.N), dtype=torch.float32).pin_memory()
    ws = torch.zeros(mpq.linear_host_workspace_size(P, 3), dtype=torch.uint8, device="cuda")
    mpq.linear_host(P, xh, yh, ws)
    torch.cuda.synchronize()
    y_ref, bnd = oracle.linear(R, x)
    assert_y_close(yh.numpy(), y_ref, bnd)


# ---------------------------------------------------------------------------
# Full-size layers in the benchmark's launch configuration, checked on
# sampled output rows the oracle computes one by one.
# ---------------------------------------------------------------------------
# Every projection of the three large workloads at every batch size they
# name: the Llama-3-8B MLP (gate, up, down) at M = 1, 8, 16, 32; the
# Llama-3-70B decoder layer (q, k, v, o, gate, up, down) at M = 1, 4, 16; the
# Llama-3-8B layer on the tensor-core path at M = 512 and 2048; plus ragged
# tensor-core batches (k at 700: k split in 4; down at 1100: not split).
FULL_CELLS = ([(3, p, (1, 8, 16, 32)) for p in range(3)] +
              [(4, p, (1, 4, 16)) for p in range(7)] +
              [(5, p, (512, 2048)) for p in range(7)] +
              [(5, 1, (700,)), (5, 6, (1100,))])


def sampled_rows(P, L, seed, n_random=96):
    """Output rows to check: random ones plus every row of the block rows that
    several decode runs share (their sums are finished by the last arriving
    run), mapped through the row order."""
    from block_wise_mixed_b200 import _lib
    lay = P.layout
    sched = _lib.plan_schedule(lay, L.bits)
    desc = sched[:lay.n_units * 32].reshape(-1, 32)
    t0, t1 = desc[:, 0].astype(np.int64), desc[:, 1].astype(np.int64)
    first, last = t0 // lay.KB, (t1 - 1) // lay.KB
    shared = set()
    for nb in np.unique(np.concatenate([first, last])):
        if int(np.sum((first <= nb) & (last >= nb))) > 1:
            shared.add(int(nb))
    shared = sorted(shared)
    rng = np.random.default_rng(seed)
    pick = rng.choice(len(shared), min(len(shared), 6), replace=False) if shared else []
    rows_p = [64 * shared[i] + r for i in pick for r in (0, 1, 31, 62, 63)]
    rows_p = np.array(rows_p, dtype=np.int64)
    rows = L.row_perm[rows_p] if L.row_perm is not None else rows_p
    rows = np.concatenate([rows, rng.choice(L.N, n_random, replace=False)])
    return np.unique(rows).astype(np.int32)


@pytest.mark.parametrize("cfg,proj,Ms", FULL_CELLS)
def test_full_size_sampled(mpq, oracle, cfg, proj, Ms):
    L = synth.config_layer(cfg, proj)
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    check_sched(P, L.bits)
    rows = sampled_rows(P, L, cfg * 10 + proj)
    for M in Ms:
        x = synth.make_x(synth.seed_of(cfg, proj), M, L.K)
        y = run_linear(mpq, P, x)
        y_ref, bnd = oracle.linear_rows(R, x, rows)
        assert_y_close(y[:, rows], y_ref, bnd)


# ---------------------------------------------------------------------------
# Tensor-core launch shapes (M > 16): split-K with a ragged last split, with
# and without the row reordering, one 128- or 256-token tile, an odd number
# of block rows, and a layer too wide for the reordering kernel's
# shared-memory row (the epilogue then scatters through row_perm itself).
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("N,K,M,perm,sampled", [
    (512, 128 * 11, 40, True, False),      # 2 splits of 6 + 5 k blocks
    (256, 128 * 37, 129, True, False),     # 8 splits of 5 (last 2), 256-token tile, ragged
    (384, 1024, 64, False, False),         # 2 splits, no row order
    (384, 512, 48, False, False),          # no split, no row order: direct stores
    (320, 512, 17, True, False),           # smallest tensor-core batch, odd number of row blocks
    (51264, 256, 20, True, True),          # a row of y beyond shared memory
    (2048, 128 * 24, 300, True, False),    # 256-token tiles, 2 rows of them (ragged), 4 splits
])
def test_tensor_core_shapes(mpq, oracle, N, K, M, perm, sampled):
    L = synth.make_layer("tc", N, K, 3.0, 4000 + N + K + M, "random")
    if not perm:
        L.row_perm = None
        L.col_perm = None
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    x = synth.make_x(4100 + M, M, K)
    y = run_linear(mpq, P, x)
    if sampled:
        rows = np.sort(np.random.default_rng(N).choice(N, 128, replace=False)).astype(np.int32)
        y_ref, bnd = oracle.linear_rows(R, x, rows)
        assert_y_close(y[:, rows], y_ref, bnd)
    else:
        y_ref, bnd = oracle.linear(R, x)
        assert_y_close(y, y_ref, bnd)


# ---------------------------------------------------------------------------
# bf16 output (mpq_linear_typed, MPQ_Y_BF16): exactly the round-to-nearest-
# even of the fp32 product, on the decode and the tensor-core paths.
# ---------------------------------------------------------------------------
def bf16_rne_bits(y32: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even of fp32 values to bf16 bit patterns (finite input)."""
    u = np.ascontiguousarray(y32, np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


@pytest.mark.parametrize("N,K,M", [(256, 512, 3), (384, 1024, 64), (4096, 4096, 1)])
def test_linear_bf16_output(mpq, oracle, N, K, M):
    import torch
    L = synth.make_layer("y16", N, K, 2.5, 5000 + N + M, "random")
    P = pack_gpu(mpq, L)
    x = synth.make_x(5100 + M, M, K)
    y32 = run_linear(mpq, P, x)
    y16 = mpq.linear(P, dev(x), ydtype=mpq.Y_BF16)
    torch.cuda.synchronize()
    assert y16.dtype == torch.bfloat16 and tuple(y16.shape) == (M, N)
    got = y16.cpu().view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, bf16_rne_bits(y32))
    # against the oracle: its bound plus the bf16 rounding of the value
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    y_ref, bnd = oracle.linear(R, x)
    yb = synth.bf16_bits_to_f32(got).astype(np.float64)
    assert np.all(np.abs(yb - y_ref) <= PER_OUT * bnd + 2.0 ** -8 * np.abs(y_ref) + 1e-30)


def test_workspace_reuse(mpq):
    """One zero-filled workspace serves a mix of calls (one-token layers whose
    decode builds its own activation records, the prologue-kernel path, the
    tensor-core path): each result equals the same call on a fresh workspace,
    so every call leaves the workspace's counters at zero; no device error."""
    import torch
    from block_wise_mixed_b200 import _lib
    small = synth.config_layer(2, 0)                       # one block per run: fused
    big = synth.config_layer(3, 0)                         # ~3 blocks per run: prologue kernel
    Ps, Pb = pack_gpu(mpq, small), pack_gpu(mpq, big)
    calls = [(Ps, 1), (Pb, 1), (Ps, 3), (Ps, 1), (Pb, 40), (Ps, 1), (Pb, 2), (Ps, 1)]
    size = max(mpq.linear_workspace_size(P, M) for P, M in calls)
    ws = torch.zeros(size, dtype=torch.uint8, device="cuda")
    for i, (P, M) in enumerate(calls):
        x = dev(synth.make_x(600 + i, M, P.K))
        got = mpq.linear(P, x, ws=ws)
        want = mpq.linear(P, x)
        torch.cuda.synchronize()
        assert torch.equal(got, want), i
    assert _lib.lib().mpq_check(ws.data_ptr(), None) == 0


@pytest.mark.parametrize("M", [1, 3, 40])
def test_linear_group(mpq, oracle, M):
    """mpq_linear_group equals one mpq_linear per layer bit for bit: one launch
    for short-run layers at M == 1, the layers one after another otherwise;
    and each output meets the oracle's bounds."""
    import torch
    specs = [("q", 1024, 1024, 2.1, "saliency"), ("k", 256, 1024, 2.5, "random"),
             ("v", 512, 1024, 3.0, "random")]
    Ls = [synth.make_layer(n, N, K, b, 7000 + i, perm) for i, (n, N, K, b, perm) in enumerate(specs)]
    Ps = [pack_gpu(mpq, L) for L in Ls]
    x_bits = synth.make_x(7100 + M, M, 1024)
    x = dev(x_bits)
    ys = mpq.linear_group(Ps, x)
    torch.cuda.synchronize()
    for L, P, y in zip(Ls, Ps, ys):
        assert torch.equal(y, mpq.linear(P, x))
        R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
        y_ref, bnd = oracle.linear(R, x_bits)
        assert_y_close(y.cpu().numpy(), y_ref, bnd)


def test_linear_group_mixed_runs(mpq):
    """A group with a long-run layer (its decode needs the prologue kernel)
    runs layer by layer and still equals the single calls."""
    import torch
    big = synth.config_layer(3, 0)                 # 14336 x 4096, ~3 blocks per run
    small = synth.config_layer(2, 0)               # 4096 x 4096, one block per run
    Ps = [pack_gpu(mpq, big), pack_gpu(mpq, small)]
    x = dev(synth.make_x(7200, 1, 4096))
    ys = mpq.linear_group(Ps, x)
    for P, y in zip(Ps, ys):
        assert torch.equal(y, mpq.linear(P, x))


# ---------------------------------------------------------------------------
# Folding one layer's output order into the next layer's input order: layer A
# runs without its row order (y in A's packed row order), layer B reads that
# output through the composed column order (mpq_fold_orders); the result of
# the pair is bit-identical to the unfolded pair, on the decode and the
# tensor-core paths.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("M", [1, 3, 40])
def test_folded_layer_chain(mpq, M):
    import torch
    A = synth.make_layer("a", 512, 1024, 2.5, 8100, "random")
    Bl = synth.make_layer("b", 256, 512, 3.0, 8200, "random")
    PA, PB = pack_gpu(mpq, A), pack_gpu(mpq, Bl)
    x = dev(synth.make_x(8300 + M, M, 1024))
    # unfolded: A scatters y to the original order, B gathers through its order
    ya = mpq.linear(PA, x)
    yb = mpq.linear(PB, ya.to(torch.bfloat16).view(torch.int16))
    # folded
    q = torch.from_numpy(mpq.fold_orders(A.row_perm, Bl.col_perm, 512)).cuda()
    PA_f = mpq.with_orders(PA, row_perm=None, keep_rows=False)
    PB_f = mpq.with_orders(PB, col_perm=q, keep_cols=False)
    ya_f = mpq.linear(PA_f, x)
    yb_f = mpq.linear(PB_f, ya_f.to(torch.bfloat16).view(torch.int16))
    torch.cuda.synchronize()
    rp = torch.from_numpy(A.row_perm.astype(np.int64)).cuda()
    assert torch.equal(ya_f, ya[:, rp])      # A's output in its packed row order
    assert torch.equal(yb_f, yb)



# ---------------------------------------------------------------------------
# TileQuant-style two-level tiles (TileQuant abstract: within each
# projection's retention budget the highest-scoring tiles stay at 16 bits and
# the rest use 8 bits): 16-bit passthrough blocks beside 8-bit ones, and
# beside every quantized width; decode (M <= 16) and tensor-core paths.
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("allowed,avg,perm", [((8, 16), 8.8, "saliency"), ((8, 16), 9.6, "identity"),
                                              ((0, 1, 2, 3, 4, 5, 6, 8, 16), 4.0, "random")])
def test_sixteen_bit_tiles(mpq, oracle, allowed, avg, perm):
    L = synth.make_layer("tq", 1024, 2048, avg, 9100 + int(10 * avg), perm, allowed=allowed)
    if not (L.bits == 16).any():          # a low average draws none: keep every 7th block whole
        L.bits[::7] = 16
    assert (L.bits == 16).any() and (L.bits != 16).any()
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    check_sched(P, L.bits)
    for M in (1, 3, 8, 16, 40, 300):
        x = synth.make_x(9200 + M, M, L.K)
        y_ref, bnd = oracle.linear(R, x)
        assert_y_close(run_linear(mpq, P, x), y_ref, bnd)


def test_sixteen_bit_range_error(mpq):
    from block_wise_mixed_b200 import MpqError
    L = synth.make_layer("r16", 64, 128, 16.0, 9300, "identity", allowed=(16,))
    W = L.W.copy()
    W[1, 2] = synth.f32_to_bf16_bits(np.array([1e5], np.float32))[0]
    with pytest.raises(MpqError) as ei:
        mpq.pack(dev(W), L.bits)
    assert ei.value.name == "MPQ_ERR_RANGE"


@pytest.mark.parametrize("M", [1, 3])     # fused one-token decode; decode after the prologue
def test_sixteen_bit_block_without_flag(mpq, oracle, M):
    """A layer whose 16-bit blocks are not announced in mpq_layer.flags runs
    the decode kernel built without the 16-bit path: the device reports
    MPQ_ERR_BITS (through mpq_check) instead of computing them, and the
    context stays usable (the flagged layer then matches the oracle)."""
    import ctypes
    import torch
    from block_wise_mixed_b200 import MpqError, _lib
    L = synth.make_layer("nf", 256, 1024, 4.0, 9400, "random", allowed=(2, 4, 16))
    L.bits[::5] = 16
    P = pack_gpu(mpq, L)
    assert P.c.flags == _lib.LAYER_16BIT
    c = _lib.Layer.from_buffer_copy(P.c)
    c.flags = 0
    x = dev(synth.make_x(9401 + M, M, L.K))
    y = torch.empty((M, L.N), dtype=torch.float32, device="cuda")
    ws = torch.zeros(mpq.linear_workspace_size(P, M), dtype=torch.uint8, device="cuda")
    st = _lib.lib().mpq_linear(ctypes.byref(c), x.data_ptr(), M, y.data_ptr(), ws.data_ptr(), ws.numel(),
                               _lib._stream(None))
    assert st == 0
    with pytest.raises(MpqError) as ei:
        _lib.check(ws)
    assert ei.value.name == "MPQ_ERR_BITS"
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    y_ref, bnd = oracle.linear(R, synth.make_x(9401 + M, M, L.K))
    assert_y_close(run_linear(mpq, P, synth.make_x(9401 + M, M, L.K)), y_ref, bnd)


@pytest.mark.parametrize("K", [40960, 65536])
def test_pack_long_rows(mpq, oracle, K):
    """Rows too long to stage in shared memory (6 K bytes > 227 KB): the pack
    reads them from global memory; byte-exact against the oracle, and the
    layer matches the oracle on the decode and tensor-core paths."""
    L = synth.make_layer("long", 128, K, 2.5, 9500 + K // 4096, "random")
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    assert_pack_equal(P, R)
    for M in (1, 40):
        x = synth.make_x(9600 + M, M, K)
        y_ref, bnd = oracle.linear(R, x)
        assert_y_close(run_linear(mpq, P, x), y_ref, bnd)


@pytest.mark.parametrize("M", [9, 13, 16])
def test_integer_tensor_core_mid_batch(mpq, oracle, M):
    """9..16 tokens on a layer of >= 100 row tiles: the integer tensor-core
    kernel.  An odd number of block rows (the last tile half empty), every
    width incl. 0-bit blocks, random orders; element by element."""
    L = synth.make_layer("itc", 64 * 201, 1024, 3.0, 9700 + M, "random")
    P = pack_gpu(mpq, L)
    R = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    x = synth.make_x(9800 + M, M, L.K)
    y_ref, bnd = oracle.linear(R, x)
    assert_y_close(run_linear(mpq, P, x), y_ref, bnd)
