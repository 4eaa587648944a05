"""Pins of the fp64 CPU oracle against what the pages and the mathematics fix.

Each check is independent of the oracle's own arithmetic: exact rational
arithmetic (``fractions.Fraction``), brute force over every code, closed forms
worked by hand (``tests/golden/rtn_groups.txt``), numpy's own float16 decoding,
and a bit-by-bit restatement of the packed layout.  A dropped term, a wrong
sign or index, or a transposed operand in the oracle fails at least one.

Method sources: ScaleBITS summary page ("Approach": per-64x128-block bits after
bi-directional reordering; "Key results"/"Limitations": RTN with group 128;
"Surprising findings": 0/1-bit minimum); SFMP abstract (row-column reordering
with activation reordering at inference).
"""
import os
from fractions import Fraction as Fr

import numpy as np
import pytest

from block_wise_mixed_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "rtn_groups.txt")
BITS = (1, 2, 3, 4, 5, 6, 8)


def f16val(bits: int) -> Fr:
    """Exact value of an fp16 bit pattern via numpy (independent decoder)."""
    return Fr(float(np.array([bits], np.uint16).view(np.float16)[0]))


def rne_fr(v: Fr) -> int:
    """Round a rational to the nearest integer, ties to even."""
    f = v.numerator // v.denominator
    r = v - f
    if r > Fr(1, 2) or (r == Fr(1, 2) and f % 2 == 1):
        return f + 1
    return f


def check_group_exact(w, b, s_bits, z_bits, q):
    """Everything the RTN definition fixes, in exact arithmetic."""
    qmax = (1 << b) - 1
    wf = [Fr(float(v)) for v in w]
    lo = min(min(wf), Fr(0))
    hi = max(max(wf), Fr(0))
    d = hi - lo
    s = f16val(s_bits)
    z = f16val(z_bits)
    assert z.denominator == 1 and 0 <= z <= qmax
    if d == 0:
        assert s == 1 and z == 0 and all(int(c) == 0 for c in q)
        return
    # scale: minimal fp16 with s*qmax >= d
    assert s * qmax >= d
    if s_bits > 1:
        assert f16val(s_bits - 1) * qmax < d
    assert s * qmax <= 65504
    # zero point
    assert z == rne_fr(-lo / s)
    for wj, qj in zip(wf, q):
        qj = int(qj)
        assert 0 <= qj <= qmax
        # brute force: the nearest grid point (k - z)*s over all k, ties -> even (k - z)
        best = None
        for k in range(qmax + 1):
            dist = abs(wj - (k - z) * s)
            key = (dist, int(k - z) % 2)
            if best is None or key < best[0]:
                best = (key, k)
        assert qj == best[1], (wj, qj, best)
        # RTN error bound |w - w_hat| <= s/2
        assert abs(wj - (qj - z) * s) <= s / 2


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def test_f16_decoder_matches_numpy(oracle):
    pats = np.arange(65536, dtype=np.uint16)
    ref = pats.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(p)) for p in pats])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got) & (got > 0), np.isinf(ref) & (ref > 0))


# ---------------------------------------------------------------------------
# RTN group quantizer
# ---------------------------------------------------------------------------

def _golden_cases():
    cases = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = [p.strip() for p in line.split("|")]
        b = int(parts[0])
        w = [float(v) for v in parts[1].split()]
        if parts[2] == "RANGE":
            cases.append((b, w, None, None, None))
        else:
            cases.append((b, w, int(parts[2], 16), int(parts[3]),
                          [int(v) for v in parts[4].split()]))
    return cases


@pytest.mark.parametrize("case", _golden_cases())
def test_rtn_hand_derived(oracle, case):
    b, w, s_bits, z, q = case
    if s_bits is None:
        with pytest.raises(oracle.OracleError) as ei:
            oracle.quantize_group(np.array(w), b)
        assert ei.value.status == oracle.ERR_RANGE
        return
    s_got, z_got, q_got = oracle.quantize_group(np.array(w), b)
    assert s_got == s_bits
    assert float(f16val(z_got)) == z
    assert list(q_got) == q


@pytest.mark.parametrize("b", BITS)
def test_rtn_bruteforce_random_groups(oracle, b):
    rng = np.random.default_rng(1234 + b)
    kinds = ["normal", "outlier", "positive", "negative", "tiny", "grid"]
    for trial in range(12):
        kind = kinds[trial % len(kinds)]
        if kind == "normal":
            w = rng.normal(0, 0.02, 128)
        elif kind == "outlier":
            w = rng.normal(0, 0.02, 128)
            w[rng.integers(128)] *= 40
        elif kind == "positive":
            w = np.abs(rng.normal(0, 1, 128)) + 0.5
        elif kind == "negative":
            w = -np.abs(rng.normal(0, 3, 128)) - 1
        elif kind == "tiny":
            w = rng.normal(0, 1e-6, 128)
        else:
            # values on a coarse grid: many exact ties at half steps
            w = rng.integers(-8, 9, 128) * 0.25
        w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w.astype(np.float32))).astype(np.float64)
        s_bits, z_bits, q = oracle.quantize_group(w, b)
        check_group_exact(w, b, s_bits, z_bits, q)


def test_rtn_lo_maps_to_zero_code(oracle):
    # lo = min(w) < 0 maps to code 0 exactly: rne(lo/s) = -rne(-lo/s) = -z
    rng = np.random.default_rng(7)
    for b in BITS:
        w = rng.normal(0, 1, 128)
        w = synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(w.astype(np.float32))).astype(np.float64)
        _, _, q = oracle.quantize_group(w, b)
        assert q[np.argmin(w)] == 0


def test_rtn_nonfinite(oracle):
    for bad in (np.nan, np.inf, -np.inf):
        w = np.zeros(128)
        w[5] = bad
        with pytest.raises(oracle.OracleError) as ei:
            oracle.quantize_group(w, 4)
        assert ei.value.status == oracle.ERR_NONFINITE


# ---------------------------------------------------------------------------
# plan / format
# ---------------------------------------------------------------------------

def test_plan_closed_forms(oracle):
    rng = np.random.default_rng(3)
    N, K = 640, 1280
    T = (N // 64) * (K // 128)
    bits = rng.choice(np.array([0, 1, 2, 3, 4, 5, 6, 8, 16], np.uint8), T)
    lay, table = oracle.plan(N, K, bits)
    assert lay.codes_bytes == 1024 * int(bits.astype(np.int64).sum())
    assert lay.n_sz == 64 * int((bits > 0).sum())
    assert lay.bit_total == int(bits.astype(np.int64).sum())
    order = [1, 2, 3, 4, 5, 6, 8, 16]
    off = 0
    for b in order:
        assert lay.seg_off[b] == off
        assert lay.seg_bytes[b] == 1024 * b * int((bits == b).sum())
        off += lay.seg_bytes[b]
    # table: bits, bit_prefix, and offsets ascending in t within each segment
    assert np.array_equal(table[:, 2], bits)
    assert np.array_equal(table[:, 3], np.concatenate([[0], np.cumsum(bits.astype(np.int64))[:-1]]))
    nz = np.nonzero(bits)[0]
    assert np.array_equal(table[nz, 1], 64 * np.arange(len(nz)))
    assert np.all(table[bits == 0, :3] == 0)
    for b in order:
        ts = np.nonzero(bits == b)[0]
        exp = lay.seg_off[b] + 1024 * b * np.arange(len(ts))
        assert np.array_equal(table[ts, 0], exp)


@pytest.mark.parametrize("N,K,bits,err", [
    (63, 128, None, "SHAPE"), (64, 100, None, "SHAPE"), (0, 128, None, "SHAPE"),
    (64, 128, [7], "BITS"), (64, 128, [9], "BITS"), (64, 128, [15], "BITS"), (64, 128, [32], "BITS")])
def test_plan_errors(oracle, N, K, bits, err):
    T = max(1, (N // 64) * (K // 128))
    b = np.array(bits if bits else [1] * T, np.uint8)
    with pytest.raises(oracle.OracleError) as ei:
        oracle.plan(N, K, b)
    assert oracle.STATUS_NAMES[ei.value.status] == err


def _pieces(b):
    return {1: [1], 2: [2], 3: [2, 1], 4: [4], 5: [4, 1], 6: [4, 2], 8: [8]}[b]


@pytest.mark.parametrize("b", BITS)
def test_payload_layout_bit_by_bit(oracle, b):
    """Restates the v1 byte layout field by field and compares the bytes."""
    rng = np.random.default_rng(50 + b)
    W = synth.f32_to_bf16_bits(rng.normal(0, 0.02, (64, 128)).astype(np.float32))
    P = oracle.pack(W, np.array([b], np.uint8))
    expect = np.zeros(1024 * b, np.uint8)
    for r in range(64):
        w = synth.bf16_bits_to_f32(W[r]).astype(np.float64)
        s_bits, z_bits, q = oracle.quantize_group(w, b)
        assert P.scales[r] == s_bits and P.zeros[r] == z_bits
        base, shift = 0, 0
        for p in _pieces(b):
            row_off = base + r * 16 * p
            for j in range(128):
                v = (int(q[j]) >> shift) & ((1 << p) - 1)
                bitpos = 32 * (j // (32 // p)) + (j % (32 // p)) * p
                for k in range(p):
                    if (v >> k) & 1:
                        pos = bitpos + k
                        expect[row_off + pos // 8] |= 1 << (pos % 8)
            base += 64 * 16 * p
            shift += p
    assert np.array_equal(P.codes, expect)


# ---------------------------------------------------------------------------
# pack / dequant / linear
# ---------------------------------------------------------------------------

def _layer(N=256, K=512, avg=2.5, seed=11, perms="random", allowed=synth.ALL_BITS):
    return synth.make_layer("t", N, K, avg, seed, perms, allowed)


def test_dequant_rows_are_group_rtn(oracle):
    """Every dequantized group equals (q - z)*s of its own RTN, at the right place."""
    L = _layer()
    P = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    What = oracle.dequant(P)
    Wf = synth.bf16_bits_to_f32(L.W).astype(np.float64)
    KB = L.K // 128
    rng = np.random.default_rng(0)
    for _ in range(40):
        i = int(rng.integers(L.N))
        kb = int(rng.integers(KB))
        b = int(L.bits[(i // 64) * KB + kb])
        n = L.row_perm[i]
        cols = L.col_perm[kb * 128:(kb + 1) * 128]
        got = What[n, cols]
        if b == 0:
            assert np.all(got == 0)
            continue
        s_bits, z_bits, q = oracle.quantize_group(Wf[n, cols], b)
        s = float(f16val(s_bits))
        z = float(f16val(z_bits))
        assert np.array_equal(got, (q.astype(np.float64) - z) * s)
        assert np.all(np.abs(Wf[n, cols] - got) <= s / 2)


def test_zero_bit_blocks_contribute_nothing(oracle):
    L = _layer(avg=3.0, seed=12)
    x = synth.make_x(12, 3, L.K)
    P1 = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    W1 = oracle.dequant(P1)
    bits2 = L.bits.copy()
    rng = np.random.default_rng(5)
    kill = rng.choice(len(bits2), len(bits2) // 3, replace=False)
    bits2[kill] = 0
    P2 = oracle.pack(L.W, bits2, L.row_perm, L.col_perm)
    # expected: W1 with the killed blocks (in reordered coordinates) zeroed
    KB = L.K // 128
    W1r = W1[L.row_perm][:, L.col_perm].copy()
    for t in kill:
        nb, kb = divmod(int(t), KB)
        if L.bits[t] != bits2[t]:
            W1r[nb * 64:(nb + 1) * 64, kb * 128:(kb + 1) * 128] = 0
    exp = np.zeros_like(W1)
    exp[np.ix_(L.row_perm, L.col_perm)] = W1r
    # blocks whose bits did not change keep their codes exactly
    assert np.array_equal(oracle.dequant(P2), exp)
    y2, _ = oracle.linear(P2, x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    assert np.allclose(y2, xf @ exp.T, rtol=1e-12, atol=1e-12)
    # all-0-bit layer: y == 0 exactly, nothing stored
    P0 = oracle.pack(L.W, np.zeros_like(L.bits), L.row_perm, L.col_perm)
    assert P0.codes.size == 0 and P0.scales.size == 0
    y0, b0 = oracle.linear(P0, x)
    assert np.all(y0 == 0) and np.all(b0 == 0)


def test_permutation_invariance(oracle):
    L = _layer(seed=13)
    Wp = L.W[L.row_perm][:, L.col_perm]
    P1 = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    P2 = oracle.pack(Wp, L.bits, None, None)
    for a in ("codes", "table", "scales", "zeros"):
        assert np.array_equal(getattr(P1, a), getattr(P2, a)), a
    D1 = oracle.dequant(P1)
    D2 = oracle.dequant(P2)
    assert np.array_equal(D1[L.row_perm][:, L.col_perm], D2)
    x = synth.make_x(13, 2, L.K)
    y1, b1 = oracle.linear(P1, x)
    y2, b2 = oracle.linear(P2, x[:, L.col_perm])
    assert np.allclose(y1[:, L.row_perm], y2, rtol=1e-12, atol=1e-13)
    assert np.allclose(b1[:, L.row_perm], b2, rtol=1e-12, atol=1e-13)


def test_linear_against_numpy_and_loops(oracle):
    L = _layer(N=128, K=256, seed=14)
    P = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    W = oracle.dequant(P)
    x = synth.make_x(14, 3, L.K)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    y, bnd = oracle.linear(P, x)
    assert np.allclose(y, xf @ W.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(bnd, np.abs(xf) @ np.abs(W).T, rtol=1e-12, atol=1e-12)
    # direct triple loop on a few outputs, and a constant activation closed form
    for m, n in [(0, 0), (2, 127), (1, 77)]:
        acc = sum(float(xf[m, k]) * float(W[n, k]) for k in range(L.K))
        assert abs(y[m, n] - acc) <= 1e-12 * max(1.0, bnd[m, n])
    c = synth.f32_to_bf16_bits(np.full((1, L.K), 0.75, np.float32))
    yc, _ = oracle.linear(P, c)
    assert np.allclose(yc[0], 0.75 * W.sum(axis=1), rtol=1e-12, atol=1e-12)


def test_linear_rows_matches_dense(oracle):
    L = _layer(N=256, K=512, seed=15)
    P = oracle.pack(L.W, L.bits, L.row_perm, L.col_perm)
    x = synth.make_x(15, 4, L.K)
    y, b = oracle.linear(P, x)
    rows = np.array([0, 5, 255, 100, 64], np.int32)
    yr, br = oracle.linear_rows(P, x, rows)
    assert np.allclose(yr, y[:, rows], rtol=1e-12, atol=1e-14)
    assert np.allclose(br, b[:, rows], rtol=1e-12, atol=1e-14)


def test_uniform_rtn_g128_special_case(oracle):
    """Every block at one width with identity order is plain uniform RTN-g128
    (the baseline of the ScaleBITS "Key results"), restated here with numpy."""
    rng = np.random.default_rng(16)
    N, K = 128, 384
    W = synth.f32_to_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    Wf = synth.bf16_bits_to_f32(W).astype(np.float64)
    for b in (2, 3, 4):
        P = oracle.pack(W, np.full((N // 64) * (K // 128), b, np.uint8))
        D = oracle.dequant(P)
        qmax = 2 ** b - 1
        g = Wf.reshape(N, K // 128, 128)
        lo = np.minimum(g.min(axis=2), 0)
        hi = np.maximum(g.max(axis=2), 0)
        d = hi - lo
        s = (d / qmax).astype(np.float16).astype(np.float64)
        # move to the smallest fp16 with s*qmax >= d
        s = np.where(s * qmax < d, np.nextafter(s.astype(np.float16), np.float16(np.inf)).astype(np.float64), s)
        prev = np.nextafter(s.astype(np.float16), np.float16(0)).astype(np.float64)
        s = np.where(prev * qmax >= d, prev, s)
        z = np.rint(-lo / s)
        q = np.clip(np.rint(g / s[..., None]) + z[..., None], 0, qmax)
        ref = ((q - z[..., None]) * s[..., None]).reshape(N, K)
        assert np.array_equal(D, ref)


def test_pack_errors(oracle):
    L = _layer(N=128, K=256, seed=17)
    bad = L.row_perm.copy()
    bad[0] = bad[1]
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(L.W, L.bits, bad, L.col_perm)
    assert ei.value.status == oracle.ERR_PERM
    W = L.W.copy()
    W[3, 7] = 0x7FC0  # bf16 NaN
    bits = np.full_like(L.bits, 2)
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(W, bits)
    assert ei.value.status == oracle.ERR_NONFINITE
    W = L.W.copy()
    W[0, 0] = synth.f32_to_bf16_bits(np.array([1e30], np.float32))[0]
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(W, bits)
    assert ei.value.status == oracle.ERR_RANGE
    # a NaN inside a 0-bit block is never read
    W = L.W.copy()
    W[0, 0] = 0x7FC0
    b0 = bits.copy()
    b0[0] = 0
    oracle.pack(W, b0)


# ---------------------------------------------------------------------------
# 16-bit passthrough blocks (TileQuant abstract: the highest-scoring tiles
# stay at 16 bits, the rest are quantized): the payload is the block's bf16
# weights, row-major; scale 1 and zero 0; dequantized exactly.
# ---------------------------------------------------------------------------
def test_sixteen_bit_payload_is_the_weights(oracle):
    L = _layer(N=128, K=256, seed=23)
    bits = np.array([16, 8, 0, 16], np.uint8)           # 2 x 2 blocks
    R = oracle.pack(L.W, bits, L.row_perm, L.col_perm)
    Wp = L.W[L.row_perm][:, L.col_perm]                   # W' as bf16 bits
    lay, table = oracle.plan(128, 256, bits)
    for t in (0, 3):
        nb, kb = divmod(t, 2)
        off = int(table[t, 0])
        block = Wp[64 * nb:64 * nb + 64, 128 * kb:128 * kb + 128]
        got = R.codes[off:off + 16384].view(np.uint16).reshape(64, 128)
        assert np.array_equal(got, block)                 # little-endian bf16, row-major
        sz = int(table[t, 1])
        assert np.all(R.scales[sz:sz + 64] == 0x3C00) and np.all(R.zeros[sz:sz + 64] == 0)
    # segments: the 16-bit payloads come last, in block order
    assert lay.seg_off[16] == lay.seg_bytes[8] and lay.seg_bytes[16] == 2 * 16384
    assert int(table[0, 0]) == lay.seg_off[16] and int(table[3, 0]) == lay.seg_off[16] + 16384
    # dequant: exactly the weights in 16-bit blocks
    What = oracle.dequant(R)
    Wf = synth.bf16_bits_to_f32(L.W).astype(np.float64)
    rows16 = L.row_perm[0:64]
    cols16 = L.col_perm[0:128]
    assert np.array_equal(What[np.ix_(rows16, cols16)], Wf[np.ix_(rows16, cols16)])
    rows16b = L.row_perm[64:128]
    cols16b = L.col_perm[128:256]
    assert np.array_equal(What[np.ix_(rows16b, cols16b)], Wf[np.ix_(rows16b, cols16b)])


def test_all_sixteen_bit_layer_is_the_dense_product(oracle):
    """A layer of 16-bit blocks only computes x W^T on the original weights."""
    L = _layer(N=128, K=256, seed=29)
    bits = np.full(4, 16, np.uint8)
    R = oracle.pack(L.W, bits, L.row_perm, L.col_perm)
    x = synth.make_x(29, 3, 256)
    y, bnd = oracle.linear(R, x)
    xf = synth.bf16_bits_to_f32(x).astype(np.float64)
    Wf = synth.bf16_bits_to_f32(L.W).astype(np.float64)
    ref = xf @ Wf.T
    mag = np.abs(xf) @ np.abs(Wf).T
    assert np.all(np.abs(y - ref) <= 1e-12 * mag)
    assert np.allclose(bnd, np.abs(xf) @ np.abs(Wf).T, rtol=1e-12)


def test_sixteen_bit_errors(oracle):
    L = _layer(N=64, K=128, seed=31)
    bits = np.array([16], np.uint8)
    W = L.W.copy()
    W[2, 3] = 0x7F80                                      # bf16 +inf
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(W, bits)
    assert ei.value.status == oracle.ERR_NONFINITE
    W = L.W.copy()
    W[2, 3] = synth.f32_to_bf16_bits(np.array([70000.0], np.float32))[0]   # beyond fp16
    with pytest.raises(oracle.OracleError) as ei:
        oracle.pack(W, bits)
    assert ei.value.status == oracle.ERR_RANGE
