"""Host-side decode schedule (mpq_plan_schedule), no GPU: the library's plan
is compared word for word with an independent restatement of its rules, and
checked for the properties the decode kernel relies on (runs tile the block
range, every shared block row owns a contiguous, disjoint range of partial
slots, run costs are balanced)."""
import numpy as np
import pytest

from block_wise_mixed_b200 import _lib as B
from block_wise_mixed_b200 import build, synth

MAX_UNITS = 148 * 16
MIN_UNIT_COST = 4096
WORK = {0: 0, 1: 2048, 2: 2048, 3: 4096, 4: 2304, 5: 4352, 6: 4352, 8: 2560}
ORDER = [1, 2, 3, 4, 5, 6, 8, 16]
DESC = 32


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()
    B.lib()


def block_cost(b):
    if b == 16:
        return 16384 + 256 + 272 + 2048
    return 32 if b == 0 else 1024 * b + 256 + 272 + WORK[b]


def restated_schedule(N, K, bits):
    """The schedule rules, restated: cost-prefix cuts (or, when there are no
    more non-zero blocks than runs, one non-zero block per run), empty runs
    dropped, 32-word run descriptors, then a 4-word stage descriptor per
    non-zero block in block order."""
    NB, KB = N // 64, K // 128
    T = NB * KB
    bits = np.asarray(bits, np.int64)
    cost = np.array([block_cost(b) if (b in WORK or b == 16) else 0 for b in range(17)], np.int64)[bits]
    pre = np.concatenate([[0], np.cumsum(cost)])
    total = int(pre[-1])
    want = max(1, min(-(-total // MIN_UNIT_COST), MAX_UNITS, T))
    bounds = [0]
    nz = np.flatnonzero(bits)
    if want >= len(nz):            # small layer: one non-zero block per run
        bounds += [int(t) for t in nz[1:]]
    else:
        for u in range(1, want):
            tgt = u * total // want
            tb = int(np.searchsorted(pre[:T], tgt, side="left"))
            if bounds[-1] < tb < T:
                bounds.append(tb)
    bounds.append(T)
    U = len(bounds) - 1
    row_first = np.zeros(NB, np.int64)
    row_last = np.zeros(NB, np.int64)
    for u in range(U - 1, -1, -1):
        row_first[bounds[u] // KB:(bounds[u + 1] - 1) // KB + 1] = u
    for u in range(U):
        row_last[bounds[u] // KB:(bounds[u + 1] - 1) // KB + 1] = u
    nc = row_last - row_first + 1
    row_slot = np.concatenate([[0], np.cumsum(np.where(nc > 1, nc, 0))])[:NB]
    seg_off, off = {}, 0
    for b in ORDER:
        seg_off[b] = off
        off += int((bits == b).sum()) * 1024 * b
    nstage = np.where(bits == 16, 2, (bits != 0).astype(np.int64))   # a 16-bit block: two halves
    words = DESC * U + 4 * int(nstage.sum())
    out = np.zeros(words, np.uint32)
    for u in range(U):
        t0, t1 = bounds[u], bounds[u + 1]
        d = out[DESC * u:DESC * (u + 1)]
        d[0], d[1] = t0, t1
        d[2] = int(nstage[:t0].sum())
        d[3] = int(nstage[t0:t1].sum())
        ra, rb = t0 // KB, (t1 - 1) // KB
        d[10], d[11], d[12] = row_slot[ra], nc[ra], u - row_first[ra]
        d[13], d[14], d[15] = row_slot[rb], nc[rb], u - row_first[rb]
    st = out[DESC * U:].reshape(-1, 4)
    si = 0
    for k, t in enumerate(nz):
        b = int(bits[t])
        for half in range(2 if b == 16 else 1):
            st[si, 0] = seg_off[b] + 1024 * b * int((bits[:t] == b).sum()) + 8192 * half
            st[si, 1] = 64 * k
            st[si, 2] = (t % KB) | (b << 16) | (half << 24)
            st[si, 3] = t // KB
            si += 1
    return out, bounds, row_slot, nc


CASES = [
    ("cfg1", synth.config_layer(1, 0)),
    ("cfg2", synth.config_layer(2, 0)),
    ("zero_heavy", synth.make_layer("z", 512, 1024, 0.6, 7, "random")),
    ("one_column", synth.make_layer("c", 1024, 128, 3.0, 8, "identity")),
    ("one_row", synth.make_layer("r", 64, 4096, 2.1, 9, "identity")),
    ("tilequant_8_16", synth.make_layer("t", 512, 2048, 8.8, 10, "saliency", allowed=(8, 16))),
]


@pytest.mark.parametrize("name,L", CASES, ids=[c[0] for c in CASES])
def test_schedule_matches_restatement(name, L):
    lay = B.plan(L.N, L.K, L.bits)
    got = B.plan_schedule(lay, L.bits)
    want, bounds, _, _ = restated_schedule(L.N, L.K, L.bits)
    assert lay.n_units == len(bounds) - 1
    assert lay.sched_words == want.size
    assert np.array_equal(got, want)


def test_schedule_long_runs_and_all_zero():
    # runs of more than 32 non-zero blocks (several chunks of stage descriptors)
    rng = np.random.default_rng(3)
    N, K = 64 * 256, 128 * 1024          # 262144 blocks > 64 * MAX_UNITS
    bits = rng.choice(np.array([0, 1, 2, 3, 4], np.uint8), size=(N // 64) * (K // 128))
    lay = B.plan(N, K, bits)
    got = B.plan_schedule(lay, bits)
    want, bounds, _, _ = restated_schedule(N, K, bits)
    assert np.array_equal(got, want)
    assert max(np.diff(bounds)) > 64
    d = got[:lay.n_units * DESC].reshape(-1, DESC)
    assert d[:, 3].max() > 32
    # an all-zero layer still has runs (they write zeros)
    z = np.zeros(4 * 8, np.uint8)
    lz = B.plan(4 * 64, 8 * 128, z)
    assert np.array_equal(B.plan_schedule(lz, z), restated_schedule(4 * 64, 8 * 128, z)[0])


@pytest.mark.parametrize("name,L", CASES, ids=[c[0] for c in CASES])
def test_schedule_properties(name, L):
    lay = B.plan(L.N, L.K, L.bits)
    s = B.plan_schedule(lay, L.bits)
    U, KB, NB = lay.n_units, lay.KB, lay.NB
    d = s[:DESC * U].reshape(U, DESC).astype(np.int64)
    # runs tile [0, T) in order, none empty
    assert d[0, 0] == 0 and d[-1, 1] == NB * KB
    assert np.all(d[:, 1] > d[:, 0]) and np.all(d[1:, 0] == d[:-1, 1])
    assert U <= MAX_UNITS
    # a run's cost exceeds the even share by less than one block
    cost = np.array([block_cost(int(b)) for b in L.bits])
    pre = np.concatenate([[0], np.cumsum(cost)])
    run = pre[d[:, 1]] - pre[d[:, 0]]
    assert run.max() <= -(-pre[-1] // U) + cost.max() + max(MIN_UNIT_COST, cost.max())
    # shared rows: contiguous, disjoint slot ranges; run index within range
    slots = {}
    for u in range(U):
        for (row, base, nc, idx) in ((d[u, 0] // KB, d[u, 10], d[u, 11], d[u, 12]),
                                     ((d[u, 1] - 1) // KB, d[u, 13], d[u, 14], d[u, 15])):
            assert 0 <= idx < nc
            if nc > 1:
                slots.setdefault(row, set()).add((base, nc, idx))
    used = []
    for row, entries in slots.items():
        bases = {(b, n) for b, n, _ in entries}
        assert len(bases) == 1
        base, nc = bases.pop()
        assert {i for _, _, i in entries} == set(range(nc))
        used.append((base, base + nc))
    used.sort()
    for (a0, a1), (b0, b1) in zip(used, used[1:]):
        assert a1 <= b0
    if used:
        assert used[-1][1] <= U + NB        # the workspace holds n_units + NB slots
