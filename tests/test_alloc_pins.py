"""Pins of the bit-allocation oracle (oracle/alloc.py), independent of its
own arithmetic: a hand-worked golden case, exhaustive search on tiny layers
(the classic greedy reaches the optimum when every block's loss is convex in
its width and widths go up one bit at a time), and the invariants the
batched search must keep (budget, maximality, iteration count)."""
import itertools
import os

import numpy as np
import pytest

from oracle import alloc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "alloc_small.txt")


def read_golden():
    rows, allowed, budget, want = [], None, None, {}
    for line in open(GOLDEN):
        f = line.split()
        if not f or f[0].startswith("#"):
            continue
        if f[0] == "loss":
            rows.append([float(v) for v in f[1:]])
        elif f[0] == "allowed":
            allowed = [int(v) for v in f[1:]]
        elif f[0] == "budget":
            budget = int(f[1])
        elif f[0] in ("classic", "batched"):
            v = [int(x) for x in f[1:]]
            want[f[0]] = (v[:-2], v[-2], v[-1])
    # spread the per-width losses into the 8 columns of the table
    loss = np.zeros((len(rows), 8), np.float32)
    for t, r in enumerate(rows):
        for b, val in zip(allowed, r):
            loss[t, alloc.WIDTHS.index(b)] = val
    return loss, allowed, budget, want


def test_golden_hand_worked():
    loss, allowed, budget, want = read_golden()
    for mode in ("classic", "batched"):
        w, it, tot = alloc.allocate(loss, allowed, budget, batched=(mode == "batched"))
        assert list(w) == want[mode][0] and tot == want[mode][2], mode
        assert it == want[mode][1] if want[mode][1] >= 0 else it <= 40, mode


def convex_instance(rng, T, allowed):
    """Strictly decreasing, strictly convex losses over the allowed widths."""
    loss = np.zeros((T, 8), np.float32)
    for t in range(T):
        steps = np.sort(rng.uniform(0.1, 10.0, len(allowed) - 1))[::-1]   # decreasing savings
        vals = np.concatenate([[steps.sum() + rng.uniform(0, 1)], np.zeros(len(allowed) - 1)])
        for i, s in enumerate(steps):
            vals[i + 1] = vals[i] - s
        for b, v in zip(allowed, vals):
            loss[t, alloc.WIDTHS.index(b)] = v
    return loss


def brute_force(loss, allowed, budget):
    best = None
    T = loss.shape[0]
    for ws in itertools.product(allowed, repeat=T):
        if sum(ws) > budget:
            continue
        v = alloc.total_loss(loss.astype(np.float64), np.array(ws))
        if best is None or v < best:
            best = v
    return best


@pytest.mark.parametrize("seed", range(6))
def test_classic_greedy_is_optimal_on_convex_unit_steps(seed):
    rng = np.random.default_rng(seed)
    allowed = [0, 1, 2, 3] if seed % 2 else [0, 1, 2, 3, 4, 5, 6]
    T = 4 if len(allowed) == 4 else 3
    loss = convex_instance(rng, T, allowed)
    for budget in range(0, T * max(allowed) + 1, 2):
        w, it, tot = alloc.allocate(loss, allowed, budget, batched=False)
        assert tot <= budget
        opt = brute_force(loss, allowed, budget)
        assert alloc.total_loss(loss.astype(np.float64), w) == pytest.approx(opt, rel=1e-12, abs=1e-9)


@pytest.mark.parametrize("allowed", [(0, 1, 2, 3, 4, 5, 6, 8), (1, 2, 3, 4, 8), (0, 1, 2, 3, 4, 8)])
def test_batched_invariants(allowed):
    rng = np.random.default_rng(len(allowed))
    T = 3000
    loss = alloc.synthetic_loss(rng.lognormal(0.0, 2.0, T))
    budget = int(2.1 * T) if min(allowed) == 0 else int(2.6 * T)
    w, it, tot = alloc.allocate(loss, allowed, budget)
    assert set(np.unique(w)) <= set(allowed)
    assert tot == int(w.sum()) <= budget
    # maximal: no block can take its next width within the leftover budget
    nxt = {a: b for a, b in zip(sorted(allowed), sorted(allowed)[1:])}
    left = budget - tot
    assert all((int(b) not in nxt) or nxt[int(b)] - int(b) > left for b in w)
    # batched search: a few dozen iterations, not one per upgrade
    assert it <= 40
    w1, it1, tot1 = alloc.allocate(loss, allowed, budget, batched=False)
    # classic: one upgrade (one step up the allowed widths) per iteration
    rank = {b: i for i, b in enumerate(sorted(allowed))}
    assert it1 == sum(rank[int(b)] for b in w1)
    # the losses are convex in the width: the threshold search lands on the
    # classic greedy's widths
    assert np.array_equal(w, w1) and tot == tot1


@pytest.mark.parametrize("seed", range(6))
def test_batched_matches_brute_force_on_convex_unit_steps(seed):
    """The threshold search reaches the exhaustive optimum where the classic
    greedy does (convex losses, unit steps)."""
    rng = np.random.default_rng(100 + seed)
    allowed = [0, 1, 2, 3]
    loss = convex_instance(rng, 4, allowed)
    for budget in range(0, 13):
        w, it, tot = alloc.allocate(loss, allowed, budget)
        assert tot <= budget
        opt = brute_force(loss, allowed, budget)
        assert alloc.total_loss(loss, w) == pytest.approx(opt, rel=1e-12, abs=1e-9)


def test_price_monotone():
    """The widths at a higher price per bit never use more bits."""
    rng = np.random.default_rng(9)
    loss = alloc.synthetic_loss(rng.lognormal(0.0, 1.5, 500))
    prev = None
    for lam in np.geomspace(1e-6, 1e3, 40):
        s = int(alloc.widths_at(loss, (0, 1, 2, 3, 4, 5, 6, 8), lam).sum())
        assert prev is None or s <= prev
        prev = s
