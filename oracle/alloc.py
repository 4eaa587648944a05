"""Budgeted bit allocation over 64x128 blocks: the CPU oracle.

TEST INFRASTRUCTURE ONLY: imported by ``tests/`` and by ``bench.py``'s CPU
baseline; the CUDA library never imports it and shares no code with it.

Source: "ScaleBITS: Scalable Bitwidth Search for Hardware-Aligned
Mixed-Precision LLMs" -- abstract (global bitwidth allocation as a
constrained optimization under a memory budget, "a scalable approximation to
the greedy algorithm"), summary page section "Approach" ("a batched
approximation to greedy knapsack bit allocation assigns precision per 64x128
block under a global budget"), "Key results" (16-36 search iterations against
about 3e6 for classic greedy) and "Limitations" (per-block surrogates for
raising and lowering precision).

The pages give no formulas.  The reading implemented here (and by the
library's kernel):

* Input: for each block t and each allowed width b, a loss ``loss[t][b]``
  (the sensitivity surrogate: the model-loss increase when block t is held
  at b bits; float32, used as fp64), the set A of allowed widths, and a
  budget B = the sum of the per-block widths (all blocks are the same size,
  so B is the average bits times the block count).
* Classic greedy: every block starts at min(A); each iteration upgrades the
  single block whose next allowed width n saves the most loss per bit,
  gain = (loss[t][w_t] - loss[t][n]) / (n - w_t), among those with gain > 0
  whose increment fits the unspent budget R; ties go to the lower block
  index.  It stops when no upgrade qualifies.  One iteration per upgrade.
* Batched greedy (the scalable approximation): a price lam >= 0 per bit;
  every block independently takes w_t(lam) = argmin_b loss[t][b] + lam * b
  (fp64, the product rounded before the sum; ties to the smaller width).
  The total S(lam) does not grow with lam.  If S(0) <= B the budget does not
  bind (lam = 0).  Otherwise lam is found by bisection between lo = 0
  (S > B) and hi = the largest per-bit saving of any block over min(A)
  (S(hi) = min(A) * T <= B; doubled while rounding leaves S(hi) > B):
  mid = (lo + hi) / 2; S(mid) <= B -> hi = mid,
  else lo = mid; until S(hi) == B, or hi - lo <= hi * 2^-20, or mid equals
  lo or hi, or 64 steps.  Then widths w(hi), and the leftover budget
  R = B - S(hi) is filled in rounds of the classic order: each round takes
  the longest prefix of the qualifying next-width upgrades (gain > 0,
  increment <= R; gain descending, index ascending) whose increments sum to
  at most R.  On losses that are convex in the width this gives the classic
  greedy's widths; each bisection step is one independent pass over the
  blocks.
* Iterations = bisection steps + fill rounds (+ 1 for the pass that finds
  hi).
"""
from __future__ import annotations

import numpy as np

WIDTHS = (0, 1, 2, 3, 4, 5, 6, 8)      # column i of the loss table is width WIDTHS[i]


def _prep(loss, allowed):
    loss = np.asarray(loss, dtype=np.float32).astype(np.float64)
    allowed = sorted(set(int(b) for b in allowed))
    cols = np.array([WIDTHS.index(b) for b in allowed])
    return loss, allowed, cols


def _next_width(allowed):
    nxt = np.full(9, -1, np.int64)
    for i, b in enumerate(allowed[:-1]):
        nxt[b] = allowed[i + 1]
    return nxt


def _fill_round(loss, allowed, w, R):
    """One round of classic-order upgrades that fit R; returns (w, taken bits)."""
    col = np.zeros(9, np.int64)
    for i, b in enumerate(WIDTHS):
        col[b] = i
    nxt = _next_width(allowed)
    idx = np.arange(loss.shape[0])
    n = nxt[w]
    has = n >= 0
    inc = np.where(has, n - w, 0)
    gain = np.where(has, (loss[idx, col[w]] - loss[idx, col[np.where(has, n, w)]]) / np.maximum(inc, 1), 0.0)
    q = has & (gain > 0) & (inc <= R)
    if not q.any():
        return w, 0
    cand = idx[q]
    order = cand[np.lexsort((cand, -gain[cand]))]          # gain descending, index ascending
    k = int(np.searchsorted(np.cumsum(inc[order]), R, side="right"))
    take = order[:k]
    w = w.copy()
    w[take] = n[take]
    return w, int(inc[take].sum())


def widths_at(loss, allowed, lam: float) -> np.ndarray:
    """w_t(lam) = argmin over allowed b of loss[t][b] + lam * b (ties: smaller b)."""
    loss, allowed, cols = _prep(loss, allowed)
    return _widths_at(loss, allowed, cols, lam)


def _widths_at(loss, allowed, cols, lam):
    b = np.array(allowed, np.float64)
    cost = loss[:, cols] + (np.float64(lam) * b)[None, :]   # product rounded, then the sum
    return np.array(allowed, np.int64)[np.argmin(cost, axis=1)]   # first minimum = smaller width


def allocate(loss, allowed, budget: int, batched: bool = True):
    """Returns (widths uint8 [T], iterations, total bits)."""
    loss, allowed, cols = _prep(loss, allowed)
    T = loss.shape[0]
    bmin = allowed[0]
    B = int(budget)
    if B < bmin * T:
        raise ValueError("budget below the smallest allowed width")
    if not batched:
        w = np.full(T, bmin, np.int64)
        R = B - int(w.sum())
        it = 0
        while True:
            col = np.zeros(9, np.int64)
            for i, b in enumerate(WIDTHS):
                col[b] = i
            nxt = _next_width(allowed)
            idx = np.arange(T)
            n = nxt[w]
            has = n >= 0
            inc = np.where(has, n - w, 0)
            gain = np.where(has, (loss[idx, col[w]] - loss[idx, col[np.where(has, n, w)]]) / np.maximum(inc, 1), 0.0)
            q = has & (gain > 0) & (inc <= R)
            if not q.any():
                break
            cand = idx[q]
            t = cand[np.lexsort((cand, -gain[cand]))][0]
            w[t] = n[t]
            R -= int(inc[t])
            it += 1
        return w.astype(np.uint8), it, int(w.sum())

    it = 1                                      # the pass that finds hi and S(0)
    w0 = _widths_at(loss, allowed, cols, 0.0)
    if int(w0.sum()) <= B:
        return w0.astype(np.uint8), it, int(w0.sum())
    base = loss[:, cols[0]][:, None]
    ups = np.array(allowed[1:], np.float64)
    hi = float(np.max((base - loss[:, cols[1:]]) / (ups - bmin)[None, :]))
    lo = 0.0
    S_hi = int(_widths_at(loss, allowed, cols, hi).sum())
    steps = 0
    while S_hi > B and steps < 64:              # rounding at the bracket's edge
        hi *= 2.0
        S_hi = int(_widths_at(loss, allowed, cols, hi).sum())
        steps += 1
    while S_hi != B and steps < 64 and (hi - lo) > hi * 2.0 ** -20:
        mid = (lo + hi) / 2.0
        if mid == lo or mid == hi:
            break
        S = int(_widths_at(loss, allowed, cols, mid).sum())
        steps += 1
        if S <= B:
            hi, S_hi = mid, S
        else:
            lo = mid
    it += steps
    w = _widths_at(loss, allowed, cols, hi)
    R = B - int(w.sum())
    while True:
        w, taken = _fill_round(loss, allowed, w, R)
        if taken == 0:
            break
        R -= taken
        it += 1
    return w.astype(np.uint8), it, int(w.sum())


def total_loss(loss: np.ndarray, widths: np.ndarray) -> float:
    loss = np.asarray(loss, dtype=np.float32).astype(np.float64)
    col = {b: i for i, b in enumerate(WIDTHS)}
    return float(sum(loss[t, col[int(b)]] for t, b in enumerate(widths)))


def synthetic_loss(block_score: np.ndarray) -> np.ndarray:
    """A loss table from per-block sensitivity scores s_t > 0: holding block t
    at b bits costs s_t * 4^-b (the RTN error variance falls by 4 per bit),
    and dropping it (0 bits) costs s_t.  Convex and decreasing in b."""
    s = np.asarray(block_score, np.float64).reshape(-1, 1)
    b = np.array(WIDTHS, np.float64).reshape(1, -1)
    out = s * np.power(4.0, -b)
    out[:, 0] = s[:, 0]
    return out.astype(np.float32)
