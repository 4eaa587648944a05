"""Budgeted bit allocation on the GPU (mpq_allocate_bits) against the CPU
oracle (oracle/alloc.py): widths bit for bit, the same iteration count and
total bits, on synthetic sensitivity surrogates shaped like the pages'
workloads (the block count of the Llama-3-70B decoder layer), on losses that
are not convex, at budgets that do and do not bind; then a layer packed with
the allocated bit map and multiplied within the parity bounds."""
import os

import numpy as np
import pytest

from block_wise_mixed_b200 import synth
from oracle import alloc

pytestmark = pytest.mark.gpu

ALL = (0, 1, 2, 3, 4, 5, 6, 8)
T70 = sum((N // 64) * (K // 128) for _, N, K in synth.LLAMA3_70B)   # 104448 blocks


@pytest.fixture(scope="module")
def mpq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from block_wise_mixed_b200 import build
    build.build()
    import block_wise_mixed_b200 as m
    return m


def run_both(mpq, loss, allowed, budget):
    import torch
    bits, it, tot = mpq.allocate_bits(torch.from_numpy(loss).cuda(), allowed, budget)
    w, it_o, tot_o = alloc.allocate(loss, allowed, budget)
    got = bits.cpu().numpy()
    assert np.array_equal(got, w), "widths differ at %d blocks" % int((got != w).sum())
    assert it == it_o and tot == tot_o
    return got, it, tot


@pytest.mark.parametrize("allowed,avg,sigma", [(ALL, 2.1, 2.0), ((0, 1, 2, 3, 4, 8), 2.5, 1.0),
                                               ((1, 2, 3, 4, 8), 3.0, 1.5), ((2, 3, 4), 3.0, 0.5)])
def test_allocation_llama70b_blocks(mpq, allowed, avg, sigma):
    rng = np.random.default_rng(int(avg * 10) + len(allowed))
    loss = alloc.synthetic_loss(rng.lognormal(0.0, sigma, T70))
    budget = int(round(avg * T70))
    w, it, tot = run_both(mpq, loss, allowed, budget)
    assert tot <= budget and it <= 40


def test_allocation_not_convex_and_not_binding(mpq):
    rng = np.random.default_rng(77)
    T = 20000
    loss = (rng.lognormal(0.0, 1.0, (T, 8)) * np.sort(rng.uniform(0.1, 1.0, (T, 8)))[:, ::-1])
    loss = loss.astype(np.float32)
    run_both(mpq, loss, ALL, int(2.1 * T))        # binding, losses not convex in the width
    run_both(mpq, loss, ALL, 8 * T)               # every block at its best width: not binding
    run_both(mpq, loss, (3,), 3 * T)              # one allowed width


def test_allocation_golden(mpq):
    from test_alloc_pins import read_golden
    loss, allowed, budget, want = read_golden()
    w, it, tot = run_both(mpq, loss, allowed, budget)
    assert list(w) == want["batched"][0] and tot == want["batched"][2]


def test_allocation_errors(mpq):
    import torch
    from block_wise_mixed_b200 import MpqError
    loss = alloc.synthetic_loss(np.ones(64))
    loss[5, 3] = np.nan
    with pytest.raises(MpqError) as ei:
        mpq.allocate_bits(torch.from_numpy(loss).cuda(), ALL, 128)
    assert ei.value.name == "MPQ_ERR_NONFINITE"
    with pytest.raises(MpqError) as ei:
        mpq.allocate_bits(torch.from_numpy(loss).cuda(), (1, 2), 10)    # below 1 bit per block
    assert ei.value.name == "MPQ_ERR_ARG"


def test_allocated_layer_packs_and_multiplies(mpq, oracle):
    """The bit map the search returns drives a full pack + linear."""
    import torch
    L = synth.config_layer(2, 0)                 # 4096 x 4096, saliency orders
    score = synth.block_saliency(L.W, L.act_ch, L.row_perm, L.col_perm).reshape(-1)
    loss = alloc.synthetic_loss(score)
    bits, it, tot = mpq.allocate_bits(torch.from_numpy(loss).cuda(), ALL, int(2.1 * score.size))
    b = bits.cpu().numpy()
    assert np.array_equal(b, alloc.allocate(loss, ALL, int(2.1 * score.size))[0])
    P = mpq.pack(torch.from_numpy(L.W.view(np.int16)).cuda(), b, L.row_perm, L.col_perm)
    R = oracle.pack(L.W, b, L.row_perm, L.col_perm)
    x = synth.make_x(synth.seed_of(2, 0), 2, L.K)
    y = mpq.linear(P, torch.from_numpy(x.view(np.int16)).cuda()).cpu().numpy().astype(np.float64)
    y_ref, bnd = oracle.linear(R, x)
    assert np.all(np.abs(y - y_ref) <= 1e-3 * bnd)
    assert np.linalg.norm(y - y_ref) <= 5e-4 * np.linalg.norm(y_ref)
