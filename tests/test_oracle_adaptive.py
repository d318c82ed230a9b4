"""Pins of the oracle's error-bound-driven FP4 budget (adaptive recovery of skipped blocks).

"DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
Attention", Abstract: the analysis separates the sparsification error from the
attention-weighted quantisation error and establishes when recovering skipped interactions
with low-bit computation tightens the output-error bound. Independent references: the
fixed-budget ranking at either end of the threshold, a brute-force count per row, and the
error decomposition (the bound must tighten).
"""
import numpy as np

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate


def test_threshold_extremes_reduce_to_fixed_budgets():
    rng = np.random.default_rng(3)
    sc = rng.random((12, 64))
    sc /= sc.sum(axis=1, keepdims=True)
    n8, nm, n4, n4max = 10, 0, 12, 22
    hi = O.rank_adaptive(sc, n8, nm, n4, n4max, tau=1e9)          # nothing recovered
    t, l8, l4 = O.rank(sc, n8, n4)
    assert np.array_equal(hi["tags"], t) and np.array_equal(hi["list8"], l8)
    assert np.array_equal(hi["list4"][:, :n4], l4) and (hi["list4"][:, n4:] == -1).all()
    assert (hi["count4"] == n4).all()
    lo = O.rank_adaptive(sc, n8, nm, n4, n4max, tau=1e-12)        # every candidate recovered
    t2, _, l42 = O.rank(sc, n8, n4max)
    assert np.array_equal(lo["tags"], t2) and np.array_equal(lo["list4"], l42)


import pytest


@pytest.mark.parametrize("n8,nm,n4,n4max,tau", [(6, 4, 10, 30, 0.012), (0, 0, 0, 20, 0.02)])
def test_recovered_blocks_brute_force(n8, nm, n4, n4max, tau):
    rng = np.random.default_rng(4)
    N = 64
    sc = rng.random((20, N)) ** 3
    sc /= sc.sum(axis=1, keepdims=True)
    r = O.rank_adaptive(sc, n8, nm, n4, n4max, tau)
    for row in range(sc.shape[0]):
        order = sorted(range(N), key=lambda j: (-sc[row, j], j))
        ck = n8 + nm + n4
        extra = [j for j in order[ck:n8 + nm + n4max] if sc[row, j] >= tau]
        want4 = sorted(order[n8 + nm:ck] + extra)
        assert r["count4"][row] == len(want4)
        assert list(r["list4"][row, :len(want4)]) == want4
        assert (r["list4"][row, len(want4):] == -1).all()
        assert sorted(np.flatnonzero(r["tags"][row] == O.TAG_FP4)) == want4
        assert list(r["listm"][row]) == sorted(order[n8:n8 + nm])


def test_adaptive_recovery_tightens_the_error_bound():
    # on the synthetic tiny layer: with the blocks above the threshold recovered at FP4, the
    # per-row bound E_sp + E_q (and the error itself) is smaller on average than with the
    # fixed budgets, and the padded entries contribute nothing
    w = scaled(WORKLOADS["tiny"], H=1, pct_fp8=10, pct_fp4=15)
    q, k, v = generate(w)
    qf, kf, vf = (x.float().numpy() for x in (q, k, v))
    res = {}
    for name, ww in (("fixed", w), ("adaptive", scaled(w, adapt_tau=0.01, pct_fp4_max=45))):
        prep = O.prepare(ww, q, k, v)
        g = prep["g"]
        sel = O.draft_select(prep)
        ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
        r = O.error_decomposition(qf, kf, vf, prep["valid"], sel["list8"], sel["list4"], ops, g.sm_scale, g)
        assert np.all(r["E_tot"] <= r["E_sp"] + r["E_q"] + 1e-12)
        res[name] = (np.mean(r["E_sp"] + r["E_q"]), np.mean(r["E_tot"]), sel)
    sel = res["adaptive"][2]
    assert (sel["count4"] > O.geometry(w).n4).any()                 # something was recovered
    assert res["adaptive"][0] < res["fixed"][0]
    assert res["adaptive"][1] < res["fixed"][1]
