"""Pins of the oracle's windowing, permutation, budgets and pooling."""
import numpy as np
import pytest

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled


def test_token_map_brute_force_and_bijection():
    for name in ("tiny", "wan480", "wan720"):
        w = scaled(WORKLOADS[name], F=2)
        g = O.geometry(w)
        blk, slot = O.token_block_slot(g)
        t = 0
        for f in range(g.F):
            for y in range(g.Hf):
                for x in range(g.Wf):
                    by, bx = y // g.ph, x // g.pw
                    assert blk[t] == (f * g.ny + by) * g.nx + bx
                    assert slot[t] == (y - by * g.ph) * g.pw + (x - bx * g.pw)
                    t += 1
        lin = blk * g.bs + slot
        assert len(np.unique(lin)) == g.T and lin.max() < g.Tp


def test_permute_inverse_identity_and_counts():
    w = scaled(WORKLOADS["wan720"], F=2, H=1, d=8)
    g = O.geometry(w)
    x = np.random.default_rng(0).standard_normal((1, 1, g.T, 8)).astype(np.float32)
    xp = O.permute(x, g)
    assert np.array_equal(O.inverse_permute(xp, g), x)
    valid = O.block_valid(g)
    assert np.all(xp[:, :, ~valid] == 0)
    c = O.block_counts(g)
    assert c.sum() == g.T
    # 45 rows in windows of 8: the last window row holds 5 valid token rows (80 of 128)
    assert sorted(set(c.tolist())) == [80, 128]
    assert (c == 80).sum() == g.F * g.nx


def test_budget_counts_table():
    import json, os
    path = os.path.join(os.path.dirname(__file__), "golden", "budget_counts.json")
    table = json.load(open(path))
    for row in table["rows"]:
        w = WORKLOADS[row["workload"]]
        g = O.geometry(w)
        assert g.N == row["N"] and g.bs == row["bs"]
        assert [g.n8, g.n4, g.N - g.n8 - g.n4] == row["fp8_fp4_skip"]


def test_pool_constant_windows():
    w = scaled(WORKLOADS["wan480"], F=2, H=1, d=4)
    g = O.geometry(w)
    valid = O.block_valid(g)
    import torch
    vals = torch.randn((1, 1, g.N, 1, 4), generator=torch.Generator().manual_seed(1))
    # bf16 values (8 significant bits): every partial sum of <= 128 copies is exact in fp32
    vals = vals.to(torch.bfloat16).float().numpy()
    xp = np.where(valid[None, None, :, :, None], np.broadcast_to(vals, (1, 1, g.N, g.bs, 4)), 0)
    avg, mx = O.pool(xp.astype(np.float32), valid)
    assert np.array_equal(avg, vals[:, :, :, 0]) and np.array_equal(mx, vals[:, :, :, 0])


def test_pool_integer_inputs_and_edge_windows():
    w = scaled(WORKLOADS["wan720"], F=1, H=2, d=8)
    g = O.geometry(w)
    x = np.random.default_rng(2).integers(-20, 21, (1, 2, g.T, 8)).astype(np.float32)
    valid = O.block_valid(g)
    avg, mx = O.pool(O.permute(x, g), valid)
    blk, _ = O.token_block_slot(g)
    for n in range(g.N):
        toks = x[:, :, blk == n, :].astype(np.float64)
        cnt = toks.shape[2]
        # small-integer sums are exact in fp32, so avg is the correctly rounded mean
        assert np.array_equal(avg[:, :, n], (toks.sum(2) / cnt).astype(np.float32))
        assert np.array_equal(mx[:, :, n], toks.max(2).astype(np.float32))
    assert np.all(mx >= avg)
