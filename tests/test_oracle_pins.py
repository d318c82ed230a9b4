"""Pins of the oracle's P quantiser, max-pooled draft map and V group scales.

Each pin is chosen so that a plausible mistake fails it:
  * P quantiser (hand-derived golden values in tests/golden/p_quant.json): a wrong P scale
    (e.g. 240 instead of 448), an unrounded or differently sized FP4 group scale, groups of
    the wrong length, ties rounded away from the even code.
  * max-pooled draft map: its half of the score must be the exact block attention mass of
    window-constant max-pooled queries and keys (full-resolution softmax); a window whose
    single spike token carries the attention must be ranked first, which only the
    max-pooled statistics can see ("DraftAttention2: Fast Video Diffusion with Low-
    Resolution-Guided Mixed-Precision Attention", Abstract: average- and max-pooled
    queries and keys give complementary regional statistics).
  * V group scales run along tokens (the P V contraction axis): groups whose 16 tokens
    reach the top E2M1 value reconstruct exactly, which groups along channels would not.
"""
import json
import os

import numpy as np
import torch

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "p_quant.json")


def _golden():
    return json.load(open(GOLDEN))


def test_p_quantiser_fp8_golden():
    cases = _golden()["fp8"]
    y = np.array([c["y"] for c in cases], dtype=np.float64)
    want = np.array([c["expected"] for c in cases], dtype=np.float64)
    p = y / 448.0
    assert np.array_equal(p * 448.0, y)                   # the inputs are exact
    got = O.quant_p(p, 8)
    assert np.array_equal(got, want / 448.0), [(c["y"], g * 448) for c, g in zip(cases, got)]


def test_p_quantiser_fp4_golden():
    for case in _golden()["fp4"]:
        y = np.array(case["y"], dtype=np.float64)[None, :]
        want = np.array(case["expected"], dtype=np.float64)[None, :]
        p = y / 448.0
        assert np.array_equal(p * 448.0, y)
        got = O.quant_p(p, 4)
        assert np.array_equal(got, want / 448.0), (case["name"], (got * 448).tolist())


def test_p_quantiser_rows_are_independent():
    # the golden rows stacked as one batch (each row padded to 32 keys with zeros): the
    # groups never reach across rows
    rows = [c for c in _golden()["fp4"]]
    y = np.zeros((len(rows), 32))
    want = np.zeros((len(rows), 32))
    for r, c in enumerate(rows):
        y[r, :len(c["y"])] = c["y"]
        want[r, :len(c["expected"])] = c["expected"]
    assert np.array_equal(O.quant_p(y / 448.0, 4), want / 448.0)


def _block_mass(g, qtok, ktok):
    """Exact attention mass of every key block, per query block, from the full-resolution
    softmax over the token matrix (torch, fp64). qtok / ktok: [T, d]; rows of one query
    block are identical here, so the first token of each query block stands for it."""
    blk, _ = O.token_block_slot(g)
    S = g.sm_scale * torch.from_numpy(qtok).double() @ torch.from_numpy(ktok).double().T
    P = torch.softmax(S, dim=-1).numpy()                    # [T, T]
    mass = np.zeros((g.T, g.N))
    np.add.at(mass, (slice(None), blk), P)
    first = np.array([np.flatnonzero(blk == n)[0] for n in range(g.N)])
    return mass[first]                                      # [N query blocks, N key blocks]


def test_max_pooled_map_is_the_block_mass_of_max_pooled_tokens():
    # Every window holds one "high" token a_n and otherwise "low" tokens b_n < a_n (per
    # channel), for Q and K alike, so that the max-pooled vector is a_n and the average
    # pooled one lies in between. The score must be one half of the exact block mass of
    # window-constant avg-pooled Q/K plus one half of that of window-constant max-pooled
    # Q/K (each from the full-resolution softmax), edge windows included.
    w = scaled(WORKLOADS["wan720"], B=1, H=1, F=2, d=16, Hf=20, Wf=40)
    g = O.geometry(w)
    rng = np.random.default_rng(11)
    blk, slot = O.token_block_slot(g)
    valid = O.block_valid(g)

    def tokens():
        a = rng.standard_normal((g.N, 16)).astype(np.float32)
        b = (a - rng.uniform(0.5, 2.0, (g.N, 16))).astype(np.float32)
        first = np.array([np.flatnonzero(blk == n)[0] for n in range(g.N)])
        x = b[blk].copy()
        x[first] = a
        return x

    q, k = tokens(), tokens()
    qavg, qmax = O.pool(O.permute(q[None, None], g), valid)
    kavg, kmax = O.pool(O.permute(k[None, None], g), valid)
    score = O.draft_scores(qavg, kavg, qmax, kmax, valid.sum(1), g.sm_scale)[0, 0]
    m_avg = _block_mass(g, qavg[0, 0][blk].astype(np.float64), kavg[0, 0][blk].astype(np.float64))
    m_max = _block_mass(g, qmax[0, 0][blk].astype(np.float64), kmax[0, 0][blk].astype(np.float64))
    assert np.allclose(score, 0.5 * (m_avg + m_max), rtol=1e-9, atol=1e-13)
    # the two halves differ, so dropping or crossing a pair of statistics is visible
    assert np.abs(m_avg - m_max).max() > 0.05


def test_spike_window_ranked_first_by_the_max_pooled_map():
    # One key window holds a single token aligned with every query while its other tokens
    # point away: its average is the lowest of all windows, its channel maxima the
    # highest. The combined score must keep that window at FP8 for every query block;
    # the average-pooled map alone would skip it.
    w = WORKLOADS["tiny"]
    g = O.geometry(w)
    d = w.d
    blk, slot = O.token_block_slot(g)
    rng = np.random.default_rng(5)
    u = np.full(d, 1.0 / np.sqrt(d))
    q = np.broadcast_to(2.0 * u, (g.T, d)).astype(np.float32)
    k = (0.1 * rng.standard_normal((g.T, d))).astype(np.float32)
    j_spike = 37
    toks = np.flatnonzero(blk == j_spike)
    k[toks] = -(20.0 / (len(toks) - 1) + 0.5) * u
    k[toks[5]] = 20.0 * u
    q4, k4 = q[None, None].copy(), k[None, None].copy()
    P = O.prepare(w.__class__(**{**w.as_dict(), "B": 1, "H": 1}), q4, k4, k4)
    sel = O.draft_select(P)
    assert np.all(sel["tags"][0, 0, :, j_spike] == O.TAG_FP8)
    # the average-pooled map alone ranks the spike window last
    avg_only = O.draft_scores(P["qavg"], P["kavg"], P["qavg"], P["kavg"], P["counts"], g.sm_scale)
    assert np.all(np.argmin(avg_only[0, 0], axis=-1) == j_spike)
    tags_avg, _, _ = O.rank(avg_only, g.n8, g.n4)
    assert np.all(tags_avg[0, 0, :, j_spike] == O.TAG_SKIP)


def test_v_group_scales_run_along_tokens():
    # V values y (already divided by the channel scale) on the E2M1 grid, with a +-6 in
    # every 16-token group of every channel: along tokens each group scale is E4M3(6/6) = 1
    # and the 4-bit copy reconstructs V exactly. Along channels most 16-channel groups of
    # a token hold no 6, their scale is not 1 and their values would not survive.
    w = scaled(WORKLOADS["tiny"], B=1, H=1, F=1)              # 16 blocks of 32 tokens, d = 64
    g = O.geometry(w)
    d = w.d
    rng = np.random.default_rng(9)
    grid = np.array([0.5, 1.0, 1.5, 2.0, 3.0, 4.0])
    y = rng.choice(grid, size=(g.N, g.bs, d)) * rng.choice([-1.0, 1.0], size=(g.N, g.bs, d))
    for grp in range(g.bs // 16):
        for c in range(d):
            y[:, 16 * grp + (c // 16), c] = 6.0 * rng.choice([-1.0, 1.0], size=g.N)
    # the last block carries each channel's amax (7) so that the outer scale is 7/448 =
    # 1/64 exactly and v = y / 64 is exact in bf16
    y[-1] = 0.0
    y[-1, 0, :] = 448.0
    vp = (y / 64.0).astype(np.float32)
    v = O.inverse_permute(vp[None, None], g)
    assert np.all(O.v_channel_amax(v) == 7.0)
    vd = O.quantise_v(O.permute(v, g), O.v_channel_amax(v))
    assert np.all(vd["s"] == np.float32(7.0 / 448.0))
    got = O.dequant_v(vd, 4)[0, 0]
    assert np.all(O.e4m3_decode(vd["sf4"][0, 0, :-1]) == 1.0)
    assert np.array_equal(got[:-1], vp[:-1].astype(np.float64))
    # grouping along channels instead would not reconstruct these values
    codes_c, sig_c = O.fp4_groups(y[:-1].astype(np.float32))
    assert not np.array_equal(O.fp4_dequant(codes_c, sig_c), y[:-1])
