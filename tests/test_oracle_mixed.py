"""Pins of the oracle's mixed precision class (E4M3 scores, E2M1 probabilities and values).

The class sits between FP8 and FP4 in the shared ranking ("DraftAttention2: Fast Video
Diffusion with Low-Resolution-Guided Mixed-Precision Attention", Abstract: higher precision
for the more important blocks, lower precision for the rest, 4- and 8-bit computation).
Independent references: hand-computed budget counts, a brute-force sort, torch SDPA on the
dequantised operands, and the FP4 path re-wired with E4M3 scores.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate


def test_budget_counts_with_a_mixed_class():
    # cumulative cuts floor((p N + 50) / 100), worked out by hand
    assert O.budget_counts3(630, 10, 10, 20) == (63, 63, 126)     # cuts 63, 126, 252
    assert O.budget_counts3(64, 15, 10, 25) == (10, 6, 16)        # cuts 10, 16, 32
    assert O.budget_counts3(588, 10, 10, 20) == (59, 59, 117)     # cuts 59, 118, 235
    for N, p8, p4 in ((630, 10, 30), (64, 15, 35), (990, 5, 25)):
        n8, nm, n4 = O.budget_counts3(N, p8, 0, p4)
        assert nm == 0 and (n8, n4) == O.budget_counts(N, p8, p4)


def test_rank_classes_brute_force_with_ties():
    rng = np.random.default_rng(8)
    N = 64
    sc = rng.random((16, N))
    sc[:, 20:30] = sc[:, 20:21]
    n8, nm, n4 = 10, 6, 16
    r = O.rank_classes(sc, n8, nm, n4)
    for row in range(sc.shape[0]):
        order = sorted(range(N), key=lambda j: (-sc[row, j], j))
        assert list(r["list8"][row]) == sorted(order[:n8])
        assert list(r["listm"][row]) == sorted(order[n8:n8 + nm])
        assert list(r["list4"][row]) == sorted(order[n8 + nm:n8 + nm + n4])
        want = np.zeros(N, np.uint8)
        want[order[:n8]] = O.TAG_FP8
        want[order[n8:n8 + nm]] = O.TAG_MIX
        want[order[n8 + nm:n8 + nm + n4]] = O.TAG_FP4
        assert np.array_equal(r["tags"][row], want)
    # without a mixed class it is the two-class ranking
    t2, a8, a4 = O.rank(sc, n8, n4)
    r0 = O.rank_classes(sc, n8, 0, n4)
    assert np.array_equal(t2, r0["tags"]) and np.array_equal(a8, r0["list8"]) and np.array_equal(a4, r0["list4"])


W = scaled(WORKLOADS["tiny"], F=2, H=2)


def _sdpa(q, k, v, scale):
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    return Fnn.scaled_dot_product_attention(q, k, v, scale=scale).numpy()


def test_mixed_blocks_use_e4m3_scores_and_e2m1_values():
    # every block mixed, P unquantised: softmax of the E4M3 scores times the E2M1 values
    w = scaled(W, pct_fp8=0, pct_mix=100, pct_fp4=0)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    assert (g.n8, g.nm, g.n4) == (0, g.N, 0)
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    o = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, quantise_p=False,
                    listm=sel["listm"])
    ref = _sdpa(O.inverse_permute(ops.q[8], g), O.inverse_permute(ops.k[8], g),
                O.inverse_permute(ops.v[4], g), g.sm_scale)
    assert np.abs(O.inverse_permute(o, g) - ref).max() < 1e-12


def test_mixed_phase_is_the_fp4_phase_on_e4m3_scores():
    # with P quantised: the mixed phase must equal the FP4 phase run on operands whose
    # 4-bit Q/K are replaced by the 8-bit ones (scores at 8 bits, P V at 4 bits)
    w = scaled(W, pct_fp8=10, pct_mix=15, pct_fp4=25)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    a = O.attention(ops, prep["valid"], sel["list8"][..., :0], sel["list4"][..., :0], g.sm_scale, True,
                    listm=sel["listm"])
    rewired = O.Operands({8: ops.q[8], 4: ops.q[8]}, {8: ops.k[8], 4: ops.k[8]}, {8: ops.v[8], 4: ops.v[4]})
    b = O.attention(rewired, prep["valid"], sel["list8"][..., :0], sel["listm"], g.sm_scale, True)
    assert np.array_equal(a, b)
    # and the three-class result differs from treating the mixed blocks as FP4 or as FP8
    full = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, True, listm=sel["listm"])
    as4 = O.attention(ops, prep["valid"], sel["list8"], np.concatenate([sel["listm"], sel["list4"]], -1),
                      g.sm_scale, True)
    assert not np.allclose(full, as4)


def test_three_classes_block_order_invariance_without_p_quantisation():
    w = scaled(W, pct_fp8=10, pct_mix=15, pct_fp4=25)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_exact(prep["qp"], prep["kp"], prep["vp"])
    a = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, False, listm=sel["listm"])
    b = O.attention(ops, prep["valid"], sel["list8"][..., ::-1], sel["list4"][..., ::-1], g.sm_scale, False,
                    listm=sel["listm"][..., ::-1])
    assert np.abs(a - b).max() < 1e-12
    # unquantised, the class split does not matter: equals block-masked SDPA of the kept set
    blk, _ = O.token_block_slot(g)
    kept = sel["tags"] > 0
    mask = kept[:, :, blk][:, :, :, blk]
    qf, kf, vf = (x.float().numpy() for x in (q, k, v))
    ref = Fnn.scaled_dot_product_attention(*(torch.from_numpy(x).double() for x in (qf, kf, vf)),
                                           attn_mask=torch.from_numpy(mask), scale=g.sm_scale).numpy()
    assert np.abs(O.inverse_permute(a, g) - ref).max() < 1e-12
