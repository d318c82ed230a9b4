"""Pins of the oracle's block-sparse mixed-precision attention and error decomposition.

Independent references: torch's scaled_dot_product_attention in fp64 (dense or with a
boolean block mask), closed-form error bounds of the P quantisers, and the triangle
inequality behind the error decomposition.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate


def _inputs(w):
    q, k, v = generate(w)
    return q, k, v


def _sdpa(q, k, v, scale, mask=None):
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    return Fnn.scaled_dot_product_attention(q, k, v, attn_mask=None if mask is None
                                            else torch.as_tensor(mask), scale=scale).numpy()


W_SMALL = scaled(WORKLOADS["tiny"], F=2, H=2)


def _block_mask(g, tags):
    blk, _ = O.token_block_slot(g)
    return tags[:, :, blk][:, :, :, blk] > 0          # [B,H,Tq,Tk]


def test_unquantised_full_budget_equals_dense_attention():
    w = scaled(W_SMALL, pct_fp8=100, pct_fp4=0)
    q, k, v = _inputs(w)
    r = O.run(w, q, k, v, quantised=False)
    ref = _sdpa(q.float(), k.float(), v.float(), r["prep"]["g"].sm_scale)
    assert np.abs(r["out"] - ref).max() < 1e-12


def test_unquantised_sparse_equals_block_masked_attention():
    w = scaled(W_SMALL, pct_fp8=15, pct_fp4=0)            # earlier DraftAttention: skip only
    q, k, v = _inputs(w)
    r = O.run(w, q, k, v, quantised=False)
    g = r["prep"]["g"]
    mask = _block_mask(g, r["sel"]["tags"])
    ref = _sdpa(q.float(), k.float(), v.float(), g.sm_scale, mask)
    assert np.abs(r["out"] - ref).max() < 1e-12


@pytest.mark.parametrize("prec", [8, 4])
def test_quantised_operands_exact_p_equal_attention_on_dequantised(prec):
    w = scaled(W_SMALL, pct_fp8=100 if prec == 8 else 0, pct_fp4=0 if prec == 8 else 100)
    q, k, v = _inputs(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    o = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale,
                    quantise_p=False)
    deq = [O.inverse_permute(ops.q[prec], g), O.inverse_permute(ops.k[prec], g),
           O.inverse_permute(ops.v[prec], g)]
    ref = _sdpa(*deq, g.sm_scale)
    assert np.abs(O.inverse_permute(o, g) - ref).max() < 1e-12
    # and the dequantised operands are close to the inputs (format error bounds)
    x = [t.float().numpy() for t in (q, k, v)]
    for a, b in zip(deq, x):
        rel = np.abs(a - b).max() / np.abs(b).max()
        assert rel < (1 / 16 if prec == 8 else 0.35)


def test_block_order_invariance_without_p_quantisation():
    # the online recurrence (running max, rescaled sum and accumulator) is exact
    w = scaled(W_SMALL, pct_fp8=10, pct_fp4=30)
    q, k, v = _inputs(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_exact(prep["qp"], prep["kp"], prep["vp"])
    a = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, False)
    b = O.attention(ops, prep["valid"], sel["list8"][..., ::-1], sel["list4"][..., ::-1],
                    g.sm_scale, False)
    assert np.abs(a - b).max() < 1e-12


@pytest.mark.parametrize("prec", [8, 4])
def test_p_quantisation_error_bound(prec):
    w = scaled(W_SMALL, pct_fp8=100 if prec == 8 else 0, pct_fp4=0 if prec == 8 else 100)
    q, k, v = _inputs(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    a = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, True)
    b = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, False)
    vmax = np.abs(ops.v[prec]).max()
    # E4M3: |p~ - p| <= p/16 + 2^-10/448; FP4 groups: <= sigma/448 + amax16/(16*448), and
    # sigma <= amax16/6 (1 + 1/16), amax16 <= 1 -> per element <= 0.25 of the group max;
    # with the sum l >= 1 at the row max, |O~ - O| <= per-element bound * keys * vmax.
    keys = g.N * g.bs
    bound = (vmax / 16 + keys * 2 ** -10 / 448 * vmax) if prec == 8 else 0.25 * vmax * 16
    err = np.abs(a - b).max()
    assert 0 < err < bound


def test_error_decomposition_triangle_bound():
    w = scaled(W_SMALL, H=1, pct_fp8=10, pct_fp4=30)
    q, k, v = _inputs(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    qf, kf, vf = (t.float().numpy() for t in (q, k, v))
    r = O.error_decomposition(qf, kf, vf, prep["valid"], sel["list8"], sel["list4"], ops,
                              g.sm_scale, g)
    assert np.all(r["E_tot"] <= r["E_sp"] + r["E_q"] + 1e-12)
    # O = (1 - m_skip) O_S + m_skip o_skip  =>  |O_S - O| <= m_skip * 2 max|v|
    assert np.all(r["E_sp"] <= r["m_skip"] * 2 * np.sqrt(g.d) * np.abs(vf).max() + 1e-12)
    # the dense reference inside the decomposition is the textbook attention
    ref = _sdpa(qf, kf, vf, g.sm_scale)
    assert np.abs(O.inverse_permute(r["O"], g) - ref).max() < 1e-12


def _decomposition(w):
    q, k, v = _inputs(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    qf, kf, vf = (t.float().numpy() for t in (q, k, v))
    r = O.error_decomposition(qf, kf, vf, prep["valid"], sel["list8"], sel["list4"], ops,
                              g.sm_scale, g)
    return g, sel, (qf, kf, vf), r


def test_error_decomposition_sparsification_term_from_torch():
    # the skipped mass and E_sp from torch alone: softmax of the full score matrix summed
    # over the skipped keys, and the distance between masked and dense SDPA; E_sp also
    # equals m_skip |O_S - o_skip| (O is the kept and skipped outputs mixed by their mass)
    g, sel, (qf, kf, vf), r = _decomposition(scaled(W_SMALL, H=1, pct_fp8=10, pct_fp4=30))
    kept = _block_mask(g, sel["tags"])
    S = g.sm_scale * np.einsum("bhqd,bhkd->bhqk", qf.astype(np.float64), kf.astype(np.float64))
    P = torch.softmax(torch.from_numpy(S), dim=-1).numpy()
    m_skip = np.where(kept, 0.0, P).sum(-1)
    assert np.abs(O.inverse_permute(r["m_skip"][..., None], g)[..., 0] - m_skip).max() < 1e-12
    dense = _sdpa(qf, kf, vf, g.sm_scale)
    sparse = _sdpa(qf, kf, vf, g.sm_scale, kept)
    skip = _sdpa(qf, kf, vf, g.sm_scale, ~kept)
    e_sp = np.linalg.norm(sparse - dense, axis=-1)
    assert np.abs(O.inverse_permute(r["E_sp"][..., None], g)[..., 0] - e_sp).max() < 1e-12
    assert np.abs(e_sp - m_skip * np.linalg.norm(sparse - skip, axis=-1)).max() < 1e-12


def test_error_decomposition_quantisation_term_bounds_the_quantisation_part():
    # O~ - O_S = sum_b w_b (o~_b - o_b) + sum_b (w~_b - w_b) o~_b, so E_q bounds |O~ - O_S|
    g, sel, _, r = _decomposition(scaled(W_SMALL, H=1, pct_fp8=10, pct_fp4=30))
    dq = np.linalg.norm(r["Ot"] - r["OS"], axis=-1)
    assert np.all(dq <= r["E_q"] + 1e-12)
    assert np.any(r["E_q"] > dq * (1 + 1e-6))            # and is not that distance itself


@pytest.mark.parametrize("prec", [8, 4])
def test_error_decomposition_quantisation_term_closed_form(prec):
    # Q = 0: every score is 0, so p = 1 on every valid key and one kept block per row gives
    # o = the mean of the block's values, o~ = the mean of their dequantised copies. FP8 keeps
    # 448 p = 448 exactly (w~ = 1); FP4 groups of p = 1 get sigma = E4M3(448 / 6) = 72 and
    # code E2M1(448 / 72) = 6, so p~ = 432 / 448 on every key and w~ = 27 / 28. Hence
    # E_q = |o~ - o| + |w~ - 1| |o~| on every row of the block.
    w = scaled(W_SMALL, H=1, pct_fp8=2 if prec == 8 else 0, pct_fp4=0 if prec == 8 else 2)
    q, k, v = _inputs(w)
    q = torch.zeros_like(q)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    assert g.n8 + g.n4 == 1
    sel = O.draft_select(prep)
    ops = O.operands_quantised(prep["Q"], prep["K"], prep["V"])
    qf, kf, vf = (t.float().numpy() for t in (q, k, v))
    r = O.error_decomposition(qf, kf, vf, prep["valid"], sel["list8"], sel["list4"], ops,
                              g.sm_scale, g)
    lst = sel["list8"] if prec == 8 else sel["list4"]
    vq = O.dequant_v(prep["V"], prec)
    wt = 1.0 if prec == 8 else 27.0 / 28.0
    for i in range(g.N):
        j = lst[0, 0, i, 0]
        ok = prep["valid"][j]
        o = prep["vp"][0, 0, j][ok].astype(np.float64).mean(0)
        ot = vq[0, 0, j][ok].mean(0)
        want = np.linalg.norm(ot - o) + abs(wt - 1.0) * np.linalg.norm(ot)
        assert np.abs(r["E_q"][0, 0, i] - want).max() < 1e-12
        assert np.abs(r["OS"][0, 0, i] - o).max() < 1e-12
        assert np.abs(r["Ot"][0, 0, i] - wt * ot).max() < 1e-12
