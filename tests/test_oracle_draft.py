"""Pins of the oracle's draft map and ranking."""
import numpy as np
import torch

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate


def test_draft_map_exact_for_window_constant_tokens():
    # Every token of window n carries the same q_n / k_n: the mass-corrected avg-pooled
    # draft map then equals the exact attention mass that the full-resolution softmax puts
    # on each key block (computed here with torch's softmax on the full token matrix).
    w = scaled(WORKLOADS["wan720"], F=2, H=2, d=16, Hf=20, Wf=40)
    g = O.geometry(w)
    rng = np.random.default_rng(3)
    # bf16-valued (8 significant bits) so that the fp32 window sums are exact
    qb = torch.from_numpy(rng.standard_normal((1, 2, g.N, 16))).to(torch.bfloat16).float().numpy()
    kb = torch.from_numpy(rng.standard_normal((1, 2, g.N, 16))).to(torch.bfloat16).float().numpy()
    blk, _ = O.token_block_slot(g)
    q, k = qb[:, :, blk], kb[:, :, blk]
    valid = O.block_valid(g)
    qavg, qmax = O.pool(O.permute(q, g), valid)
    kavg, kmax = O.pool(O.permute(k, g), valid)
    c = valid.sum(1)
    S = g.sm_scale * torch.einsum("bhqd,bhkd->bhqk", torch.from_numpy(q).double(),
                                  torch.from_numpy(k).double())
    P = torch.softmax(S, dim=-1).numpy()                      # [1,2,T,T]
    mass = np.zeros((1, 2, g.T, g.N))
    np.add.at(mass, (slice(None), slice(None), slice(None), blk), P)
    first_tok = np.array([np.flatnonzero(blk == n)[0] for n in range(g.N)])
    exact = mass[:, :, first_tok]                             # one row per query block
    sc = O.draft_scores(qavg, kavg, qmax, kmax, c, g.sm_scale)
    assert np.allclose(sc, exact, atol=1e-12, rtol=1e-9)      # avg == max for constants


def test_draft_map_error_shrinks_with_smoothness():
    # Earlier DraftAttention's analysis (news article, theory paragraph): the draft map's
    # Frobenius-norm error against the full map falls as tokens vary less within a window.
    w = scaled(WORKLOADS["tiny"], H=2)
    g = O.geometry(w)
    blk, _ = O.token_block_slot(g)
    valid = O.block_valid(g)
    errs = []
    for noise in (0.6, 0.3, 0.0):
        e = []
        for seed in range(3):
            gen = torch.Generator().manual_seed(seed)
            base = generate(w, seed=100 + seed)
            q = base[0].float() + noise * torch.randn(base[0].shape, generator=gen)
            k = base[1].float() + noise * torch.randn(base[1].shape, generator=gen)
            q, k = q.numpy(), k.numpy()
            qa, qm = O.pool(O.permute(q, g), valid)
            ka, km = O.pool(O.permute(k, g), valid)
            qa64 = torch.from_numpy(qa).double()
            ka64 = torch.from_numpy(ka).double()
            lg = g.sm_scale * qa64 @ ka64.transpose(-1, -2) + torch.log(
                torch.from_numpy(valid.sum(1)).double())
            draft = torch.softmax(lg, -1).numpy()
            P = torch.softmax(g.sm_scale * torch.from_numpy(q).double()
                              @ torch.from_numpy(k).double().transpose(-1, -2), -1).numpy()
            mass = np.zeros(P.shape[:3] + (g.N,))
            np.add.at(mass, (slice(None), slice(None), slice(None), blk), P)
            full = np.zeros(mass.shape[:2] + (g.N, g.N))
            np.add.at(full, (slice(None), slice(None), blk), mass)
            full /= valid.sum(1)[None, None, :, None]
            e.append(np.linalg.norm(draft - full))
        errs.append(np.mean(e))
    assert errs[0] > errs[1] > errs[2]


def test_rank_brute_force_with_ties():
    rng = np.random.default_rng(4)
    N = 64
    sc = rng.random((20, N))
    sc[:, 10:20] = sc[:, 10:11]            # a run of exact ties
    sc[5] = 0.5                            # an all-tie row
    n8, n4 = 10, 22
    tags, l8, l4 = O.rank(sc, n8, n4)
    for r in range(sc.shape[0]):
        order = sorted(range(N), key=lambda j: (-sc[r, j], j))
        assert sorted(order[:n8]) == list(l8[r])
        assert sorted(order[n8:n8 + n4]) == list(l4[r])
        want = np.zeros(N, np.uint8)
        want[order[:n8]] = 2
        want[order[n8:n8 + n4]] = 1
        assert np.array_equal(tags[r], want)


def test_rank_degenerate_budgets():
    sc = np.random.default_rng(5).random((3, 7))
    tags, l8, l4 = O.rank(sc, 0, 0)
    assert tags.sum() == 0 and l8.shape == (3, 0) and l4.shape == (3, 0)
    tags, l8, l4 = O.rank(sc, 7, 0)
    assert np.all(tags == 2) and np.array_equal(l8, np.tile(np.arange(7), (3, 1)))


def test_draft_selection_tracks_true_block_mass():
    # [DA2] Abstract: the low-resolution draft map estimates block importance. Against the
    # true attention mass of each key block (dense fp64 softmax over the valid tokens,
    # averaged over the query block's rows), the kept set must share far more blocks with
    # the true top set than chance (half of them here: 32 kept of 64) would; a reversed
    # ranking shares about a quarter.
    w = WORKLOADS["tiny"]
    q, k, v = generate(w, device="cpu")
    for h in range(w.H):
        w1 = scaled(w, B=1, H=1)
        qh, kh, vh = (x[:, h:h + 1] for x in (q, k, v))
        P = O.prepare(w1, qh, kh, vh)
        sel = O.draft_select(P)
        g = P["g"]
        qp, kp = (O.permute(x.float().numpy(), g).astype(np.float64) for x in (qh, kh))
        Q, K = qp[0, 0], kp[0, 0].reshape(g.N * g.bs, -1)
        valid = np.asarray(P["valid"]).reshape(-1).astype(bool)
        nk = g.n8 + g.n4
        shared = []
        for i in range(g.N):
            S = g.sm_scale * Q[i] @ K.T
            S[:, ~valid] = -np.inf
            S -= S.max(axis=1, keepdims=True)
            Pm = np.exp(S)
            Pm /= Pm.sum(axis=1, keepdims=True)
            mass = Pm.reshape(g.bs, g.N, g.bs).sum(axis=2).mean(axis=0)
            top = np.argsort(-mass, kind="stable")[:nk]
            kept = np.union1d(sel["list8"][0, 0, i], sel["list4"][0, 0, i])
            shared.append(len(np.intersect1d(top, kept)) / nk)
        assert np.mean(shared) >= 0.65, (h, np.mean(shared))
