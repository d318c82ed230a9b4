"""Pins of the oracle's bf16 top tier (a class above FP8 in the shared ranking).

"DraftAttention2: Fast Video Diffusion with Low-Resolution-Guided Mixed-Precision
Attention", Abstract: higher precision for the more important blocks, lower precision for
the rest. Reading: bf16, the inputs' own precision, is the highest class; its blocks run
Q K^T and P V on the input values with P rounded to bf16, first in the phase order, under
the same online softmax. Only the oracle implements the tier.

Independent references: hand-derived values (tests/golden/bf16_tier.json), torch's
fp32 -> bf16 conversion, hand-computed budget cuts, a brute-force sort and torch SDPA.
"""
import json
import pathlib

import numpy as np
import torch
import torch.nn.functional as Fnn

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate

GOLDEN = json.loads((pathlib.Path(__file__).parent / "golden" / "bf16_tier.json").read_text())


def test_bf16_round_hand_values():
    for c in GOLDEN["round"]:
        assert O.bf16_round(c["x"]) == c["expected"], c["why"]


def test_bf16_round_matches_torch_on_fp32_values():
    # every fp32 value is exact in fp64, so torch's single rounding fp32 -> bf16 is the
    # reference; random bit patterns cover all binades, subnormals and overflow to inf
    rng = np.random.default_rng(16)
    bits = rng.integers(0, 2 ** 32, size=1 << 18, dtype=np.uint64).astype(np.uint32)
    # plus every tie and near-tie around 1 and around the bf16 subnormal / normal boundary
    near = np.array([0x3F800000 + i for i in range(0, 1 << 17, 97)] +
                    [0x00800000 + i for i in range(-4096, 4096, 3)], dtype=np.uint32)
    x = np.concatenate([bits, near]).view(np.float32)
    x = x[np.isfinite(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).double().numpy()
    got = O.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, want)


def test_budget_counts_with_a_bf16_tier():
    # cumulative cuts floor((p N + 50) / 100), worked out by hand
    assert O.budget_counts_tiers(630, 5, 10, 10, 20) == (32, 63, 63, 126)   # cuts 32, 95, 158, 284
    assert O.budget_counts_tiers(64, 10, 15, 0, 25) == (6, 10, 0, 16)       # cuts 6, 16, 16, 32
    for N, p8, pm, p4 in ((630, 10, 10, 20), (64, 15, 0, 35), (990, 5, 0, 25)):
        assert O.budget_counts_tiers(N, 0, p8, pm, p4) == (0,) + O.budget_counts3(N, p8, pm, p4)


def test_rank_with_a_bf16_tier_brute_force():
    rng = np.random.default_rng(9)
    N = 64
    sc = rng.random((16, N))
    sc[:, 5:12] = sc[:, 5:6]                           # ties resolved by block index
    n16, n8, nm, n4 = 4, 6, 5, 16
    r = O.rank_classes(sc, n8, nm, n4, n16)
    ra = O.rank_adaptive(sc, n8, nm, n4, n4 + 8, 0.5, n16)
    for row in range(sc.shape[0]):
        order = sorted(range(N), key=lambda j: (-sc[row, j], j))
        cuts = np.cumsum([0, n16, n8, nm, n4])
        for name, a, b in zip(("list16", "list8", "listm", "list4"), cuts[:-1], cuts[1:]):
            assert list(r[name][row]) == sorted(order[a:b])
        want = np.zeros(N, np.uint8)
        for tag, a, b in zip((O.TAG_BF16, O.TAG_FP8, O.TAG_MIX, O.TAG_FP4), cuts[:-1], cuts[1:]):
            want[order[a:b]] = tag
        assert np.array_equal(r["tags"][row], want)
        # adaptive budget: blocks after all four cuts, in rank order, join FP4 while their
        # score reaches the threshold, up to 8 more
        extra = [j for j in order[cuts[-1]:cuts[-1] + 8] if sc[row, j] >= 0.5]
        extra = order[cuts[-1]:cuts[-1] + len(extra)]
        want4 = sorted(order[cuts[3]:cuts[4]] + list(extra))
        assert list(ra["list4"][row][:len(want4)]) == want4
        assert list(ra["list16"][row]) == sorted(order[:n16])


def test_bf16_phase_rounds_p_to_bf16_and_sums_it_unrounded():
    a = GOLDEN["attention"]
    x = np.array(a["x"])
    bs = d = 16
    q = np.zeros((1, 1, 1, bs, d))
    q[..., 0] = 1.0
    k = np.zeros((1, 1, 1, bs, d))
    k[0, 0, 0, :, 0] = np.log(x)
    v = np.eye(bs)[None, None, None]
    ops = O.Operands({16: q, 8: q, 4: q}, {16: k, 8: k, 4: k}, {16: v, 8: v, 4: v})
    valid = np.ones((1, bs), dtype=bool)
    none = np.zeros((1, 1, 1, 0), dtype=np.int64)
    one = np.zeros((1, 1, 1, 1), dtype=np.int64)
    out = O.attention(ops, valid, none, none, 1.0, quantise_p=True, list16=one)
    want = np.array(a["kept"]) / x.sum()
    assert np.abs(out[0, 0, 0] - want[None, :]).max() < 1e-14
    # 8-bit probabilities would differ: the check above tells the precisions apart
    assert np.abs(O.quant_p(x, 8) - np.array(a["kept"])).max() > 1e-3


W = scaled(WORKLOADS["tiny"], F=2, H=2)


def _dense(q, k, v, scale, mask=None):
    q, k, v = (torch.from_numpy(x.float().numpy()).double() for x in (q, k, v))
    m = None if mask is None else torch.from_numpy(mask)
    return Fnn.scaled_dot_product_attention(q, k, v, attn_mask=m, scale=scale).numpy()


def test_bf16_tier_on_every_block_is_attention_on_the_inputs():
    w = scaled(W, pct_bf16=100, pct_fp8=0, pct_fp4=0)
    q, k, v = generate(w)
    r = O.run(w, q, k, v)
    g = r["prep"]["g"]
    assert (g.n16, g.n8, g.nm, g.n4) == (g.N, 0, 0, 0)
    assert (r["sel"]["tags"] == O.TAG_BF16).all()
    ref = _dense(q, k, v, g.sm_scale)
    err16 = np.abs(r["out"] - ref).max()
    # P rounded to bf16 (relative step 2^-8 at most): the output moves by well under 1 %
    assert 0 < err16 < 4e-3 * np.abs(ref).max()
    # unrounded P: the textbook attention of the bf16 inputs
    r0 = O.run(w, q, k, v, quantised=False)
    assert np.abs(r0["out"] - ref).max() < 1e-12
    # the same blocks at FP8 are an order of magnitude less accurate
    w8 = scaled(W, pct_bf16=0, pct_fp8=100, pct_fp4=0)
    err8 = np.abs(O.run(w8, q, k, v)["out"] - ref).max()
    assert err8 > 10 * err16


def test_five_class_split_without_p_quantisation_is_masked_attention():
    # exact operands and unquantised P: the class of a block does not matter, only the kept
    # set does (one softmax state and accumulator across all four phases)
    w = scaled(W, pct_bf16=5, pct_fp8=10, pct_mix=10, pct_fp4=20)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    assert g.n16 > 0 and g.n8 > 0 and g.nm > 0 and g.n4 > 0
    ops = O.operands_exact(prep["qp"], prep["kp"], prep["vp"])
    o = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, False,
                    listm=sel["listm"], list16=sel["list16"])
    blk, _ = O.token_block_slot(g)
    kept = sel["tags"] > 0
    assert (kept.sum(-1) == g.n16 + g.n8 + g.nm + g.n4).all()
    mask = kept[:, :, blk][:, :, :, blk]
    ref = _dense(q, k, v, g.sm_scale, mask)
    assert np.abs(O.inverse_permute(o, g) - ref).max() < 1e-12


def test_bf16_tier_takes_the_top_ranked_blocks_and_lowers_the_error():
    # same kept set (top 50 %, all 8-bit), the top 10 % moved from FP8 to bf16: those
    # blocks carry the most mass, so the quantisation error drops well below the all-FP8 one
    w1 = scaled(W, pct_bf16=10, pct_fp8=40, pct_fp4=0)
    w0 = scaled(W, pct_bf16=0, pct_fp8=50, pct_fp4=0)
    q, k, v = generate(w1)
    r1, r0 = O.run(w1, q, k, v), O.run(w0, q, k, v)
    s1, s0 = r1["sel"], r0["sel"]
    assert np.array_equal(s1["tags"] > 0, s0["tags"] > 0)
    sc = s1["scores"]
    lo16 = np.where(s1["tags"] == O.TAG_BF16, sc, np.inf).min(-1)
    hi8 = np.where(s1["tags"] == O.TAG_FP8, sc, -np.inf).max(-1)
    assert (lo16 >= hi8).all()
    assert np.array_equal(np.sort(np.concatenate([s1["list16"], s1["list8"]], -1), -1), s0["list8"])
    g = r1["prep"]["g"]
    blk, _ = O.token_block_slot(g)
    kept = s1["tags"] > 0
    ref = _dense(q, k, v, g.sm_scale, kept[:, :, blk][:, :, :, blk])
    e1 = np.linalg.norm(r1["out"] - ref)
    e0 = np.linalg.norm(r0["out"] - ref)
    assert e1 < 0.9 * e0
