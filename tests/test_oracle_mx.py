"""Pins of the oracle's block-scaled FP8 variant (MXFP8: 32 elements share one E8M0 scale
2^e, elements are E4M3 values of x / 2^e) against brute force, torch's float8_e4m3fn
conversion and torch's scaled_dot_product_attention.

The shared exponent is checked against a search over every E8M0 exponent (the smallest e
with amax / 2^e below 512, the first power of two past E4M3's largest binade), not against
the logarithm the oracle takes; the elements against torch's cast of x / 2^e.
"""
import numpy as np
import pytest
import torch
import torch.nn.functional as Fnn

import oracle as O
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled, generate


def _exp_brute(amax: float) -> int:
    if amax == 0:
        return -127
    for e in range(-127, 128):
        if amax * 2.0 ** -e < 512.0:
            return e
    raise AssertionError("amax beyond the E8M0 range")


def _torch_e4m3(y):
    y = torch.as_tensor(np.asarray(y, dtype=np.float32)).clamp(-448, 448)
    return y.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def _mx_reference(x):
    """Blocks of 32 along the last axis: brute-force exponents, torch-cast elements."""
    x = np.asarray(x, dtype=np.float32)
    xb = x.reshape(x.shape[:-1] + (-1, 32))
    amax = np.abs(xb).max(axis=-1)
    e = np.vectorize(_exp_brute, otypes=[np.int64])(amax.astype(np.float64))
    y = (xb.astype(np.float64) * np.power(2.0, -e)[..., None]).astype(np.float32)
    codes = _torch_e4m3(y).reshape(x.shape)
    vals = torch.from_numpy(codes.reshape(xb.shape)).view(torch.float8_e4m3fn).double().numpy()
    return codes, e, (vals * np.power(2.0, e)[..., None]).reshape(x.shape)


def _random_blocks(rng, nblk):
    """Blocks whose magnitudes span many binades, each with its own range."""
    mag = 2.0 ** rng.uniform(-20, 20, size=(nblk, 1))
    x = rng.standard_normal((nblk, 32)) * mag * 2.0 ** rng.uniform(-6, 0, size=(nblk, 32))
    return x.astype(np.float32)


def test_shared_exponent_matches_search_over_e8m0():
    rng = np.random.default_rng(7)
    ks = np.arange(-110, 110)
    amax = np.concatenate([
        2.0 ** ks, 1.5 * 2.0 ** ks, 448 * 2.0 ** (ks - 8), 511.75 * 2.0 ** (ks - 8),
        2.0 ** rng.uniform(-118, 118, 2000), [0.0, 2.0 ** -126, 2.0 ** -130, 2.0 ** -149,
                                              np.finfo(np.float32).max]])
    got = O.e8m0_scale_exp(amax)
    ref = np.array([_exp_brute(a) for a in amax])
    assert np.array_equal(got, ref)
    assert O.e8m0_scale_exp(1.5 * 2.0 ** 3) == 3 - 8
    assert O.e8m0_scale_exp(0.0) == -127 and O.e8m0_scale_exp(2.0 ** -140) == -127


def test_elements_match_torch_cast_of_scaled_block():
    rng = np.random.default_rng(11)
    x = _random_blocks(rng, 4000)
    codes, e = O.quantise_mx8(x)
    rc, re_, rv = _mx_reference(x)
    assert np.array_equal(e[:, 0], re_[:, 0]) and e.shape == (4000, 1)
    assert np.array_equal(codes, rc)
    assert np.array_equal(O.dequant_mx8(codes, e), rv)


def test_known_values():
    k = 5
    x = np.zeros(32, np.float32)
    x[3] = 1.5 * 2 ** k
    codes, e = O.quantise_mx8(x)
    assert e[0] == k - 8
    assert O.e4m3_decode(codes[3]) == 384.0                # 1.5 * 2^8, exact in E4M3
    assert O.dequant_mx8(codes, e)[3] == x[3]
    x[3] = 448 * 2.0 ** -4                                 # top of E4M3's range
    codes, e = O.quantise_mx8(x)
    assert e[0] == -4 and O.e4m3_decode(codes[3]) == 448.0
    x[3] = 500.0                                           # 500 / 2^0 saturates
    codes, e = O.quantise_mx8(x)
    assert e[0] == 0 and codes[3] == 0x7E and O.dequant_mx8(codes, e)[3] == 448.0
    x[3] = -500.0
    codes, e = O.quantise_mx8(x)
    assert codes[3] == 0xFE
    codes, e = O.quantise_mx8(np.zeros(64, np.float32))
    assert np.array_equal(e, [-127, -127]) and not codes.any()


def test_powers_of_two_in_range_are_exact():
    for top in (-30, 0, 17):
        j = np.arange(top - 17, top + 1)               # 2^-9 .. 2^8 relative to the scale
        x = np.zeros(32, np.float32)
        x[:len(j)] = 2.0 ** j
        x[20] = -2.0 ** top
        codes, e = O.quantise_mx8(x)
        assert e[0] == top - 8
        assert np.array_equal(O.dequant_mx8(codes, e), x.astype(np.float64))


def test_roundtrip_error_bound():
    rng = np.random.default_rng(3)
    x = _random_blocks(rng, 3000).astype(np.float64)
    codes, e = O.quantise_mx8(x)
    err = np.abs(O.dequant_mx8(codes, e) - x)
    scale = np.power(2.0, e)                             # [nblk, 1], broadcasts over 32
    # E4M3 has 3 mantissa bits; below 2^-6 the quantum is 2^-9 (relative to the scale);
    # above 448 (a block max in [448, 512) times the scale) the element saturates.
    sat = np.abs(x) > 448 * scale
    assert sat.any()
    assert np.all((err <= np.maximum(np.abs(x) * 2.0 ** -4, scale * 2.0 ** -10))[~sat])
    deq = O.dequant_mx8(codes, e)
    assert np.array_equal(deq[sat], np.sign(x[sat]) * 448 * np.broadcast_to(scale, x.shape)[sat])
    # Every block's largest element lands in [256, 448] after scaling.
    y = np.abs(x).max(axis=1) / scale[:, 0]
    assert np.all((y >= 256) & (y < 512))


def test_blocks_are_independent_and_axis_is_respected():
    rng = np.random.default_rng(5)
    x = _random_blocks(rng, 6).reshape(2, 96)
    codes, e = O.quantise_mx8(x)
    for b in range(3):
        cb, eb = O.quantise_mx8(x[:, 32 * b:32 * (b + 1)])
        assert np.array_equal(codes[:, 32 * b:32 * (b + 1)], cb) and np.array_equal(e[:, b], eb[:, 0])
    y = x.copy()
    y[0, 40] *= 1e4                                      # only block 1 of row 0 changes
    cy, ey = O.quantise_mx8(y)
    assert ey[0, 1] != e[0, 1]
    keep = np.ones_like(codes, bool)
    keep[0, 32:64] = False
    assert np.array_equal(cy[keep], codes[keep])
    ct, et = O.quantise_mx8(x.T.copy(), axis=0)          # blocked along the first axis
    assert np.array_equal(ct.T, codes) and np.array_equal(et.T, e)


W_SMALL = scaled(WORKLOADS["tiny"], F=2, H=2)


def test_operand_blocking_follows_the_contraction_axes():
    q, k, v = generate(W_SMALL)
    prep = O.prepare(W_SMALL, q, k, v)
    qm, km, vm = O.quantise_mx_operands(prep["qp"], prep["kp"], prep["vp"])
    B, H, N, bs, d = prep["qp"].shape
    assert qm["e"].shape == (B, H, N, bs, d // 32) and km["e"].shape == (B, H, N, bs, d // 32)
    assert vm["e"].shape == (B, H, N, bs // 32, d)
    # V: one exponent per channel over 32 tokens of a key block
    rc, re_, rv = _mx_reference(np.swapaxes(prep["vp"], 3, 4))
    assert np.array_equal(np.swapaxes(vm["q8"], 3, 4), rc)
    assert np.array_equal(np.swapaxes(vm["e"], 3, 4), re_)
    rc, re_, rv = _mx_reference(prep["kp"])
    assert np.array_equal(km["q8"], rc) and np.array_equal(km["e"], re_)


def test_quant_p_mx():
    rng = np.random.default_rng(9)
    p = np.exp(-rng.exponential(4.0, size=(64, 128)))
    p[:, 5] = 1.0                                       # the row max of the first key group
    pq = O.quant_p_mx(p, 8)
    rc, re_, rv = _mx_reference(p)
    assert np.array_equal(pq, rv)
    assert np.all(re_[:, 0] == -8) and np.all(pq[:, 5] == 1.0)
    assert np.array_equal(O.quant_p_mx(p, 4), O.quant_p(p, 4))


def _sdpa(q, k, v, scale):
    q, k, v = (torch.as_tensor(np.asarray(x, dtype=np.float64)) for x in (q, k, v))
    return Fnn.scaled_dot_product_attention(q, k, v, scale=scale).numpy()


def test_full_fp8_budget_without_p_quantisation_is_dense_attention_on_mx_operands():
    w = scaled(W_SMALL, pct_fp8=100, pct_fp4=0)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    sel = O.draft_select(prep)
    mx = O.quantise_mx_operands(prep["qp"], prep["kp"], prep["vp"])
    ops = O.operands_mx(prep["Q"], prep["K"], prep["V"], *mx)
    o = O.attention(ops, prep["valid"], sel["list8"], sel["list4"], g.sm_scale, quantise_p=False)
    deq = [O.inverse_permute(_mx_reference(x)[2], g) for x in (prep["qp"], prep["kp"])]
    vd = np.swapaxes(_mx_reference(np.swapaxes(prep["vp"], 3, 4))[2], 3, 4)
    ref = _sdpa(deq[0], deq[1], O.inverse_permute(vd, g), g.sm_scale)
    assert np.abs(O.inverse_permute(o, g) - ref).max() < 1e-12


def test_one_key_block_with_p_quantisation_matches_closed_form():
    w = scaled(W_SMALL, pct_fp8=100, pct_fp4=0)
    q, k, v = generate(w)
    prep = O.prepare(w, q, k, v)
    g = prep["g"]
    B, H, N, bs, d = prep["qp"].shape
    mx = O.quantise_mx_operands(prep["qp"], prep["kp"], prep["vp"])
    ops = O.operands_mx(prep["Q"], prep["K"], prep["V"], *mx)
    j = 3
    list8 = np.full((B, H, N, 1), j)
    list4 = np.zeros((B, H, N, 0), dtype=np.int64)
    o = O.attention(ops, prep["valid"], list8, list4, g.sm_scale, pquant=O.quant_p_mx)
    qd = _mx_reference(prep["qp"])[2]
    kd = _mx_reference(prep["kp"])[2]
    vd = np.swapaxes(_mx_reference(np.swapaxes(prep["vp"], 3, 4))[2], 3, 4)
    for b, h, i in [(0, 0, 0), (0, 1, 7), (0, 1, N - 1)]:
        S = g.sm_scale * qd[b, h, i] @ kd[b, h, j].T
        p = np.exp(S - S.max(axis=1, keepdims=True))
        pq = _mx_reference(p)[2]
        ref = (pq @ vd[b, h, j]) / p.sum(axis=1, keepdims=True)
        assert np.abs(o[b, h, i] - ref).max() < 1e-13


def test_mx_keeps_small_tokens_of_a_block_with_an_outlier():
    """One token 2^12 times larger than the rest of its block: the per-block scale pushes
    the others into E4M3's subnormals, the per-32-channel scale does not."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((1, 1, 1, 32, 64)).astype(np.float32)
    x[..., 0, :] *= 4096
    valid = np.ones((1, 32), bool)
    per_block = O.dequant_qk(O.quantise_qk(x, valid), 8)
    codes, e = O.quantise_mx8(x)
    mx = O.dequant_mx8(codes, e)
    rest = slice(1, None)
    rel = lambda y: np.sqrt(np.mean(((y[..., rest, :] - x[..., rest, :]) / x[..., rest, :]) ** 2))
    assert rel(mx) <= 2.0 ** -5                          # RMS relative error of the others
    assert rel(per_block) > 4 * rel(mx)


def test_run_mx_changes_only_the_8bit_class():
    w = scaled(W_SMALL, pct_fp8=0, pct_fp4=100)
    q, k, v = generate(w)
    a = O.run(w, q, k, v)
    b = O.run(w, q, k, v, fp8="mx")
    assert np.array_equal(a["out"], b["out"])
    w8 = scaled(W_SMALL, pct_fp8=100, pct_fp4=0)
    q, k, v = generate(w8)
    exact = O.run(w8, q, k, v, quantised=False)["out"]
    e_mx = np.abs(O.run(w8, q, k, v, fp8="mx")["out"] - exact).max()
    e_sc = np.abs(O.run(w8, q, k, v)["out"] - exact).max()
    assert 0 < e_mx < 0.05 * np.abs(exact).max() and 0 < e_sc
    with pytest.raises(ValueError):
        O.run(w8, q, k, v, fp8="e5m2")
