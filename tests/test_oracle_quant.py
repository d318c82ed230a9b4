"""Pins of the oracle's quantisers against a library routine and brute force.

E4M3 is checked against torch's float8_e4m3fn conversion (an independent implementation
of the OCP FP8 format) on every finite bf16 input; E2M1 against a brute-force nearest
search over its 15 signed values with ties to the even code.
"""
import numpy as np
import pytest
import torch

import oracle as O


def all_finite_bf16():
    bits = torch.arange(0, 1 << 16, dtype=torch.int32).to(torch.int16)
    x = bits.view(torch.bfloat16).float()
    x = x[torch.isfinite(x)]
    return x.numpy().astype(np.float32)


def test_e4m3_matches_torch_on_all_bf16():
    x = all_finite_bf16()
    ref = torch.from_numpy(x).clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_code(x)
    assert np.array_equal(got, ref)
    assert np.array_equal(O.e4m3_decode(got), O.e4m3_round(x))


def test_e4m3_ties_go_to_even_code():
    codes = np.arange(0, 0x7F, dtype=np.uint8)           # non-negative finite codes
    vals = O.e4m3_decode(codes)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)  # exact in fp32
    got = O.e4m3_code(mids)
    ref = torch.from_numpy(mids).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(got, ref)
    assert np.all(got % 2 == 0)
    # saturation
    assert O.e4m3_code(np.float32(1e6)) == 0x7E and O.e4m3_code(np.float32(-1e6)) == 0xFE


def _e2m1_brute(x):
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    out = np.empty(x.shape, dtype=np.uint8)
    for n, v in enumerate(x.astype(np.float64)):
        a = min(abs(v), 6.0)
        dist = np.abs(grid - a)
        best = np.flatnonzero(dist == dist.min())
        idx = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
        out[n] = idx | (8 if np.signbit(v) else 0)
    return out


def test_e2m1_brute_force_on_all_bf16_in_range():
    x = all_finite_bf16()
    x = x[np.abs(x) <= 16]
    assert np.array_equal(O.e2m1_code(x), _e2m1_brute(x))


def test_e2m1_grid_and_ties():
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0], dtype=np.float32)
    assert list(O.e2m1_round(ties)) == [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0]
    codes = np.arange(16, dtype=np.uint8)
    assert np.array_equal(O.e2m1_code(O.e2m1_decode(codes).astype(np.float32)), codes)


def test_fp4_group_exact_when_scale_is_exact():
    # amax16 = 6 -> sigma = E4M3(1) = 1 exactly, so grid values survive unchanged
    rng = np.random.default_rng(0)
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6, -.5, -1, -1.5, -2, -3, -4, -6], np.float32)
    y = rng.choice(grid, size=(50, 32)).astype(np.float32)
    y[:, 0] = 6.0
    y[:, 16] = -6.0
    codes, sig = O.fp4_groups(y)
    assert np.all(O.e4m3_decode(sig) == 1.0)
    assert np.array_equal(O.fp4_dequant(codes, sig), y.astype(np.float64))


def test_fp4_group_error_bound_and_zero_groups():
    rng = np.random.default_rng(1)
    y = (rng.standard_normal((200, 64)) * rng.uniform(1e-3, 50, (200, 1))).astype(np.float32)
    y[:3, :16] = 0.0
    codes, sig = O.fp4_groups(y)
    deq = O.fp4_dequant(codes, sig)
    assert np.all(deq[:3, :16] == 0) and np.all(sig[:3, 0] == 0)
    yg = y.reshape(200, 4, 16).astype(np.float64)
    dg = deq.reshape(200, 4, 16)
    s = O.e4m3_decode(sig)[..., None]
    amax = np.abs(yg).max(-1, keepdims=True)
    # half a grid step (<= 1 sigma at the top binade) plus the sigma rounding (<= 1/16)
    assert np.all(np.abs(dg - yg) <= s * 1.0 + amax / 16 + 1e-12)


def test_outer_scale():
    amax = np.array([0.0, 1.0, 448.0, 3.5, 1e-20], np.float32)
    s, inv = O.outer_scale(amax)
    assert s[0] == 1 and inv[0] == 1
    assert np.allclose(s[1:] * 448, amax[1:], rtol=1e-7)
    assert np.allclose(inv[1:] * amax[1:], 448, rtol=1e-7)
