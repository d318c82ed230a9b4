"""da2_forward_noalloc: the whole path with the library's built-in device scratch.

Some callers cannot allocate device memory when they run the attention -- a plug-in
inside a host framework that owns all device memory, or a serving loop that forbids
cudaMalloc after start-up. This checks, through the C ABI, that the allocation-free entry
point gives the same output as da2_forward with a caller-owned workspace, on two calls in
a row (the second call reuses the scratch the first one left behind), and that a
configuration too large for the scratch is refused before anything runs.

Named so that pytest collects it last.
"""
import ctypes

import pytest
import torch

import sparse_mixed_precision_b200 as da2
from sparse_mixed_precision_b200.synth import WORKLOADS, generate, scaled

pytestmark = pytest.mark.gpu

ATOL, RTOL_L2 = 2e-2, 1e-2      # the parity tolerance of the other GPU tests


def _reference(w, q, k, v):
    cfg = da2.config(w)
    ws = torch.empty(da2.workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    da2.forward(cfg, q, k, v, out, ws)
    torch.cuda.synchronize()
    return out.float()


def test_noalloc_matches_forward_on_two_calls_in_a_row():
    for name, w in (("tiny", WORKLOADS["tiny"]), ("wan720-1head", scaled(WORKLOADS["wan720"], H=1))):
        q, k, v = generate(w, device="cuda")
        ref = _reference(w, q, k, v)
        cfg = da2.config(w)
        for call in range(2):
            out = torch.full_like(q, float("nan"))
            da2.forward_noalloc(cfg, q, k, v, out)
            torch.cuda.synchronize()
            assert da2.get_error(cfg, None) == 0, (name, call)   # the scratch's error word
            o = out.float()
            assert torch.isfinite(o).all(), (name, call)
            err = (o - ref).abs().max().item()
            rel = ((o - ref).norm() / ref.norm()).item()
            assert err <= ATOL and rel <= RTOL_L2, (name, call, err, rel)


def test_noalloc_refuses_a_workspace_larger_than_its_scratch():
    w = scaled(WORKLOADS["hunyuan720"], H=1)        # needs about 76 MiB of workspace
    cfg = da2.config(w)
    q = torch.empty((1, 1, w.T, w.d), dtype=torch.bfloat16, device="cuda")
    st = da2.lib().da2_forward_noalloc(ctypes.byref(cfg), ctypes.c_void_p(q.data_ptr()),
                                       ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(q.data_ptr()),
                                       ctypes.c_void_p(q.data_ptr()), None)
    assert st == 7
    assert b"64 MiB" in da2.lib().da2_status_string(7)


def test_noalloc_reports_a_wait_that_ran_out():
    # the built-in scratch's error word is readable: a call whose bounded wait must run out
    # (test-only flag) reports DA2_ERR_TIMEOUT through da2_get_error(NULL, ...); the next
    # normal call is again equal to da2_forward's output
    w = WORKLOADS["tiny"]
    q, k, v = generate(w, device="cuda")
    ref = _reference(w, q, k, v)
    out = torch.empty_like(q)
    cfg_stall = da2.config(w, flags=da2.FLAG_TEST_STALL)
    da2.forward_noalloc(cfg_stall, q, k, v, out)
    torch.cuda.synchronize()
    word = ctypes.c_uint32()
    st = da2.lib().da2_get_error(None, 0, ctypes.byref(cfg_stall),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                 ctypes.byref(word))
    assert st == 6 and (word.value & 1), (st, word.value)
    cfg = da2.config(w)
    da2.forward_noalloc(cfg, q, k, v, out)
    torch.cuda.synchronize()
    assert da2.get_error(cfg, None) == 0
    o = out.float()
    assert (o - ref).abs().max().item() <= ATOL and ((o - ref).norm() / ref.norm()).item() <= RTOL_L2
