"""Failure detection on the GPU without a fault: a bounded device wait that runs out.

The test-only flag DA2_FLAG_TEST_STALL makes the attention kernel's copy engine withhold
its first K/V tile (nothing will ever complete that stage) and shortens every bounded wait
to 50 ms. The launch must then record the timeout in the workspace error word, drain and
end on its own; da2_get_error reports DA2_ERR_TIMEOUT and clears the word; the context
stays usable, and the next normal call matches the CPU oracle.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle as O
import sparse_mixed_precision_b200 as da2
from sparse_mixed_precision_b200.synth import WORKLOADS, generate
from layout import WsReader

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_then_the_next_call_is_correct():
    w = WORKLOADS["tiny"]
    q, k, v = generate(w, device="cuda")
    cfg_stall = da2.config(w, flags=da2.FLAG_TEST_STALL)
    ws = torch.empty(da2.workspace_size(cfg_stall), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    da2.forward(cfg_stall, q, k, v, out, ws)
    torch.cuda.synchronize()
    elapsed = time.perf_counter() - t0
    word = ctypes.c_uint32()
    st = da2.lib().da2_get_error(ctypes.c_void_p(ws.data_ptr()), ws.numel(), ctypes.byref(cfg_stall),
                                 ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                 ctypes.byref(word))
    assert st == 6 and (word.value & 1), (st, word.value)    # DA2_ERR_TIMEOUT, wait-timeout bit
    assert elapsed < 5.0, elapsed                              # 50 ms limits, not the 2 s ones
    assert da2.get_error(cfg_stall, ws) == 0                   # reading cleared the word

    # the same context, a normal call: equal to the oracle on the CUDA path's selection
    cfg = da2.config(w)
    out = torch.full_like(q, float("nan"))
    da2.forward(cfg, q, k, v, out, ws)
    torch.cuda.synchronize()
    assert da2.get_error(cfg, ws) == 0
    rd = WsReader(ws, da2.workspace_views(cfg), w.d)
    l8, l4 = rd.lists(0, w.B * w.H)
    r = O.run(w, q.cpu(), k.cpu(), v.cpu(), quantised=True,
              lists=(l8.reshape(w.B, w.H, *l8.shape[1:]), l4.reshape(w.B, w.H, *l4.shape[1:])))
    got = out.float().cpu().numpy()
    err = np.abs(got - r["out"]).max()
    rel = np.linalg.norm(got - r["out"]) / np.linalg.norm(r["out"])
    assert err <= 2e-2 and rel <= 1e-2, (err, rel)
