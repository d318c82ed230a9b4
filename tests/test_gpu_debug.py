"""Debug aids on a GPU: the workspace guard regions (DA2_FLAG_DEBUG_CANARY), the check of the
selection's output contract (da2_check_selection) and the DA2_DEBUG build of the library.

The corruptions these tests plant are ordinary writes from the host side into the test's
own workspace (a guard byte, one list entry, one tag) between two library calls; nothing
here makes a kernel read or write outside its buffers."""
import pytest
import torch

import sparse_mixed_precision_b200 as da2
from sparse_mixed_precision_b200.synth import WORKLOADS, generate, scaled

pytestmark = pytest.mark.gpu

REGIONS = ("q8", "k8", "v8", "q4", "k4", "v4", "sfq4", "sfk4", "sfv4", "sq", "sk", "sv", "vamax",
           "qavg", "qmax", "kavg", "kmax", "tags", "list8", "list4", "listm", "dlog", "qt", "kt", "err")

CASES = {
    "tiny": WORKLOADS["tiny"],
    "wan720-mixed-adaptive": scaled(WORKLOADS["wan720"], H=2, F=3, pct_fp8=10, pct_mix=5, pct_fp4=15,
                                    pct_fp4_max=35, adapt_tau=0.004),
}


def run(w, flags=0):
    q, k, v = generate(w, device="cuda")
    cfg = da2.config(w, flags=flags)
    ws = torch.zeros(da2.workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    da2.prepare(cfg, q, k, v, ws)
    da2.draft_select(cfg, ws)
    da2.attention(cfg, ws, out)
    torch.cuda.synchronize()
    return cfg, ws, out


def spans(views):
    """(start, end) of every region: up to the next region (or the end of the workspace)."""
    order = sorted(REGIONS, key=lambda r: views[r])
    ends = [views[order[i + 1]] for i in range(len(order) - 1)] + [views["total"]]
    return {r: (views[r], e) for r, e in zip(order, ends)}


@pytest.mark.parametrize("name", list(CASES))
def test_canary_run_matches_the_plain_run(name):
    w = CASES[name]
    cfg_p, ws_p, out_p = run(w)
    cfg_g, ws_g, out_g = run(w, flags=da2.FLAG_DEBUG_CANARY)
    assert da2.get_error(cfg_g, ws_g) == 0
    assert torch.equal(out_p, out_g)
    sp, sg = spans(da2.workspace_views(cfg_p)), spans(da2.workspace_views(cfg_g))
    for r in REGIONS:
        if r == "err":
            continue
        (a0, a1), (b0, _) = sp[r], sg[r]
        assert torch.equal(ws_p[a0:a1], ws_g[b0:b0 + (a1 - a0)]), r
        # the guard after the region still holds its pattern
        guard = ws_g[b0 + (a1 - a0):b0 + (a1 - a0) + 256]
        assert bool((guard == 0xA5).all()), r


def test_canary_catches_an_overwritten_guard_and_recovers():
    w = WORKLOADS["tiny"]
    q, k, v = generate(w, device="cuda")
    cfg = da2.config(w, flags=da2.FLAG_DEBUG_CANARY)
    ws = torch.zeros(da2.workspace_size(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q)
    views = da2.workspace_views(cfg)
    sg = spans(views)
    da2.prepare(cfg, q, k, v, ws)
    torch.cuda.synchronize()
    assert da2.get_error(cfg, ws) == 0
    # the guard after the tags region: the last 256 bytes before the next region
    guard_end = sg["tags"][1]
    ws[guard_end - 7] = 0
    da2.draft_select(cfg, ws)
    assert da2.get_error(cfg, ws) & 4                  # bit 4: a guard region changed
    # the next call refills the guards and clears the word
    da2.prepare(cfg, q, k, v, ws)
    da2.draft_select(cfg, ws)
    da2.attention(cfg, ws, out)
    torch.cuda.synchronize()
    assert da2.get_error(cfg, ws) == 0


@pytest.mark.parametrize("name", list(CASES))
def test_check_selection_accepts_the_selection(name):
    cfg, ws, _ = run(CASES[name])
    da2.check_selection(cfg, ws)
    assert da2.get_error(cfg, ws) == 0


@pytest.mark.parametrize("corruption", ["index_out_of_range", "not_ascending", "wrong_tag", "count"])
def test_check_selection_catches_a_broken_selection(corruption):
    w = CASES["wan720-mixed-adaptive"]
    cfg, ws, _ = run(w)
    v = da2.workspace_views(cfg)
    N, n8 = v["N"], v["n8"]
    l8 = ws[v["list8"]:v["list8"] + 2 * n8].view(torch.int16)          # row 0 of list8
    tags0 = ws[v["tags"]:v["tags"] + N]                                 # row 0 of tags
    if corruption == "index_out_of_range":
        l8[0] = N
    elif corruption == "not_ascending":
        a, b = int(l8[0]), int(l8[1])
        l8[0], l8[1] = b, a
    elif corruption == "wrong_tag":
        tags0[int(l8[0])] = 1
    else:                                                               # one FP8 tag too many
        skipped = torch.nonzero(tags0 == 0)
        tags0[int(skipped[0])] = 2
    torch.cuda.synchronize()
    da2.check_selection(cfg, ws)
    assert da2.get_error(cfg, ws) & 2                  # bit 2: bad index or count


@pytest.mark.parametrize("name", list(CASES))
def test_debug_build_matches_the_release_build(name):
    """libda2_debug.so (DA2_DEBUG: every stage waits and reports the error word, the selection
    is checked before the attention) gives the release build's bytes and output."""
    w = CASES[name]
    cfg_r, ws_r, out_r = run(w)
    prev = da2.use_library(da2.LIB_DEBUG_PATH)
    try:
        cfg_d, ws_d, out_d = run(w)
        assert da2.get_error(cfg_d, ws_d) == 0
    finally:
        da2.use_library(prev)
    assert torch.equal(out_r, out_d)
    sp = spans(da2.workspace_views(cfg_r))
    for r in REGIONS:
        if r != "err":
            a0, a1 = sp[r]
            assert torch.equal(ws_r[a0:a1], ws_d[a0:a1]), r


def test_debug_build_reports_a_set_error_word_at_the_call():
    """A DA2_DEBUG stage call waits for its stream and returns DA2_ERR_TIMEOUT as soon as the
    error word is set; the release build returns at once and leaves the word for
    da2_get_error. The word is set by the host between two calls (the draft kernels only
    ever set it, never read it)."""
    w = WORKLOADS["tiny"]
    cfg, ws, _ = run(w)
    err = da2.workspace_views(cfg)["err"]

    def draft_with_word_set():
        ws[err:err + 4] = torch.tensor([1, 0, 0, 0], dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()
        da2.draft_select(cfg, ws)
        torch.cuda.synchronize()

    draft_with_word_set()                                  # release build: no error raised
    assert da2.get_error(cfg, ws) == 1                     # the word was left for get_error
    prev = da2.use_library(da2.LIB_DEBUG_PATH)
    try:
        with pytest.raises(da2.DA2Error) as e:
            draft_with_word_set()
        assert e.value.status == 6
        assert da2.get_error(cfg, ws) == 1                 # still set; get_error clears it
        assert da2.get_error(cfg, ws) == 0
    finally:
        da2.use_library(prev)
