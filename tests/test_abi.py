"""The C-ABI library loads and exports every symbol include/*.h declares; host-only calls
(workspace size / views, argument validation) behave as documented. No compute calls."""
import ctypes
import glob
import os
import re

import pytest

import sparse_mixed_precision_b200 as da2
from sparse_mixed_precision_b200.synth import WORKLOADS, scaled

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(da2_[a-z_0-9]+)\s*\(",
                                src, re.M))
    return names


def test_library_exports_every_declared_symbol():
    names = declared_symbols()
    assert {"da2_prepare", "da2_draft_select", "da2_attention"} <= names
    L = da2.lib()
    for n in sorted(names):
        assert hasattr(L, n), n
    assert set(da2.EXPORTED) >= names - set()  # the binding wraps every declared call


def test_workspace_views_consistent():
    for name in ("tiny", "wan480", "wan720", "hunyuan720"):
        w = WORKLOADS[name]
        cfg = da2.config(w)
        v = da2.workspace_views(cfg)
        assert v["total"] == da2.workspace_size(cfg)
        import oracle as O
        g = O.geometry(w)
        assert (v["N"], v["bs"], v["T"], v["Tp"], v["n8"], v["n4"]) == (g.N, g.bs, g.T, g.Tp, g.n8, g.n4)
        offs = sorted((v[k], k) for k in ("q8", "k8", "v8", "q4", "k4", "v4", "sfq4", "sfk4",
                                           "sfv4", "sq", "sk", "sv", "tags", "list8", "list4",
                                           "listm", "err"))
        assert all(o % 256 == 0 for o, _ in offs)
        assert len({o for o, _ in offs}) == len(offs)
    # exporting scores grows the workspace by 4 B H N^2 (rounded to 256)
    w = WORKLOADS["tiny"]
    a = da2.workspace_size(da2.config(w))
    b = da2.workspace_size(da2.config(w, flags=da2.FLAG_EXPORT_SCORES))
    assert b - a >= 4 * w.B * w.H * 64 * 64


@pytest.mark.parametrize("change,status", [
    (dict(d=96), 2), (dict(ph=3, pw=8), 2), (dict(pct_fp8=60, pct_fp4=50), 1),
    (dict(pct_fp8=-1), 1), (dict(B=0), 1), (dict(F=200, Hf=90, Wf=160), 2),
])
def test_invalid_configs_rejected(change, status):
    cfg = da2.config(scaled(WORKLOADS["tiny"], **change))
    n = ctypes.c_size_t()
    assert da2.lib().da2_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == status


def test_config_limits_and_degenerate_budgets():
    L = da2.lib()
    n = ctypes.c_size_t()
    w = WORKLOADS["tiny"]
    def status(cfg):
        return L.da2_workspace_size(ctypes.byref(cfg), ctypes.byref(n))
    # 4096 blocks is the largest supported per (b, h); one more is refused
    assert status(da2.config(scaled(w, F=32, Hf=64, Wf=64, ph=4, pw=8))) == 0      # N = 4096
    assert status(da2.config(scaled(w, F=33, Hf=64, Wf=64, ph=4, pw=8))) == 2      # N = 4224
    # a negative or non-finite softmax scale is an argument error; 0 selects 1/sqrt(d)
    assert status(da2.config(w, sm_scale=-1.0)) == 1
    assert status(da2.config(w, sm_scale=float("inf"))) == 1
    assert status(da2.config(w, sm_scale=0.0)) == 0
    # budgets: nothing kept, everything FP8, everything FP4 are all valid
    for f8, f4 in ((0, 0), (100, 0), (0, 100)):
        v = da2.workspace_views(da2.config(scaled(w, pct_fp8=f8, pct_fp4=f4)))
        assert v["n8"] == v["N"] * f8 // 100 and v["n4"] == v["N"] * f4 // 100


def test_flags_checked_and_layout_flag_keeps_the_workspace():
    L = da2.lib()
    n = ctypes.c_size_t()
    w = WORKLOADS["tiny"]
    assert L.da2_workspace_size(ctypes.byref(da2.config(w, flags=16)), ctypes.byref(n)) == 1
    # the token-major layout changes where q/k/v/out live, not the workspace
    assert da2.workspace_views(da2.config(w, flags=da2.FLAG_LAYOUT_BTHD)) == da2.workspace_views(da2.config(w))


def test_stage_calls_reject_bad_pointers_without_touching_the_device():
    L = da2.lib()
    cfg = da2.config(WORKLOADS["tiny"])
    n = da2.workspace_size(cfg)
    # null workspace / misaligned workspace / too-small workspace: checked on the host
    assert L.da2_draft_select(ctypes.byref(cfg), None, n, None) == 1
    assert L.da2_draft_select(ctypes.byref(cfg), ctypes.c_void_p(0x1008), n, None) == 3
    assert L.da2_draft_select(ctypes.byref(cfg), ctypes.c_void_p(0x100000), n - 1, None) == 4
    assert L.da2_prepare(ctypes.byref(cfg), None, None, None, ctypes.c_void_p(0x100000), n, None) == 1
    assert L.da2_status_string(6).startswith(b"device error word")


def test_noalloc_host_side_refusals():
    # da2_forward_noalloc checks its arguments before it touches the device: a missing or
    # invalid configuration, exported scores (they would stay in the hidden scratch), a
    # workspace larger than the 64 MiB scratch, missing tensors
    L = da2.lib()
    p = ctypes.c_void_p(0x100000)
    assert L.da2_forward_noalloc(None, p, p, p, p, None) == 1
    bad = da2.config(WORKLOADS["tiny"], flags=16)
    assert L.da2_forward_noalloc(ctypes.byref(bad), p, p, p, p, None) == 1
    assert L.da2_forward_noalloc(ctypes.byref(da2.config(scaled(WORKLOADS["tiny"], d=96))),
                                 p, p, p, p, None) == 2
    sc = da2.config(WORKLOADS["tiny"], flags=da2.FLAG_EXPORT_SCORES)
    assert L.da2_forward_noalloc(ctypes.byref(sc), p, p, p, p, None) == 1
    big = da2.config(WORKLOADS["wan720"])                       # about 2.2 GB of workspace
    assert da2.workspace_size(big) > 64 << 20
    assert L.da2_forward_noalloc(ctypes.byref(big), p, p, p, p, None) == 7
    tiny = da2.config(WORKLOADS["tiny"])
    assert L.da2_forward_noalloc(ctypes.byref(tiny), None, p, p, p, None) == 1
    assert L.da2_forward_noalloc(ctypes.byref(tiny), p, p, p, None, None) == 1
    # reading the scratch's error word needs a valid configuration first
    word = ctypes.c_uint32()
    assert L.da2_get_error(None, 0, ctypes.byref(bad), None, ctypes.byref(word)) == 1


def test_last_cuda_error_is_host_only():
    # no library call has failed with DA2_ERR_CUDA in this thread: cudaSuccess
    assert da2.lib().da2_last_cuda_error() == 0


def test_mixed_budget_counts_and_limits():
    # three cumulative cuts, each rounded half up; the percentages may not exceed 100
    L = da2.lib()
    n = ctypes.c_size_t()
    w = scaled(WORKLOADS["wan720"], pct_fp8=10, pct_mix=10, pct_fp4=20)
    v = da2.workspace_views(da2.config(w))
    assert (v["n8"], v["nm"], v["n4"]) == (63, 63, 126)
    v0 = da2.workspace_views(da2.config(WORKLOADS["wan720"]))
    assert (v0["n8"], v0["nm"], v0["n4"]) == (63, 0, 189)
    bad = da2.config(scaled(WORKLOADS["tiny"], pct_fp8=40, pct_mix=40, pct_fp4=30))
    assert L.da2_workspace_size(ctypes.byref(bad), ctypes.byref(n)) == 1
    neg = da2.config(scaled(WORKLOADS["tiny"], pct_mix=-1))
    assert L.da2_workspace_size(ctypes.byref(neg), ctypes.byref(n)) == 1


def test_adaptive_budget_views_and_limits():
    L = da2.lib()
    n = ctypes.c_size_t()
    w = scaled(WORKLOADS["wan720"], pct_fp8=10, pct_fp4=20, pct_fp4_max=40, adapt_tau=0.002)
    v = da2.workspace_views(da2.config(w))
    assert (v["n8"], v["n4"], v["n4max"]) == (63, 126, 252)       # cuts 63, 189, 315
    assert da2.workspace_views(da2.config(WORKLOADS["wan720"]))["n4max"] == 189
    for bad in (dict(pct_fp4_max=10, adapt_tau=0.01), dict(pct_fp4_max=90, adapt_tau=0.01),
                dict(pct_fp4_max=50, adapt_tau=-1.0), dict(pct_fp4_max=50, adapt_tau=float("inf"))):
        cfg = da2.config(scaled(WORKLOADS["tiny"], **bad))
        assert L.da2_workspace_size(ctypes.byref(cfg), ctypes.byref(n)) == 1, bad


REGIONS = ("q8", "k8", "v8", "q4", "k4", "v4", "sfq4", "sfk4", "sfv4", "sq", "sk", "sv", "vamax",
           "qavg", "qmax", "kavg", "kmax", "tags", "list8", "list4", "listm", "dlog", "qt", "kt", "err")


@pytest.mark.parametrize("name", ["tiny", "wan720", "hunyuan720"])
def test_canary_layout_puts_a_guard_after_every_region(name):
    """DA2_FLAG_DEBUG_CANARY: every region keeps its size and is followed by at least 256
    bytes that no region uses; the workspace grows by one guard per region."""
    w = WORKLOADS[name]
    plain = da2.workspace_views(da2.config(w))
    guarded = da2.workspace_views(da2.config(w, flags=da2.FLAG_DEBUG_CANARY))
    for k in ("N", "bs", "n8", "n4", "n4max", "nm", "tile8_qk", "tile4_qk", "tile8_v", "tile4_v"):
        assert guarded[k] == plain[k], k

    def spans(v):
        order = sorted(REGIONS, key=lambda r: v[r])
        nxt = {r: (v[order[i + 1]] if i + 1 < len(order) else v["total"]) for i, r in enumerate(order)}
        return order, nxt

    order_p, next_p = spans(plain)
    order_g, next_g = spans(guarded)
    assert order_p == order_g
    for r in order_g:
        # the region's bytes in the plain layout (up to its 256-byte rounding) are followed
        # by a guard of at least 256 bytes in the guarded layout
        size = next_p[r] - plain[r]
        assert next_g[r] - guarded[r] >= size + 256, r
    assert guarded["total"] >= plain["total"] + 256 * len(REGIONS)


def test_debug_library_exports_every_declared_symbol():
    """The DA2_DEBUG build (built by __graft_entry__.build) exports the same C ABI."""
    if not os.path.exists(da2.LIB_DEBUG_PATH):
        pytest.skip("libda2_debug.so not built")
    L = ctypes.CDLL(da2.LIB_DEBUG_PATH)
    for n in sorted(declared_symbols()):
        assert hasattr(L, n), n


def test_check_selection_rejects_bad_arguments_without_touching_the_device():
    L = da2.lib()
    cfg = da2.config(WORKLOADS["tiny"])
    n = da2.workspace_size(cfg)
    assert L.da2_check_selection(None, ctypes.c_void_p(0x100000), n, None) == 1
    assert L.da2_check_selection(ctypes.byref(cfg), None, n, None) == 1
    assert L.da2_check_selection(ctypes.byref(cfg), ctypes.c_void_p(0x1008), n, None) == 3
    assert L.da2_check_selection(ctypes.byref(cfg), ctypes.c_void_p(0x100000), n - 1, None) == 4


def test_binding_refuses_a_bf16_budget():
    # the bf16 tier exists in the oracle only: a configuration with bf16 blocks is refused
    # instead of being run as if those blocks were skipped
    with pytest.raises(ValueError, match="bf16"):
        da2.config(scaled(WORKLOADS["tiny"], pct_bf16=5))
    assert da2.config(scaled(WORKLOADS["tiny"], pct_bf16=0)).pct_fp8 == WORKLOADS["tiny"].pct_fp8


def test_config_checks_cannot_overflow():
    # budgets and shapes far outside the supported set are refused before any sum or product
    # of them can overflow a machine integer
    L = da2.lib()
    n = ctypes.c_size_t()
    w = WORKLOADS["tiny"]
    big = 2 ** 31 - 1

    def status(**change):
        cfg = da2.config(scaled(w, **change))
        return L.da2_workspace_size(ctypes.byref(cfg), ctypes.byref(n))
    assert status(pct_fp8=big, pct_fp4=1) == 1            # the sum wraps below 100 in 32 bits
    assert status(pct_fp8=big, pct_fp4=big, pct_mix=2) == 1
    assert status(pct_fp4=101, pct_fp8=0) == 1
    assert status(adapt_tau=0.5, pct_fp4_max=big) == 1
    assert status(Hf=big) == 2                            # Hf + ph - 1 wraps in 32 bits
    assert status(Wf=big, Hf=1) == 2
    assert status(F=big, Hf=4, Wf=8) == 2                 # one block per frame, 2^31 - 1 frames
    assert status(B=2 ** 20, H=2 ** 20) == 2              # B * H * N * N wraps in 64 bits
    assert status(B=1, H=65535) == 0                      # the largest head count
    assert status(B=1, H=65536) == 2                      # one more than the grid's y axis
    assert status(B=3, H=21846) == 2


def test_plain_c_caller(tmp_path):
    # the boundary is plain C: a C99 program includes the header, links the library and
    # sizes a workspace and its views without Python or torch (host-only calls, no GPU)
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    cuda_inc = "/usr/local/cuda/include"
    if gcc is None or not os.path.isdir(cuda_inc):
        pytest.skip("gcc or the CUDA headers are not installed")
    src = tmp_path / "caller.c"
    src.write_text(r"""
#include <stdio.h>
#include "da2.h"
int main(void) {
  da2_config c = {0};
  c.B = 1; c.H = 2; c.d = 64; c.F = 4; c.Hf = 16; c.Wf = 32; c.ph = 4; c.pw = 8;
  c.pct_fp8 = 15; c.pct_fp4 = 35;
  size_t bytes = 0;
  da2_views v;
  if (da2_workspace_size(&c, &bytes) != DA2_OK) return 1;
  if (da2_workspace_views(&c, &v) != DA2_OK) return 2;
  c.d = 96;
  if (da2_workspace_size(&c, &bytes) != DA2_ERR_UNSUPPORTED) return 3;
  printf("%zu %d %d %d %s\n", v.total, v.N, v.n8, v.n4, da2_status_string(DA2_ERR_WORKSPACE));
  return 0;
}
""")
    libdir = os.path.dirname(da2.LIB_PATH)
    exe = tmp_path / "caller"
    subprocess.run([gcc, "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                    str(src), "-o", str(exe), "-L", libdir, "-l:libda2.so", f"-Wl,-rpath,{libdir}"],
                   check=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    v = da2.workspace_views(da2.config(WORKLOADS["tiny"]))
    assert [int(x) for x in out[:4]] == [v["total"], v["N"], v["n8"], v["n4"]]
    assert " ".join(out[4:]) == "workspace too small"


def test_binding_checks_tensors_before_the_library_sees_them():
    # the C ABI receives bare pointers, so the binding rejects a tensor of the wrong type,
    # shape, layout or placement before any call (these raise on a machine without a GPU)
    import torch
    w = WORKLOADS["tiny"]
    cfg = da2.config(w)
    shape = (w.B, w.H, w.F * w.Hf * w.Wf, w.d)
    assert da2.activation_shape(cfg) == shape
    assert da2.activation_shape(da2.config(w, flags=da2.FLAG_LAYOUT_BTHD)) == (shape[0], shape[2], shape[1], shape[3])
    bf = lambda s=shape: torch.zeros(s, dtype=torch.bfloat16)
    ws = torch.zeros(16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="bfloat16"):
        da2.forward(cfg, bf(), bf(), torch.zeros(shape), bf(), ws)
    with pytest.raises(ValueError, match="shape"):
        da2.prepare(cfg, bf(), bf(), bf((w.B, w.H, 100, w.d)), ws)
    with pytest.raises(ValueError, match="shape"):                 # token-major tensor, head-major config
        da2.forward(cfg, *(bf((shape[0], shape[2], shape[1], shape[3])) for _ in range(4)), ws)
    nc = torch.zeros((shape[0], shape[2], shape[1], shape[3]), dtype=torch.bfloat16).transpose(1, 2)
    with pytest.raises(ValueError, match="contiguous"):
        da2.forward(cfg, nc, bf(), bf(), bf(), ws)
    with pytest.raises(ValueError, match="CUDA tensor"):           # host memory handed to a kernel
        da2.forward(cfg, bf(), bf(), bf(), bf(), ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        da2.draft_select(cfg, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        da2.forward_noalloc(cfg, bf(), bf(), bf(), bf())
    with pytest.raises(TypeError):
        da2.attention(cfg, None, bf())
    # host-buffer call: host tensors on the host, staging buffers and workspace on the device
    with pytest.raises(ValueError, match="shape"):
        da2.forward_host(cfg, bf(), bf(), bf(), bf((1, 2, 3, 4)), bf(), bf(), bf(), bf(), ws)
    with pytest.raises(ValueError, match="dq must be a CUDA tensor"):
        da2.forward_host(cfg, bf(), bf(), bf(), bf(), bf(), bf(), bf(), bf(), ws)
