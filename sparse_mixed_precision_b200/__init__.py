"""Python binding of libda2 (the DraftAttention2 hot path on B200, sm_100a).

Argument marshalling only: every step of the path runs in the CUDA library. The names
follow the C ABI in include/da2.h. Because that ABI receives bare pointers, the binding
checks each tensor's dtype, shape, contiguity and device before a call. Tensors are torch tensors (device memory and streams
come from PyTorch); the library itself allocates no device memory.

    cfg = config(workload)                      # da2_config from a synth.Workload
    ws  = torch.empty(workspace_size(cfg), dtype=torch.uint8, device="cuda")
    prepare(cfg, q, k, v, ws); draft_select(cfg, ws); attention(cfg, ws, out)

Token-major activations ([B, T, H, d], heads of one token adjacent) go in as they are with
`config(w, flags=FLAG_LAYOUT_BTHD)`. Sequence-parallel callers (each rank holding T/P of
the tokens) exchange to all tokens of H/P heads with `seqpar.seq_to_heads` before the call
and back with `seqpar.heads_to_seq` after it. `forward_host` takes pinned host buffers and
overlaps the copies with the compute over groups of heads.

The extension must be built first (`python -m sparse_mixed_precision_b200.build` or
`__graft_entry__.build()`); there is no fallback when it is missing.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libda2.so")
LIB_DEBUG_PATH = os.path.join(_HERE, "libda2_debug.so")   # DA2_DEBUG build (see use_library)

FLAG_EXPORT_SCORES = 1
FLAG_NO_MASS_CORRECTION = 2
FLAG_LAYOUT_BTHD = 4          # q, k, v, out token-major [B, T, H, d]
FLAG_DEBUG_CANARY = 8         # guard region after every workspace region, checked per stage
FLAG_TEST_STALL = 256         # test hook: a bounded wait of the attention kernel runs out

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "misaligned pointer",
          4: "workspace too small", 5: "CUDA error", 6: "device error word set",
          7: "workspace larger than the built-in 64 MiB device scratch"}


class Config(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "H", "d", "F", "Hf", "Wf", "ph", "pw",
                                             "pct_fp8", "pct_fp4")] + \
               [("sm_scale", ctypes.c_float), ("flags", ctypes.c_int), ("pct_mix", ctypes.c_int),
                ("adapt_tau", ctypes.c_float), ("pct_fp4_max", ctypes.c_int)]


_VIEW_INTS = ("N", "bs", "T", "Tp", "ny", "nx", "n8", "n4", "kv4")
_VIEW_SIZES = ("tile8_qk", "tile4_qk", "tile8_v", "tile4_v", "sf_qk", "sf_v",
               "q8", "k8", "v8", "q4", "k4", "v4", "sfq4", "sfk4", "sfv4",
               "sq", "sk", "sv", "vamax", "qavg", "qmax", "kavg", "kmax",
               "tags", "list8", "list4", "scores", "err", "total")


class Views(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in _VIEW_INTS] + [(n, ctypes.c_size_t) for n in _VIEW_SIZES] + \
               [("nm", ctypes.c_int), ("listm", ctypes.c_size_t), ("n4max", ctypes.c_int),
                ("dlog", ctypes.c_size_t), ("np", ctypes.c_int), ("qt", ctypes.c_size_t),
                ("kt", ctypes.c_size_t)]


class DA2Error(RuntimeError):
    def __init__(self, fn, status):
        detail = ""
        if status == 5 and _lib is not None and hasattr(_lib, "da2_last_cuda_error"):
            detail = f", cudaError_t {_lib.da2_last_cuda_error()}"
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status}{detail})")
        self.status = status


_lib = None


def use_library(path: str) -> str:
    """Selects the build of the library that the binding calls from the next call on (for
    example LIB_DEBUG_PATH, built by `python -m sparse_mixed_precision_b200.build --debug`);
    returns the previous path."""
    global LIB_PATH, _lib
    prev, LIB_PATH, _lib = LIB_PATH, path, None
    return prev


def lib():
    """The loaded library (libda2.so unless use_library chose another build); raises if it
    has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{os.path.basename(LIB_PATH)} not built ({LIB_PATH}); "
                               "run sparse_mixed_precision_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, sz, cp = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(Config)
        sigs = {
            "da2_workspace_size": [cp, ctypes.POINTER(ctypes.c_size_t)],
            "da2_workspace_views": [cp, ctypes.POINTER(Views)],
            "da2_prepare": [cp, vp, vp, vp, vp, sz, vp],
            "da2_draft_select": [cp, vp, sz, vp],
            "da2_attention": [cp, vp, sz, vp, vp],
            "da2_forward": [cp, vp, vp, vp, vp, vp, sz, vp],
            "da2_forward_host": [cp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp],
            "da2_get_error": [vp, sz, cp, vp, ctypes.POINTER(ctypes.c_uint32)],
            "da2_forward_noalloc": [cp, vp, vp, vp, vp, vp],
            "da2_check_selection": [cp, vp, sz, vp],
        }
        for name, args in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = args
            fn.restype = ctypes.c_int
        if hasattr(L, "da2_last_cuda_error"):
            L.da2_last_cuda_error.argtypes = []
            L.da2_last_cuda_error.restype = ctypes.c_int
        L.da2_status_string.argtypes = [ctypes.c_int]
        L.da2_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


EXPORTED = ("da2_workspace_size", "da2_workspace_views", "da2_prepare", "da2_draft_select",
            "da2_attention", "da2_forward", "da2_forward_host", "da2_get_error",
            "da2_status_string", "da2_forward_noalloc", "da2_last_cuda_error",
            "da2_check_selection")


def config(w, flags: int = 0, sm_scale: float = 0.0) -> Config:
    """da2_config of a synth.Workload (or any object with the same fields).

    The library has no bf16 tier (a workload with pct_bf16 > 0): such a workload is refused
    here rather than run without its bf16 blocks."""
    if int(getattr(w, "pct_bf16", 0)) != 0:
        raise ValueError("the library has no bf16 tier: pct_bf16 must be 0")
    return Config(w.B, w.H, w.d, w.F, w.Hf, w.Wf, w.ph, w.pw, w.pct_fp8, w.pct_fp4,
                  float(sm_scale), int(flags), int(getattr(w, "pct_mix", 0)),
                  float(getattr(w, "adapt_tau", 0.0)), int(getattr(w, "pct_fp4_max", 0)))


def _check(fn, st):
    if st != 0:
        raise DA2Error(fn, st)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def activation_shape(cfg: Config) -> tuple:
    """Shape of q, k, v and out for a configuration: [B, H, T, d], or [B, T, H, d] with
    FLAG_LAYOUT_BTHD (T = F * Hf * Wf)."""
    T = cfg.F * cfg.Hf * cfg.Wf
    return (cfg.B, T, cfg.H, cfg.d) if cfg.flags & FLAG_LAYOUT_BTHD else (cfg.B, cfg.H, T, cfg.d)


def _check_tensors(fn, cfg, acts, bufs=(), host=(), stream=None):
    """The C ABI takes plain pointers and cannot see a tensor's size, type or placement, so
    the binding checks them before the call: a wrong tensor raises here instead of sending
    a kernel out of bounds. acts: (name, tensor) pairs of bf16 activations on the device;
    host: the same on the host (forward_host); bufs: byte buffers (the workspace) on the
    device. Every device tensor must sit on the device of the stream the call runs on."""
    import torch
    want = activation_shape(cfg)
    for name, t in list(acts) + list(host):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{fn}: {name} must be a torch.Tensor")
        if t.dtype != torch.bfloat16:
            raise ValueError(f"{fn}: {name} must be bfloat16, not {t.dtype}")
        if tuple(t.shape) != want:
            raise ValueError(f"{fn}: {name} has shape {tuple(t.shape)}; the configuration needs {want}")
    for name, t in list(acts) + list(host) + list(bufs):
        if not isinstance(t, torch.Tensor):
            raise TypeError(f"{fn}: {name} must be a torch.Tensor")
        if not t.is_contiguous():
            raise ValueError(f"{fn}: {name} must be contiguous")
    for name, t in host:
        if t.device.type != "cpu":
            raise ValueError(f"{fn}: {name} must be a host tensor, not on {t.device}")
    dev = list(acts) + list(bufs)
    for name, t in dev:
        if t.device.type != "cuda":
            raise ValueError(f"{fn}: {name} must be a CUDA tensor, not on {t.device}")
    if dev:
        sdev = (torch.cuda.current_stream() if stream is None else stream).device
        for name, t in dev:
            if t.device != sdev:
                raise ValueError(f"{fn}: {name} is on {t.device} but the call runs on {sdev}")


def _nbytes(t):
    return t.numel() * t.element_size()


def _stream(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def workspace_size(cfg: Config) -> int:
    n = ctypes.c_size_t()
    _check("da2_workspace_size", lib().da2_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def workspace_views(cfg: Config) -> dict:
    v = Views()
    _check("da2_workspace_views", lib().da2_workspace_views(ctypes.byref(cfg), ctypes.byref(v)))
    return {n: getattr(v, n) for n in _VIEW_INTS + _VIEW_SIZES + ("nm", "listm", "n4max", "dlog", "np", "qt", "kt")}


def prepare(cfg, q, k, v, ws, stream=None):
    _check_tensors("da2_prepare", cfg, (("q", q), ("k", k), ("v", v)), (("ws", ws),), stream=stream)
    _check("da2_prepare", lib().da2_prepare(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(ws), _nbytes(ws), _stream(stream)))


def draft_select(cfg, ws, stream=None):
    _check_tensors("da2_draft_select", cfg, (), (("ws", ws),), stream=stream)
    _check("da2_draft_select", lib().da2_draft_select(ctypes.byref(cfg), _ptr(ws), _nbytes(ws),
                                                      _stream(stream)))


def check_selection(cfg, ws, stream=None):
    """Debug aid: checks the selection's lists and tags in ws (da2_check_selection); a
    violation shows up in get_error."""
    _check_tensors("da2_check_selection", cfg, (), (("ws", ws),), stream=stream)
    _check("da2_check_selection", lib().da2_check_selection(ctypes.byref(cfg), _ptr(ws), _nbytes(ws),
                                                            _stream(stream)))


def attention(cfg, ws, out, stream=None):
    _check_tensors("da2_attention", cfg, (("out", out),), (("ws", ws),), stream=stream)
    _check("da2_attention", lib().da2_attention(ctypes.byref(cfg), _ptr(ws), _nbytes(ws),
                                                _ptr(out), _stream(stream)))


def forward(cfg, q, k, v, out, ws, stream=None):
    _check_tensors("da2_forward", cfg, (("q", q), ("k", k), ("v", v), ("out", out)), (("ws", ws),),
                   stream=stream)
    _check("da2_forward", lib().da2_forward(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v),
                                            _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)))


def forward_host(cfg, q_host, k_host, v_host, out_host, dq, dk, dv, dout, ws, stream=None):
    """q_host, k_host, v_host, out_host: host tensors (pinned for overlapped copies); dq, dk,
    dv, dout: device staging tensors of the same shape; ws: the device workspace."""
    _check_tensors("da2_forward_host", cfg, (("dq", dq), ("dk", dk), ("dv", dv), ("dout", dout)),
                   (("ws", ws),), (("q_host", q_host), ("k_host", k_host), ("v_host", v_host),
                                   ("out_host", out_host)), stream=stream)
    _check("da2_forward_host", lib().da2_forward_host(
        ctypes.byref(cfg), _ptr(q_host), _ptr(k_host), _ptr(v_host), _ptr(out_host),
        _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dout), _ptr(ws), _nbytes(ws), _stream(stream)))


def forward_noalloc(cfg, q, k, v, out, stream=None):
    """The whole path with the library's built-in 64 MiB device scratch as workspace, for
    callers that cannot allocate device memory (see da2_forward_noalloc in include/da2.h).
    Calls on one device must not overlap on the GPU: they share that scratch. Its device
    error word is read with get_error(cfg, None)."""
    _check_tensors("da2_forward_noalloc", cfg, (("q", q), ("k", k), ("v", v), ("out", out)),
                   stream=stream)
    _check("da2_forward_noalloc", lib().da2_forward_noalloc(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(out), _stream(stream)))


def get_error(cfg, ws, stream=None) -> int:
    """Reads and clears the workspace's device error word (synchronises the stream).
    ws=None reads the word of forward_noalloc's built-in scratch."""
    if ws is not None:
        _check_tensors("da2_get_error", cfg, (), (("ws", ws),), stream=stream)
    word = ctypes.c_uint32()
    st = lib().da2_get_error(_ptr(ws), 0 if ws is None else _nbytes(ws), ctypes.byref(cfg),
                             _stream(stream), ctypes.byref(word))
    if st not in (0, 6):
        raise DA2Error("da2_get_error", st)
    return word.value
