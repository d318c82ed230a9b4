"""Benchmark of the DraftAttention2 hot path (prepare + draft_select + attention) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan720] [--impl ours|reference]

One step = one whole attention call on one synthetic Wan2.1-14B-like 720p layer (B=1,
H=40, d=128, 21x45x80 = 75 600 tokens, 8x16 windows, FP8 10% / FP4 30% / skip 60%),
inputs resident in HBM. Timed with CUDA events on the launching stream, L2 flushed
between steps, max over ranks. Under torchrun every rank runs its own replica (weak
scaling; the path has no exchange step). Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

from sparse_mixed_precision_b200.synth import WORKLOADS, generate  # noqa: E402

METRIC = "dense-equivalent TFLOP/s of one DraftAttention2 attention call (75.6k tokens)"
UNIT = "TFLOP/s"


def kernels_per_step(w) -> int:
    """Library kernels launched by one step: k_prepare_qk, k_prepare_v, the draft selection
    (k_draft_logits_tc + k_draft_rank up to 1024 key blocks, else k_draft_select) and
    k_attention_tc."""
    import math as _m
    N = w.F * _m.ceil(w.Hf / w.ph) * _m.ceil(w.Wf / w.pw)
    return 5 if N <= 1024 else 4


def dense_flops(w) -> float:
    return 4.0 * w.B * w.H * float(w.T) ** 2 * w.d


def executed_flops(w):
    """(FP8, FP4) tensor FLOPs actually executed: kept block pairs x 4 bs^2 d (half of it
    Q K^T, half P V); a mixed block's Q K^T counts as FP8 and its P V as FP4."""
    import math as _m
    ny, nx = _m.ceil(w.Hf / w.ph), _m.ceil(w.Wf / w.pw)
    N = w.F * ny * nx
    bs = w.ph * w.pw
    pm = getattr(w, "pct_mix", 0)
    p4 = w.pct_fp4_max if getattr(w, "adapt_tau", 0.0) > 0 else w.pct_fp4   # the kernel runs the cap
    c8 = (w.pct_fp8 * N + 50) // 100
    c8m = ((w.pct_fp8 + pm) * N + 50) // 100
    ck = ((w.pct_fp8 + pm + p4) * N + 50) // 100
    rows = w.B * w.H * N
    per = 4.0 * bs * bs * w.d
    nm = c8m - c8
    return rows * (c8 + 0.5 * nm) * per, rows * (ck - c8m + 0.5 * nm) * per


def draft_flops(w) -> float:
    """Algorithmic FLOP of the draft maps: two (N x d) @ (d x N) logit products per head."""
    import math as _m
    N = w.F * _m.ceil(w.Hf / w.ph) * _m.ceil(w.Wf / w.pw)
    return 2.0 * 2.0 * N * N * w.d * w.B * w.H


def fp32_fma_peak_tflops(sm_mhz: float, sms: int = 148) -> float:
    """fp32 FMA peak from the unit counts: 128 FMA lanes per SM per clock, 2 FLOP each."""
    return sms * 128 * 2 * sm_mhz * 1e6 / 1e12


def prep_bytes(w) -> float:
    """Algorithmic HBM bytes of the preparation stage (reads once, writes once)."""
    import math as _m
    ny, nx = _m.ceil(w.Hf / w.ph), _m.ceil(w.Wf / w.pw)
    N = w.F * ny * nx
    bs = w.ph * w.pw
    BH = w.B * w.H
    Tp = N * bs
    kv4 = max(bs, 64)
    rd = 3 * BH * w.T * w.d * 2
    wr = BH * Tp * w.d * 3 + BH * Tp * w.d // 2 * 2 + BH * N * w.d * kv4 // 2 \
        + BH * N * (w.d // 64) * 512 * 2 + BH * N * (kv4 // 64) * 512 + 4 * BH * N * w.d * 4
    return float(rd + wr)


ATTN_SOURCES = ("attn_tc.cu", "tc.cuh", "common.cuh")


def attn_source_hash() -> str:
    """sha256 over the attention kernel's sources (the DRAM counters belong to one version)."""
    import hashlib
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "sparse_mixed_precision_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attention_traffic(w):
    """DRAM bytes (read + write) of one attention launch on this workload, from the ncu
    counters stored in profiles/traffic.json, scaled by (batch x heads) from the captured
    case; None when there are none or the kernel sources changed since they were taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    rec = json.load(open(path))
    if rec.get("source_sha256") != attn_source_hash() or rec.get("workload") != w.name:
        return None
    return rec["attention_dram_bytes"] * (w.B * w.H) / rec["captured_bh"]


def draft_bytes(w) -> float:
    """Algorithmic HBM bytes of the draft stage: reads the four pooled fp32 [N, d] arrays
    per head, writes the u8 tags [N, N] and the i16 lists of the kept classes per head."""
    import math as _m
    N = w.F * _m.ceil(w.Hf / w.ph) * _m.ceil(w.Wf / w.pw)
    pm = getattr(w, "pct_mix", 0)
    p4 = w.pct_fp4_max if getattr(w, "adapt_tau", 0.0) > 0 else w.pct_fp4
    c8 = (w.pct_fp8 * N + 50) // 100
    c8m = ((w.pct_fp8 + pm) * N + 50) // 100
    ck = ((w.pct_fp8 + pm + p4) * N + 50) // 100
    kept = max(c8, 1) + max(ck - c8m, 1) + (c8m - c8 if pm > 0 else 0)
    BH = w.B * w.H
    return float(BH * (4 * N * w.d * 4 + N * N + N * kept * 2))


def hbm_entry(bytes_: float, ms: float, peaks: dict) -> dict:
    gbs = bytes_ / (ms * 1e-3) / 1e9
    return {"achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
            "bytes": bytes_}


def tensor_roofline_ms(w, peaks: dict, sustained: bool = False) -> float:
    """Precision-weighted tensor-core time of the executed FP8 and FP4 work: FP8 at 2x and
    FP4 at 4x the measured bf16 rate (NVIDIA's nominal dense ratios 2.25 : 4.5 : 9 PFLOP/s).
    The burst bf16 figure fits a kernel timed alone; the sustained one a long loop at the
    power cap."""
    bf16 = peaks.get("bf16_tflops_sustained" if sustained else "bf16_tflops", peaks.get("bf16_tflops"))
    f8, f4 = executed_flops(w)
    return (f8 / (2.0 * bf16 * 1e12) + f4 / (4.0 * bf16 * 1e12)) * 1e3


def draft_tensor_entry(w, draft_ms: float, peaks: dict) -> dict:
    """The draft stage against the tensor cores that run its logits (up to 1024 key blocks):
    three kind::tf32 products per K step (operands split into tf32 high parts and
    remainders) of the two (N x d) @ (d x N) maps per head, against the tf32 rate taken as
    half the measured burst bf16 rate (NVIDIA's nominal dense 2.25 : 1.1 PFLOP/s). The stage
    also ranks every row (instruction-bound), so the fraction is of the whole stage."""
    tf32 = peaks.get("bf16_tflops", 1590.0) / 2.0
    achieved = 3.0 * draft_flops(w) / (draft_ms * 1e-3) / 1e12
    return {"bound": "tensor", "achieved": achieved, "peak": tf32, "unit": "TFLOP/s",
            "frac": achieved / tf32,
            "note": "3 tf32 MMA products per K step; peak = measured burst bf16 / 2"}


def draft_alu_entry(w, draft_ms: float, peaks: dict) -> dict:
    """The draft stage above 1024 key blocks against its bound: fp32 FMA throughput (the
    logits on the FMA pipe), peak from the unit counts at the measured max SM clock."""
    peak = fp32_fma_peak_tflops(peaks.get("sm_max_mhz", 1965.0))
    achieved = draft_flops(w) / (draft_ms * 1e-3) / 1e12
    return {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "note": "fp32 FMA peak = 148 SMs x 128 lanes x 2 FLOP x SM clock"}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


class ClockSampler:
    """Samples SM clocks and throttle reasons with nvidia-smi during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.lines = index, None, []
        self.t0 = self.t1 = None

    def __enter__(self):
        """Starts sampling every 50 ms and returns once the first sample has arrived, so
        that the samples cover the whole region that follows."""
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            deadline = time.time() + 5.0
            while not self.lines and time.time() < deadline:
                time.sleep(0.01)
        except (OSError, FileNotFoundError):
            self.proc = None
        self.t0 = time.time()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def __exit__(self, *exc):
        self.t1 = time.time()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ts, ln in self.lines:
            if self.t0 is None or not (self.t0 <= ts <= (self.t1 or ts)):
                continue                              # only samples taken in the region
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


def dist_setup(backend: str = "nccl"):
    """One process per GPU under torchrun (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from
    the environment). The path has no exchange step: the process group only serves the
    barriers around the timed region and the max over ranks of the timings. `backend`
    "gloo" runs the same plumbing on CPU (tests)."""
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, ws: int) -> float:
    """The largest of the ranks' values (each rank's device-timed milliseconds)."""
    if ws == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(w, world: int, ms: float) -> float:
    """Whole-job dense-equivalent TFLOP/s: every rank runs one call on its own replica of
    the workload (weak scaling), so world calls complete in the slowest rank's ms."""
    return dense_flops(w) * world / (ms * 1e-3) / 1e12


# ------------------------------------------------------------------------------------------
# CPU oracle timing (reported baseline; also the reference arm)
# ------------------------------------------------------------------------------------------
def oracle_sample(w, q, k, v, n_blocks: int):
    """Times the oracle on one head: the whole preparation and selection, and the
    attention of `n_blocks` query blocks; returns (seconds per call extrapolated to all
    heads and query blocks, description)."""
    import numpy as np
    import oracle as O
    from sparse_mixed_precision_b200.synth import scaled
    wh = scaled(w, B=1, H=1)
    qh, kh, vh = (x[:1, :1].cpu() for x in (q, k, v))
    from threadpoolctl import threadpool_limits
    limiter = threadpool_limits(1)        # the oracle runs on one host thread
    t0 = time.perf_counter()
    P = O.prepare(wh, qh, kh, vh)
    sel = O.draft_select(P)
    t1 = time.perf_counter()
    g = P["g"]
    ops = O.operands_quantised(P["Q"], P["K"], P["V"])
    blocks = [(0, 0, i) for i in np.linspace(0, g.N - 1, n_blocks).astype(int)]
    t2 = time.perf_counter()
    O.attention(ops, P["valid"], sel["list8"], sel["list4"], g.sm_scale, True, blocks=blocks)
    t3 = time.perf_counter()
    limiter.unregister() if hasattr(limiter, "unregister") else limiter.restore_original_limits()
    per_head = (t1 - t0) + (t3 - t2) * g.N / len(blocks)
    sec = per_head * w.B * w.H
    desc = (f"oracle on head (0,0): prepare+select {t1 - t0:.2f} s, attention of {len(blocks)}"
            f" of {g.N} query blocks {t3 - t2:.2f} s; extrapolated x{g.N / len(blocks):.1f}"
            f" blocks and x{w.B * w.H} heads; one host thread (BLAS limited to 1) of"
            f" {os.cpu_count()} on the host")
    return sec, desc


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # pragma: no cover
        return 1


def run_reference(args, w, ws_size, rank):
    if rank != 0:
        return
    gen_dev = "cuda" if torch.cuda.is_available() else "cpu"
    q, k, v = generate(w, device=gen_dev)
    per_step = []
    desc = ""
    for s in range(args.warmup + args.steps):
        sec, desc = oracle_sample(w, q, k, v, args.ref_blocks)
        if s >= args.warmup:
            per_step.append(sec)
    sec = statistics.mean(per_step)
    value = dense_flops(w) / sec / 1e12
    cores = 1
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": sec * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_dict(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def config_dict(w, args):
    return {"workload": f"{w.name}: B={w.B} H={w.H} d={w.d} {w.F}x{w.Hf}x{w.Wf} tokens"
                        f" ({w.T}), window {w.ph}x{w.pw}, FP8 {w.pct_fp8}% / FP4 {w.pct_fp4}%"
                        f" / skip {100 - w.pct_fp8 - w.pct_fp4}%",
            "tokens": w.T, "batch": w.B, "heads": w.H, "head_dim": w.d,
            "l2": "flushed between steps (512 MiB write); inputs 774 MB per tensor",
            "parallelism": f"replicas x{args.gpus}" if args.gpus > 1 else "single GPU"}


def time_stages(da2, w, q, k, v, steps, warmup, dev, flush, clocks=None):
    """Runs `warmup` untimed and `steps` timed calls (prepare, draft_select, attention on one
    stream, L2 flushed before each) and returns the per-stage CUDA-event times (ms lists),
    the workspace and the output of the last call."""
    cfg = da2.config(w)
    ws = torch.empty(da2.workspace_size(cfg), dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        da2.prepare(cfg, q, k, v, ws, stream)
        if ev is not None:
            ev[1].record(stream)
        da2.draft_select(cfg, ws, stream)
        if ev is not None:
            ev[2].record(stream)
        da2.attention(cfg, ws, out, stream)
        if ev is not None:
            ev[3].record(stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert da2.get_error(cfg, ws) == 0
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.__enter__()
    for s_ in range(steps):
        flush.zero_()
        step(events[s_])
    torch.cuda.synchronize()
    if clocks is not None:
        clocks.__exit__(None, None, None)
    assert da2.get_error(cfg, ws) == 0
    stage = {"prepare": [], "draft_select": [], "attention": [], "total": []}
    for ev in events:
        stage["prepare"].append(ev[0].elapsed_time(ev[1]))
        stage["draft_select"].append(ev[1].elapsed_time(ev[2]))
        stage["attention"].append(ev[2].elapsed_time(ev[3]))
        stage["total"].append(ev[0].elapsed_time(ev[3]))
    return stage, cfg, ws, out


def dense_rel_l2(q, k, v, out, heads, rows=4096, seed=0):
    """Relative L2 error of the call's output against dense fp32 softmax attention (torch
    on the GPU, a reference computation), on `rows` seeded query rows of each listed head."""
    g = torch.Generator().manual_seed(seed)
    res = {}
    for b, h in heads:
        r = torch.randperm(q.shape[2], generator=g)[:rows].to(q.device)
        S = (q[b, h, r].float() @ k[b, h].float().T) / math.sqrt(q.shape[-1])
        ref = torch.softmax(S, -1) @ v[b, h].float()
        got = out[b, h, r].float()
        res[f"b{b}h{h}"] = ((got - ref).norm() / ref.norm()).item()
    return res


def workload_entry(w, stage, peaks):
    """ms, dense-equivalent TFLOP/s and roofline fractions of one workload's call."""
    ms = statistics.mean(stage["total"])
    attn = statistics.mean(stage["attention"])
    t8 = tensor_roofline_ms(w, peaks)
    return {"ms": ms, "tflops": dense_flops(w) / (ms * 1e-3) / 1e12,
            "stages_ms": {k_: statistics.mean(v_) for k_, v_ in stage.items() if k_ != "total"},
            "attention_frac": t8 / attn, "t_roof_attention_ms": t8,
            "prepare_hbm_frac": prep_bytes(w) / (statistics.mean(stage["prepare"]) * 1e-3) / 1e9 / peaks["hbm_gbs"],
            "draft_hbm_frac": draft_bytes(w) / (statistics.mean(stage["draft_select"]) * 1e-3) / 1e9 / peaks["hbm_gbs"]}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="wan720", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-blocks", type=int, default=8)
    ap.add_argument("--heads", type=int, default=0,
                    help="override the head count (small cases for profiling)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the per-workload lines (the other configurations)")
    args = ap.parse_args()
    w = WORKLOADS[args.workload]
    if args.heads > 0:
        from sparse_mixed_precision_b200.synth import scaled
        w = scaled(w, H=args.heads)
    world, rank, local = dist_setup()

    if args.impl == "reference":
        run_reference(args, w, None, rank)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return

    import sparse_mixed_precision_b200 as da2
    dev = torch.device("cuda", local)
    q, k, v = generate(w, device=dev, seed=w.seed + rank)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    barrier(world)
    clk = ClockSampler(local)
    stage, cfg, ws, out = time_stages(da2, w, q, k, v, args.steps, args.warmup, dev, flush, clocks=clk)
    barrier(world)
    ms_local = statistics.mean(stage["total"])
    ms = max_over_ranks(ms_local, world)
    value = job_throughput(w, world, ms)

    # roofline of the dominant kernel (attention): precision-weighted tensor bound, against
    # the burst bf16 figure (the kernel is timed alone, one call at a time) and, beside it,
    # the sustained one
    peaks, src = load_peaks()
    f8, f4 = executed_flops(w)
    attn_ms = statistics.mean(stage["attention"])
    t_roof = tensor_roofline_ms(w, peaks)
    t_roof_sus = tensor_roofline_ms(w, peaks, sustained=True)
    achieved = (f8 + f4) / (attn_ms * 1e-3) / 1e12
    peak_eff = (f8 + f4) / (t_roof * 1e-3) / 1e12
    prep_ms = statistics.mean(stage["prepare"])
    draft_ms = statistics.mean(stage["draft_select"])
    pb, db = prep_bytes(w), draft_bytes(w)
    traffic = attention_traffic(w)
    bf16 = peaks.get("bf16_tflops")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3/e2m1 MMA, f32 accumulate", "data": "synthetic (seeded smooth field + noise + sinks)",
        "config": config_dict(w, args),
        "stages_ms": {k_: statistics.mean(v_) for k_, v_ in stage.items() if k_ != "total"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_eff, "unit": "TFLOP/s",
                     "frac": t_roof / attn_ms, "traffic": traffic,
                     "frac_sustained_peak": t_roof_sus / attn_ms,
                     "note": f"attention kernel; peak = precision-weighted ({f8:.3e} FP8 + {f4:.3e} FP4 FLOP"
                             f" at {2 * bf16:.0f} / {4 * bf16:.0f} TFLOP/s = 2x / 4x the {src} burst bf16"
                             f" cuBLAS rate, t_roof {t_roof:.2f} ms; frac_sustained_peak uses the"
                             f" sustained bf16 rate, t_roof {t_roof_sus:.2f} ms)"},
        "prepare_hbm": hbm_entry(pb, prep_ms, peaks),
        "draft_hbm": hbm_entry(db, draft_ms, peaks),
        ("draft_tensor" if kernels_per_step(w) == 5 else "draft_alu"):
            (draft_tensor_entry if kernels_per_step(w) == 5 else draft_alu_entry)(w, draft_ms, peaks),
        "step_roofline_frac": (t_roof + (pb + db) / (peaks["hbm_gbs"] * 1e9) * 1e3) / ms,
        "gpu_launches": kernels_per_step(w) * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and args.heads == 0:
        line["dense_rel_l2"] = dense_rel_l2(q, k, v, out, [(0, 0), (w.B - 1, w.H - 1)])

    # end to end through the C ABI with host buffers (pinned), copies inside the timed region
    if not args.no_e2e:
        qh, kh, vh = (x.cpu().pin_memory() for x in (q, k, v))
        oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        da2.forward_host(cfg, qh, kh, vh, oh, q, k, v, out, ws, stream)
        barrier(world)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(2, min(args.steps, 5))
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(n_e2e):
            da2.forward_host(cfg, qh, kh, vh, oh, q, k, v, out, ws, stream)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / n_e2e, world)
        nbytes = q.numel() * q.element_size()
        line["e2e"] = {"value": job_throughput(w, world, e2e_ms), "unit": UNIT,
                       "ms_per_step": e2e_ms, "h2d_bytes_per_step": 3 * nbytes,
                       "d2h_bytes_per_step": nbytes}
        del qh, kh, vh, oh

    # the other configurations: per-workload ms, TFLOP/s and roofline fractions (the
    # headline value above stays on the 720p layer); rank 0 of a single-GPU run only
    if rank == 0 and world == 1 and not args.no_workloads and args.heads == 0:
        del ws, out
        others = {}
        for name in ("wan480", "hunyuan720", "sweep0", "sweep1", "sweep2", "sweep3", "sweep4", "wan720mix",
                     "wan720adapt"):
            if name == w.name:
                continue
            wo = WORKLOADS[name]
            qo, ko, vo = generate(wo, device=dev)
            st, _, wso, oo = time_stages(da2, wo, qo, ko, vo, 5, 3, dev, flush)
            others[name] = workload_entry(wo, st, peaks)
            del qo, ko, vo, wso, oo
            torch.cuda.empty_cache()
        line["workloads"] = others

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sec, desc = oracle_sample(w, q, k, v, args.ref_blocks)
        line["cpu_baseline"] = {"value": dense_flops(w) / sec / 1e12, "unit": UNIT,
                                "cores": 1, "kind": "oracle", "sample": desc,
                                "ms_per_call": sec * 1e3}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
