"""bench.py's work counts and bounds (host arithmetic only)."""
import pytest

import bench
from sparse_mixed_precision_b200.synth import WORKLOADS


def test_work_counts_of_the_wan720_call():
    w = WORKLOADS["wan720"]
    assert bench.dense_flops(w) == pytest.approx(1.1705e14, rel=1e-3)      # 4 B H T^2 d
    f8, f4 = bench.executed_flops(w)
    assert (f8, f4) == (pytest.approx(1.332e13, rel=1e-3), pytest.approx(3.995e13, rel=1e-3))
    assert bench.prep_bytes(w) == pytest.approx(4.31e9, rel=1e-2)
    assert bench.draft_flops(w) == pytest.approx(2 * 2 * 630 ** 2 * 128 * 40)


def test_draft_alu_bound():
    w = WORKLOADS["wan720"]
    assert bench.fp32_fma_peak_tflops(1965.0) == pytest.approx(148 * 128 * 2 * 1.965e9 / 1e12)
    e = bench.draft_alu_entry(w, 1.0, {"sm_max_mhz": 1965.0})
    assert e["bound"] == "alu" and e["frac"] == pytest.approx(e["achieved"] / e["peak"])
    assert e["achieved"] == pytest.approx(bench.draft_flops(w) / 1e-3 / 1e12)


def test_draft_bytes_and_tensor_roofline():
    w = WORKLOADS["wan720"]
    # pooled fp32 [N, d] x 4 read, u8 tags [N, N] and i16 lists [N, 63 + 189] written, 40 heads
    assert bench.draft_bytes(w) == pytest.approx(40 * (4 * 630 * 128 * 4 + 630 * 630 + 630 * 252 * 2))
    peaks = {"bf16_tflops": 1655.5, "bf16_tflops_sustained": 1405.2}
    f8, f4 = bench.executed_flops(w)
    assert bench.tensor_roofline_ms(w, peaks) == pytest.approx(
        (f8 / 3311e12 + f4 / 6622e12) * 1e3)                      # 10.06 ms at the burst rate
    assert bench.tensor_roofline_ms(w, peaks) == pytest.approx(10.06, rel=2e-3)
    assert bench.tensor_roofline_ms(w, peaks, sustained=True) > bench.tensor_roofline_ms(w, peaks)


def test_draft_tensor_bound_and_launch_count():
    w = WORKLOADS["wan720"]
    e = bench.draft_tensor_entry(w, 1.0, {"bf16_tflops": 1655.5})
    assert e["bound"] == "tensor" and e["peak"] == pytest.approx(1655.5 / 2)
    assert e["achieved"] == pytest.approx(3 * bench.draft_flops(w) / 1e-3 / 1e12)
    assert bench.kernels_per_step(w) == 5                     # N = 630: two draft kernels
    from sparse_mixed_precision_b200.synth import scaled
    assert bench.kernels_per_step(scaled(WORKLOADS["wan480"], ph=4, pw=8)) == 4   # N = 1176
