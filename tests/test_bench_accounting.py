"""The bench's algorithmic byte and flop counts (the roofline numerators) against the figures worked
out by hand for the workloads: touched experts' weights once, router, x read once, out written once
(CPU only)."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402
import workloads  # noqa: E402


def _counts(E, touched, rows=1):
    c = np.zeros(E, dtype=np.int64)
    c[:touched] = rows
    return c


def test_decode_f32_t1_layer_bytes():
    # 8 experts x 3 x 704 x 2816 f32 weights (23.79 MB each) + the 128 x 2816 f32 router + x and out
    s = workloads.CONFIGS["decode_f32_t1"]
    _, layer, touched = bench.algorithmic(s, _counts(s.E, 8))
    assert touched == 8
    expert = 3 * 704 * 2816 * 4
    assert expert == 23_789_568
    assert layer["bytes"] == 8 * expert + 128 * 2816 * 4 + 2 * 2816 * 4
    assert layer["bytes"] == pytest.approx(191.8e6, rel=1e-3)
    assert layer["flops"] == 2.0 * (128 * 2816 + 8 * 3 * 2816 * 704)


def test_prefill_layer_bytes_and_flops():
    # 64 experts x 12.58 MB of bf16 weights + router + x + out = 809.7 MB; 51.67 GFLOP
    s = workloads.CONFIGS["prefill_bf16_t512"]
    k, layer, touched = bench.algorithmic(s, _counts(s.E, 64, rows=64))
    assert touched == 64
    assert layer["bytes"] == 64 * 3 * 1024 * 2048 * 2 + 64 * 2048 * 2 + 2 * 512 * 2048 * 2
    assert layer["bytes"] == pytest.approx(809.7e6, rel=1e-3)
    assert layer["flops"] == pytest.approx(51.67e9, rel=1e-3)
    # the gate/up GEMM: both weight stacks once, gathered rows in, bf16 h out
    P = 512 * 8
    assert k["expert_gate_up_gemm"]["bytes"] == 64 * 2 * 1024 * 2048 * 2 + P * 2048 * 2 + P * 1024 * 2
    assert k["expert_gate_up_gemm"]["flops"] == 2.0 * P * 2 * 1024 * 2048


def test_untouched_experts_cost_nothing():
    s = workloads.CONFIGS["q8_0_decode_t16"]
    _, a, _ = bench.algorithmic(s, _counts(s.E, 80))
    _, b, _ = bench.algorithmic(s, _counts(s.E, 81))
    per_expert = 3 * s.I * s.H * (1 + 2.0 / 32)  # Q8_0: one byte per code plus an fp16 scale per 32
    assert b["bytes"] - a["bytes"] == pytest.approx(per_expert)


def test_kquant_bytes_per_weight():
    s = workloads.CONFIGS["q4k_q6k_decode_t16"]
    _, a, _ = bench.algorithmic(s, _counts(s.E, 10))
    _, b, _ = bench.algorithmic(s, _counts(s.E, 11))
    # Q4_K: 144 bytes per 256 weights (gate, up); Q6_K: 210 bytes per 256 (down)
    assert b["bytes"] - a["bytes"] == pytest.approx((2 * 144 + 210) / 256 * s.I * s.H)


def test_kernel_roofline_fractions():
    peaks = {"hbm_gbs": 6500.0, "bf16_tflops": 1600.0, "bf16_tflops_sustained": 1400.0}
    # 1 TFLOP over 1 GB in 1 ms: 1000 TFLOP/s, far above the ridge -> tensor bound
    r = bench.kernel_roofline({"flops": 1e12, "bytes": 1e9}, 1.0, peaks, "measured")
    assert r["bound"] == "tensor" and r["achieved"] == pytest.approx(1000.0)
    assert r["frac"] == pytest.approx(1000 / 1400) and r["frac_burst"] == pytest.approx(1000 / 1600)
    assert r["frac_nominal"] == pytest.approx(1000 / 2250)
    # 1 GB and 1 GFLOP in 0.5 ms: 2000 GB/s -> HBM bound
    r = bench.kernel_roofline({"flops": 1e9, "bytes": 1e9}, 0.5, peaks, "measured")
    assert r["bound"] == "hbm" and r["achieved"] == pytest.approx(2000.0)
    assert r["frac"] == pytest.approx(2000 / 6500) and r["frac_nominal"] == pytest.approx(0.25)


def test_expert_load_summary():
    a = np.array([0, 5, 1, 0, 9])
    b = np.array([2, 2, 2, 2, 0])
    d = bench.expert_load([a, b])
    assert d["touched_mean"] == 3.5 and d["max_rows"] == 9 and d["min_nonzero_rows"] == 1
    assert d["max_rows_mean"] == 5.5 and d["min_nonzero_rows_mean"] == 1.5
    assert d["batch0_rows_desc"] == [9, 5, 1]
