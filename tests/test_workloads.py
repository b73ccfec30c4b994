"""The seeded input generator: determinism, independence of streams, distributions (CPU only)."""
import numpy as np

import workloads
from tests._helpers import widen


def test_deterministic_and_counter_based():
    a = workloads.normal(1, 3, (1000,), 1.0, "f32")
    b = workloads.normal(1, 3, (1000,), 1.0, "f32")
    assert np.array_equal(a, b)
    # element i does not depend on how many elements are drawn
    c = workloads.normal(1, 3, (10,), 1.0, "f32")
    assert np.array_equal(a[:10], c)
    assert not np.array_equal(a, workloads.normal(1, 4, (1000,), 1.0, "f32"))
    assert not np.array_equal(a, workloads.normal(2, 3, (1000,), 1.0, "f32"))


def test_normal_moments():
    a = workloads.normal(9, 1, (400000,), 0.02, "f32").astype(np.float64)
    assert abs(a.mean()) < 0.02 * 0.01 and abs(a.std() / 0.02 - 1) < 0.01


def test_bf16_is_rne_of_f32_sample():
    f = workloads.normal(5, 7, (4096,), 3.0, "f32")
    b = workloads.normal(5, 7, (4096,), 3.0, "bf16")
    assert np.array_equal(b, workloads.f32_to_bf16(f))
    # round to nearest: |bf16 - f32| <= half an ulp of bf16 (2^-8 relative)
    assert np.all(np.abs(widen(b, "bf16") - f) <= np.abs(f) * 2.0 ** -8 + 1e-30)


def test_q8_0_blocks_ranges():
    blk = workloads.q8_0_blocks(3, 2, (2, 8, 64))
    assert blk.shape == (2, 8, 2, 34)
    d = blk[..., :2].copy().view(np.float16).astype(np.float64)
    q = blk[..., 2:].copy().view(np.int8)
    assert d.min() >= 0.001 * (1 - 2 ** -11) and d.max() <= 0.01 * (1 + 2 ** -11)
    assert q.min() >= -127 and q.max() <= 127
    assert len(np.unique(q)) > 200


def test_zipf_bias():
    b = workloads.zipf_log_bias(256).astype(np.float64)
    r = np.arange(1, 257.0)
    p = r ** -1.1 / np.sum(r ** -1.1)
    assert np.allclose(b, 2 * np.log(p), rtol=1e-6)
    assert np.all(np.diff(b) < 0)


def test_configs_shapes():
    s = workloads.CONFIGS["prefill_bf16_t512"]
    assert (s.T, s.H, s.E, s.I, s.K) == (512, 2048, 64, 1024, 8)
    wl = workloads.make(workloads.Spec(T=3, H=64, E=4, I=32, K=2, shared_I=32, shared_gated=True), seed=1)
    assert wl.x.shape == (3, 64) and wl.x.dtype == np.uint16
    assert wl.gate.shape == (4, 32, 64) and wl.down.shape == (4, 64, 32)
    assert wl.sh_gate.shape == (32, 64) and wl.sh_down.shape == (64, 32) and wl.sh_gate_w.shape == (64,)


def test_token_batches():
    spec = workloads.Spec(T=3, H=64, E=4, I=32, K=2)
    wl = workloads.make(spec, seed=5)
    assert np.array_equal(workloads.token_batch(spec, 0, seed=5), wl.x)  # batch 0 is the workload's own x
    b1, b2 = workloads.token_batch(spec, 1, seed=5), workloads.token_batch(spec, 2, seed=5)
    assert b1.shape == wl.x.shape and b1.dtype == wl.x.dtype
    assert not np.array_equal(b1, wl.x) and not np.array_equal(b1, b2)
    assert np.array_equal(b1, workloads.token_batch(spec, 1, seed=5))
    # no further batch shares a stream with the weights
    assert not np.array_equal(workloads.token_batch(spec, 1, seed=5).reshape(-1)[:16],
                              wl.gate.reshape(-1)[:16])
