"""Failure detection without a GPU fault: bounded waits run out and are reported.

A debug switch makes the TMA producer of CTA 0 leave one shared-memory stage
unfilled, so the MMA issuer's wait on that stage can never complete.  With a
short wait limit (about 10 ms of SM cycles) every role of that CTA gives up,
lets its in-flight copies land, frees its tensor memory and exits; the host
reads MOE_ERR_TIMEOUT from the status word.  The same context then computes a
correct layer, which shows nothing was left hung.  The grid barriers of the
two cooperative kernels are tested the same way with a late arrival of CTA 0.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402


def test_wait_timeout_is_reported_and_context_survives():
    s = workloads.Spec(T=200, H=256, E=16, I=128, K=4, name="timeout_case")
    wl = workloads.make(s, seed=3)
    desc, w, x = _gpu.upload(wl)
    assert moe.last_device_status() == moe.MOE_OK
    out = torch.empty((s.T, s.H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    try:
        moe.debug_set_wait_limit(20_000_000)
        moe.debug_set_skip_stage(True)
        moe.layer(desc, x, w, out, ws)
        assert moe.last_device_status() == moe.MOE_ERR_TIMEOUT
    finally:
        moe.debug_set_skip_stage(False)
        moe.debug_set_wait_limit(0)
    assert moe.last_device_status() == moe.MOE_OK
    out = _gpu.run_layer(desc, w, x)
    _, gids, _, _ = _gpu.run_route(desc, w, x)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out), exp, "bf16", "after timeout")


def _late_barrier_then_normal(s, act_dtype):
    """CTA 0 of the cooperative kernel arrives late at its first grid barrier: the other CTAs' bounded waits
    run out and MOE_ERR_TIMEOUT is reported; CTA 0 still arrives, so later launches on the same barrier counter
    compute correct layers."""
    wl = workloads.make(s, seed=5)
    desc, w, x = _gpu.upload(wl)
    assert moe.last_device_status() == moe.MOE_OK
    out = torch.empty((s.T, s.H), dtype=x.dtype, device="cuda")
    ws = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    try:
        moe.debug_set_wait_limit(20_000_000)       # about 10 ms of SM cycles
        moe.debug_set_barrier_delay(80_000_000)    # CTA 0 arrives about 40 ms late
        moe.layer(desc, x, w, out, ws)
        assert moe.last_device_status() == moe.MOE_ERR_TIMEOUT
    finally:
        moe.debug_set_barrier_delay(0)
        moe.debug_set_wait_limit(0)
    assert moe.last_device_status() == moe.MOE_OK
    _, gids, _, _ = _gpu.run_route(desc, w, x)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    for _ in range(3):
        out = _gpu.run_layer(desc, w, x)
        _gpu.assert_close(_gpu.to_np(out), exp, act_dtype, "after a late barrier")


def test_front_barrier_timeout_is_reported_and_counter_survives():
    # bf16, T > 64, E % 32 == 0: the tensor-core router and the cooperative prefill front
    _late_barrier_then_normal(workloads.Spec(T=200, H=512, E=64, I=64, K=8, name="front_timeout"), "bf16")


def test_decode_barrier_timeout_is_reported_and_counter_survives():
    # f32, T <= 64: the whole layer as the cooperative decode kernel
    _late_barrier_then_normal(workloads.Spec(T=4, H=256, E=16, I=64, K=2, act_dtype="f32", w_dtype="f32",
                                             router_dtype="f32", name="decode_timeout"), "f32")
