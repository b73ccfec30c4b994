"""Failure detection without a GPU fault: a bounded pipeline wait runs out and is reported.

A debug switch makes the TMA producer of CTA 0 leave one shared-memory stage
unfilled, so the MMA issuer's wait on that stage can never complete.  With a
short wait limit (about 10 ms of SM cycles) every role of that CTA gives up,
lets its in-flight copies land, frees its tensor memory and exits; the host
reads MOE_ERR_TIMEOUT from the status word.  The same context then computes a
correct layer, which shows nothing was left hung.
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
