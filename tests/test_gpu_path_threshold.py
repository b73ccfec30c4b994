"""Both paths of a bf16 layer on either side of a token threshold (moe_set_tensor_min_tokens):
the tensor-core path on 16..64 tokens and the weight-streaming path on more than 64, each against the oracle,
so the threshold can be set anywhere the measured crossover puts it."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402


@pytest.mark.parametrize("T,threshold", [(16, 1), (48, 1), (64, 1), (100, 1000), (160, 1000)])
def test_layer_on_either_path(T, threshold):
    s = workloads.Spec(T=T, H=512, E=32, I=256, K=8, shared_I=128, shared_gated=True, name=f"thr_{T}")
    wl = workloads.make(s, seed=53)
    moe.set_tensor_min_tokens(threshold)
    try:
        desc, w, x = _gpu.upload(wl)
        out = _gpu.run_layer(desc, w, x)
        logits, ids, _, _ = _gpu.run_route(desc, w, x)
        n0 = moe.launch_count()
        _gpu.run_layer(desc, w, x)
        launches = moe.launch_count() - n0
    finally:
        moe.set_tensor_min_tokens(_gpu.DEFAULT_TENSOR_MIN_TOKENS)
    assert moe.last_device_status() == moe.MOE_OK
    L = oracle.from_workload(wl)
    exp, flagged = _gpu.expected_layer(L, ids.cpu().numpy(), gpu_logits=logits.cpu().numpy().astype(np.float64))
    _gpu.assert_close(_gpu.to_np(out), exp, "bf16", f"T={T}")
    # the fused decode layer (streaming path, at most 64 tokens) is one launch; the other forms take several
    assert (launches == 1) == (threshold > T and T <= 64)
