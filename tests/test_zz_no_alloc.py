"""moe_layer_noalloc: the layer for callers that cannot allocate device memory.

Such a caller (a host whose HBM already belongs to its own pool, code that may
not take cudaMalloc's implicit synchronisation, a plain C caller without an
allocator) gets the same layer with the scratch held in a static 32 MiB device
array inside libmoe.  This file is collected last so that, if it fails, a run
that stops at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
from mixture_experts_ffn_07_b200 import _lib  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402


def _noalloc(desc, x, w, out):
    d, cw = desc.c(), w.c()
    return _lib.lib().moe_layer_noalloc(ctypes.byref(d), x.data_ptr(), ctypes.byref(cw), out.data_ptr(),
                                        torch.cuda.current_stream().cuda_stream)


@pytest.mark.parametrize("spec", [
    workloads.Spec(T=200, H=256, E=16, I=128, K=4, shared_I=64, shared_gated=True, name="noalloc_tensor"),
    # E % 32 == 0 and T > 64: the tensor-core router with split-K partials and the fused selection / permutation
    # / gather kernel, whose partial-logit and count regions of the static scratch then hold the first call's data
    workloads.Spec(T=200, H=256, E=32, I=128, K=4, shared_I=64, shared_gated=True, name="noalloc_tensor_front"),
    workloads.Spec(T=16, H=2048, E=128, I=768, K=8, act_dtype="f32", w_dtype="q8_0", router_dtype="f32",
                   name="noalloc_q8_decode"),
], ids=lambda s: s.name)
def test_noalloc_matches_moe_layer_on_two_calls(spec):
    wl = workloads.make(spec, seed=41)
    desc, w, x1 = _gpu.upload(wl)
    assert moe.workspace_bytes(desc) <= _lib.MOE_NOALLOC_SCRATCH_BYTES
    # a second, different input so the second call runs over the first call's leftovers
    x2 = torch.flip(x1, dims=[0]).contiguous() * 0.5
    for x in (x1, x2):
        ref = _gpu.run_layer(desc, w, x)
        out = torch.full_like(ref, float("nan"))
        assert _noalloc(desc, x, w, out) == moe.MOE_OK
        torch.cuda.synchronize()
        assert moe.last_device_status() == moe.MOE_OK
        r, o = _gpu.to_np(ref), _gpu.to_np(out)
        assert np.all(np.isfinite(o))
        assert float(np.max(np.abs(o - r))) <= _gpu.tolerance(r, spec.act_dtype)


def test_noalloc_rejects_descriptors_beyond_the_static_scratch():
    desc = moe.Desc(T=4096, H=2048, E=256, I=512, top_k=8)
    assert moe.workspace_bytes(desc) > _lib.MOE_NOALLOC_SCRATCH_BYTES
    d, w = desc.c(), moe.Weights().c()
    n0 = moe.launch_count()
    rc = _lib.lib().moe_layer_noalloc(ctypes.byref(d), None, ctypes.byref(w), None, None)
    assert rc == moe.MOE_ERR_WORKSPACE
    assert moe.launch_count() == n0
