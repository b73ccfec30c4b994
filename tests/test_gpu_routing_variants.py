"""Routing variants (sigmoid gating, group-limited selection) on every router
path: the cluster router (small batches), the tensor-core router + top-K, the
fused decode kernel and the fused prefill front.  Selection is compared bit
for bit with the oracle fed the GPU's own f32 logits; weights to f32
rounding; layer outputs within the usual tolerances."""
import dataclasses

import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
from tests import _gpu  # noqa: E402
from tests.test_gpu_parity import make, spec  # noqa: E402


def vspec(base, gating="softmax", n_groups=1, topk_groups=1):
    return dataclasses.replace(base, gating=gating, n_groups=n_groups, topk_groups=topk_groups)


CASES = {
    # (spec, bias?)
    "cluster_f32_sigmoid": (vspec(spec(9, 256, 32, 64, 4, dt="f32"), "sigmoid"), False),
    "cluster_f32_sigmoid_no_renorm": (vspec(spec(9, 256, 32, 64, 4, dt="f32", renorm=False), "sigmoid"), True),
    "cluster_bf16_grouped": (vspec(spec(40, 512, 64, 64, 6), "softmax", 8, 3), False),
    "cluster_f32_grouped_sigmoid_bias": (vspec(spec(16, 256, 64, 64, 8, dt="f32"), "sigmoid", 8, 4), True),
    "tensor_grouped_sigmoid": (vspec(spec(300, 512, 64, 64, 8), "sigmoid", 8, 4), False),
    "tensor_grouped_softmax_no_renorm_bias": (vspec(spec(200, 256, 256, 64, 8, renorm=False), "softmax", 32, 4), True),
    "tensor_sigmoid_E256": (vspec(spec(150, 256, 256, 64, 8), "sigmoid"), False),
    "groups_of_one_expert": (vspec(spec(100, 256, 32, 64, 4), "softmax", 32, 5), False),
}


def _wl(s, bias, seed):
    return make(s, seed=seed, bias_values=(np.linspace(-2, 2, s.E)[::-1] if bias else None))


@pytest.mark.parametrize("case", sorted(CASES))
def test_route_variants(case):
    s, bias = CASES[case]
    wl = _wl(s, bias, 61)
    desc, w, x = _gpu.upload(wl)
    logits, ids, tw, _ = _gpu.run_route(desc, w, x)
    gl = logits.cpu().numpy().astype(np.float64)
    ref_ids, ref_w = oracle.select(gl, s.K, s.renormalize, gating=s.gating, n_groups=s.n_groups,
                                   topk_groups=s.topk_groups)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) < 2e-6
    if s.n_groups > 1:  # every chosen expert sits in one of the kept groups
        gs = s.E // s.n_groups
        assert np.all(np.array([len(set(r // gs)) for r in ids.cpu().numpy()]) <= s.topk_groups)


@pytest.mark.parametrize("case", sorted(CASES))
def test_layer_variants(case):
    s, bias = CASES[case]
    wl = _wl(s, bias, 67)
    desc, w, x = _gpu.upload(wl)
    out = _gpu.run_layer(desc, w, x)
    _, gids, _, _ = _gpu.run_route(desc, w, x)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out), exp, s.act_dtype, case)


def test_grouped_sigmoid_workload_routing():
    """The measurement workload (T=512, E=64 in 8 groups, 4 kept, sigmoid) at full size."""
    import workloads
    s = workloads.CONFIGS["grouped_sigmoid_t512"]
    wl = workloads.make(s, seed=workloads.BASE_SEED + workloads.CONFIG_ORDER.index(s.name))
    desc, w, x = _gpu.upload(wl)
    logits, ids, tw, _ = _gpu.run_route(desc, w, x)
    ref_ids, ref_w = oracle.select(logits.cpu().numpy().astype(np.float64), s.K, s.renormalize, gating="sigmoid",
                                   n_groups=8, topk_groups=4)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) < 2e-6
    out = _gpu.run_layer(desc, w, x)
    tok = np.arange(0, s.T, 37)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), ids.cpu().numpy(), tokens=tok)
    _gpu.assert_close(_gpu.to_np(out)[tok], exp, s.act_dtype, "grouped_sigmoid_t512 sampled")
