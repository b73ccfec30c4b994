"""The fused decode kernel (the whole layer as one cooperative launch for
1..64 tokens on the weight-streaming path) against the step-by-step launches,
moe_route and the oracle.

Routing has one correct answer for tie-free logits and the fused kernel adds
the router's chunk partials in the same order as the router kernels, so its
logits, ids, weights and permutation must equal the step-by-step path's bit
for bit.  The expert outputs may differ in rounding (the fused kernel plans
its K ranges for a different shared-memory budget), so `out` is compared with
the oracle within the f32 / bf16 tolerances.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
from tests import _gpu  # noqa: E402
from tests.test_gpu_parity import make, spec  # noqa: E402

CASES = {
    "f32_gelu_T1": (spec(1, 256, 16, 96, 4, act="gelu_tanh", dt="f32"), {}),
    "f32_T64_shared_gated_bias": (spec(64, 512, 32, 128, 8, dt="f32", shared=64, gated=True), dict(bias=True)),
    "q8_T16_shared_gated": (spec(16, 256, 32, 128, 8, dt="f32", w_dt="q8_0", r_dt="f32", shared=64, gated=True), {}),
    "q8_T3_ungated_shared_bf16_router": (spec(3, 512, 16, 64, 2, dt="f32", w_dt="q8_0", r_dt="bf16", shared=32), {}),
    "bf16_T40": (spec(40, 256, 32, 128, 8), {}),
    "bf16_T64_no_renorm": (spec(64, 384, 64, 64, 6, renorm=False), {}),
    "f32x_bf16w_T3": (spec(3, 384, 8, 64, 2, dt="f32", w_dt="bf16", r_dt="f32"), {}),
    "K_equals_E": (spec(5, 128, 4, 64, 4, dt="f32"), {}),
    "long_rows_split_K": (spec(6, 4096, 8, 64, 2, dt="f32", shared=32), {}),
    "max_pairs_E256_K32": (spec(64, 128, 256, 32, 32, dt="f32"), {}),
    "skew_all_to_two": (spec(48, 256, 8, 64, 2, dt="f32"), dict(skew=True)),
    # one token: the CTA-wide ranking; logits = bias exactly (zero router), five values over 64 experts
    "T1_tied_logits": (spec(1, 256, 64, 64, 8, dt="f32"), dict(ties=True)),
    "T1_tied_logits_no_renorm_E256": (spec(1, 256, 256, 32, 8, dt="f32", renorm=False), dict(ties=True)),
}


def _workload(s, opt, seed):
    bias = None
    if opt.get("bias"):
        bias = np.linspace(2, -2, s.E)
    if opt.get("skew"):
        bias = np.array([50.0, 40.0] + [0.0] * (s.E - 2))
    if opt.get("ties"):
        return make(s, seed=seed, bias_values=[float((e * 7) % 5) for e in range(s.E)], router_std=0.0)
    return make(s, seed=seed, bias_values=bias)


def _run(desc, w, x, fused):
    moe.set_fused_decode(fused)
    try:
        out = torch.empty((desc.T, desc.H), dtype=x.dtype, device="cuda")
        ws = torch.zeros(max(moe.workspace_bytes(desc), 256), dtype=torch.uint8, device="cuda")
        n0 = moe.launch_count()
        moe.layer(desc, x, w, out, ws)
        torch.cuda.synchronize()
        launches = moe.launch_count() - n0
        assert moe.last_device_status() == moe.MOE_OK
    finally:
        moe.set_fused_decode(True)
    reg = moe.workspace_regions(desc)
    T, E, K = desc.T, desc.E, desc.top_k
    P = T * K

    def view(name, n, dtype):
        off = reg[name]
        return ws[off:off + 4 * n].view(dtype).clone()

    routing = {
        "logits": view("logits", T * E, torch.float32),
        "topk_ids": view("topk_ids", P, torch.int32),
        "topk_w": view("topk_w", P, torch.float32),
        "counts": view("counts", E, torch.int32),
        "offsets": view("offsets", E + 1, torch.int32),
        "sorted_pairs": view("sorted_pairs", P, torch.int32),
        "pair_pos": view("pair_pos", P, torch.int32),
    }
    if desc.shared_I and desc.has_shared_gate:
        routing["shared_gate"] = view("shared_gate", T, torch.float32)
    return out, routing, launches


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.fixture(autouse=True)
def _bf16_on_the_streaming_path():
    with _gpu.streaming_path():  # the bf16 cases are decode batches on the streaming path
        yield


@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_matches_steps_and_oracle(case):
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=41)
    desc, w, x = _gpu.upload(wl)
    out_f, rt_f, n_f = _run(desc, w, x, True)
    out_s, rt_s, n_s = _run(desc, w, x, False)
    assert n_f == 1, "the fused path is one launch"
    assert n_s >= 4
    for k in rt_s:
        assert torch.equal(_bits(rt_f[k]), _bits(rt_s[k])), f"{case}: {k} differs between fused and step paths"
    # the same routing as moe_route
    logits, gids, gw, _ = _gpu.run_route(desc, w, x)
    assert torch.equal(_bits(rt_f["topk_ids"]), _bits(gids.reshape(-1)))
    assert torch.equal(_bits(rt_f["logits"]), _bits(logits.reshape(-1)))
    assert torch.equal(_bits(rt_f["topk_w"]), _bits(gw.reshape(-1)))
    if opt.get("ties"):  # logits equal the bias: the K largest, the lower expert first among equal values
        b = np.array([float((e * 7) % 5) for e in range(s.E)])
        want = sorted(range(s.E), key=lambda e: (-b[e], e))[: s.K]
        assert rt_f["topk_ids"].cpu().numpy().tolist() == want
    # the permutation is the stable counting sort of the ids
    ids = rt_f["topk_ids"].cpu().numpy()
    order = np.argsort(ids, kind="stable")
    assert np.array_equal(rt_f["sorted_pairs"].cpu().numpy(), order)
    assert np.array_equal(rt_f["pair_pos"].cpu().numpy()[order], np.arange(len(ids)))
    # outputs against the oracle (near-tie protocol on the GPU's ids)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out_f), exp, s.act_dtype, case + " fused")
    _gpu.assert_close(_gpu.to_np(out_s), exp, s.act_dtype, case + " steps")


def test_fused_is_deterministic():
    s, opt = CASES["q8_T16_shared_gated"]
    wl = _workload(s, opt, seed=43)
    desc, w, x = _gpu.upload(wl)
    a, ra, _ = _run(desc, w, x, True)
    b, rb, _ = _run(desc, w, x, True)
    assert torch.equal(_bits(a), _bits(b))
    for k in ra:
        assert torch.equal(_bits(ra[k]), _bits(rb[k]))


def test_fused_back_to_back_calls_share_the_barrier():
    """Many fused launches in a row on one stream (the grid barrier's counter
    carries over from launch to launch) all give the same result."""
    s, opt = CASES["f32_gelu_T1"]
    wl = _workload(s, opt, seed=47)
    desc, w, x = _gpu.upload(wl)
    ref, _, _ = _run(desc, w, x, True)
    out = torch.empty_like(ref)
    ws = torch.full((max(moe.workspace_bytes(desc), 256),), 0xFF, dtype=torch.uint8, device="cuda")
    for _ in range(50):
        moe.layer(desc, x, w, out, ws)
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.MOE_OK
    assert torch.equal(_bits(out), _bits(ref))
