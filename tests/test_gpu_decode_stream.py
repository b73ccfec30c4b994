"""The fused decode kernel's gate/up + down stream (a ring of stages per CTA fed by the copy engine from one
issuing warp, work items from a device-wide queue, down items waiting on their expert's gate/up counter)
against the two-phase form of the same kernel and against the oracle, for f32, bf16 and Q8_0 weights (f32 or
bf16 activations): one token, several tokens per expert (token chunks), the shared expert (gated and not),
rows longer than one stage, Q8_0 rows of 1024-code stages with a partial last stage, the most pairs (E = 256,
K = 32), and all pairs on two experts."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
from tests import _gpu  # noqa: E402
from tests.test_gpu_parity import make, spec  # noqa: E402

CASES = {
    "f32_gelu_T1": (spec(1, 512, 16, 256, 4, act="gelu_tanh", dt="f32"), {}),
    "f32_T1_long_rows": (spec(1, 2816, 32, 704, 8, act="gelu_tanh", dt="f32"), {}),
    "f32_T64_shared_gated_bias": (spec(64, 512, 32, 128, 8, dt="f32", shared=64, gated=True), dict(bias=True)),
    "bf16_T40": (spec(40, 256, 32, 128, 8), {}),
    "bf16_T5_shared_ungated": (spec(5, 512, 16, 256, 2, shared=256), {}),
    "f32_skew_chunks": (spec(40, 512, 8, 256, 2, dt="f32"), dict(skew=True)),
    "f32x_bf16w_T3": (spec(3, 384, 8, 64, 2, dt="f32", w_dt="bf16", r_dt="f32"), {}),
    "max_pairs_E256_K32": (spec(64, 128, 256, 32, 32, dt="f32"), {}),
    "skew_all_to_two": (spec(48, 256, 8, 64, 2, dt="f32"), dict(skew=True)),
    "q8_T1": (spec(1, 1024, 16, 512, 4, dt="f32", w_dt="q8_0", r_dt="f32"), {}),
    "q8_T16": (spec(16, 512, 32, 256, 8, dt="f32", w_dt="q8_0", r_dt="f32"), {}),
    "q8_T16_long_rows_shared": (spec(16, 2048, 32, 768, 8, dt="f32", w_dt="q8_0", r_dt="f32", shared=256,
                                     gated=True), {}),
    "q8_T5_ungated_shared_bf16_router": (spec(5, 512, 16, 256, 2, dt="f32", w_dt="q8_0", r_dt="bf16",
                                              shared=256), {}),
    "q8_skew_chunks": (spec(40, 512, 8, 256, 2, dt="f32", w_dt="q8_0", r_dt="f32"), dict(skew=True)),
}


def _workload(s, opt, seed):
    bias = None
    if opt.get("bias"):
        bias = np.linspace(2, -2, s.E)
    if opt.get("skew"):
        bias = np.array([50.0, 40.0] + [0.0] * (s.E - 2))
    return make(s, seed=seed, bias_values=bias)


def _run(desc, w, x, stream: bool):
    moe.set_decode_stream(stream)
    try:
        out = torch.full((desc.T, desc.H), float("nan"), dtype=x.dtype, device="cuda")
        # every workspace byte 0xFF (NaN as f32): a read of a row before it is written shows in the output
        ws = torch.full((max(moe.workspace_bytes(desc), 256),), 0xFF, dtype=torch.uint8, device="cuda")
        n0 = moe.launch_count()
        moe.layer(desc, x, w, out, ws)
        torch.cuda.synchronize()
        assert moe.launch_count() - n0 == 1, "the whole layer is one launch"
        assert moe.last_device_status() == moe.MOE_OK
    finally:
        moe.set_decode_stream(True)
    return out


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.fixture(autouse=True)
def _bf16_on_the_streaming_path():
    with _gpu.streaming_path():  # the bf16 cases are decode batches on the streaming path
        yield


@pytest.mark.parametrize("case", sorted(CASES))
def test_stream_matches_two_phases_and_oracle(case):
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=59)
    desc, w, x = _gpu.upload(wl)
    a = _run(desc, w, x, True)
    b = _run(desc, w, x, False)
    logits, gids, _, _ = _gpu.run_route(desc, w, x)
    exp, flagged = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy(),
                                       gpu_logits=logits.cpu().numpy().astype(np.float64))
    err_a = _gpu.assert_close(_gpu.to_np(a), exp, s.act_dtype, case + " stream")
    err_b = _gpu.assert_close(_gpu.to_np(b), exp, s.act_dtype, case + " two phases")
    # the same exact products summed in a different order: the two forms agree to f32 rounding
    assert np.max(np.abs(_gpu.to_np(a) - _gpu.to_np(b))) <= _gpu.tolerance(exp, s.act_dtype)
    print(f"\n{case}: max|stream-oracle| {err_a:.3e}, max|two phases-oracle| {err_b:.3e}, {flagged} flagged")


@pytest.mark.parametrize("case", ["f32_T64_shared_gated_bias", "f32_T1_long_rows", "f32_skew_chunks",
                                  "q8_T16_long_rows_shared", "q8_skew_chunks"])
def test_stream_is_deterministic(case):
    """Whichever warp takes an item, its arithmetic is fixed: the same bits on every call."""
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=61)
    desc, w, x = _gpu.upload(wl)
    ref = _run(desc, w, x, True)
    for _ in range(5):
        assert torch.equal(_bits(_run(desc, w, x, True)), _bits(ref))
