"""The routed gate/up GEMM reading its x rows straight from x with copy-engine row gathers (tile::gather4,
four token rows per load) against the same layer reading a copy of the rows in expert order
(moe_set_tma_gather(0)): the same products in the same order, so the same bits, on single-CTA and CTA-pair
launches, ragged tiles, the last tile of the last expert (rows past the pairs read a clamped row), the
step-by-step entry point, and against the oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402

CASES = {
    "single_cta_ragged": workloads.Spec(T=200, H=256, E=16, I=160, K=4, name="g_single"),
    "pair_and_tails": workloads.Spec(T=1400, H=256, E=4, I=256, K=2, name="g_pair"),
    "shared_expert_E32": workloads.Spec(T=333, H=512, E=32, I=256, K=8, shared_I=96, shared_gated=True,
                                        name="g_shared"),
    "wide_H": workloads.Spec(T=130, H=4096, E=8, I=64, K=2, act="gelu_tanh", name="g_wide"),
}


def _layer(wl, gather):
    moe.set_tma_gather(gather)
    try:
        desc, w, x = _gpu.upload(wl)
        out = _gpu.run_layer(desc, w, x)
    finally:
        moe.set_tma_gather(False)
    assert moe.last_device_status() == moe.MOE_OK
    return desc, w, x, out


@pytest.mark.parametrize("case", sorted(CASES))
def test_gather_matches_copied_rows_bit_for_bit(case):
    wl = workloads.make(CASES[case], seed=67)
    desc, w, x, a = _layer(wl, True)
    *_, b = _layer(wl, False)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    logits, ids, _, _ = _gpu.run_route(desc, w, x)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), ids.cpu().numpy(),
                                 gpu_logits=logits.cpu().numpy().astype(np.float64))
    _gpu.assert_close(_gpu.to_np(a), exp, "bf16", case)


def test_gather_in_expert_ffn_step():
    """moe_expert_ffn (f32 weighted slot rows) on the tensor path with gathered rows."""
    s = CASES["single_cta_ragged"]
    wl = workloads.make(s, seed=71)
    desc, w, x = _gpu.upload(wl)
    moe.set_tma_gather(True)
    L = oracle.from_workload(wl)
    ref = oracle.layer(L)
    ids = ref["ids"]
    P = s.T * s.K
    d_ids = torch.from_numpy(ids.reshape(-1).astype(np.int32)).cuda()
    tw = torch.from_numpy(ref["w"].reshape(-1).astype(np.float32)).cuda()
    counts = torch.empty(s.E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(s.E + 1, dtype=torch.int32, device="cuda")
    sp = torch.empty(P, dtype=torch.int32, device="cuda")
    pp = torch.empty(P, dtype=torch.int32, device="cuda")
    moe.permute(desc, d_ids, counts, offsets, sp, pp)
    y = torch.full((P, s.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    try:
        moe.expert_ffn(desc, x, w, offsets, sp, tw, y, ws)
        torch.cuda.synchronize()
    finally:
        moe.set_tma_gather(False)
    assert moe.last_device_status() == moe.MOE_OK
    got = y.cpu().numpy().astype(np.float64)
    exp = np.zeros_like(got)
    for p in range(P):
        t, k = divmod(p, s.K)
        exp[p] = ref["w"][t, k] * oracle.expert(L, t, int(ids[t, k]))
    _gpu.assert_close(got, exp, "bf16", "expert_ffn gathered")


def test_workspace_shrinks_by_the_copied_rows():
    desc = moe.Desc(T=4096, H=2048, E=256, I=512, top_k=8)
    with_copy = moe.workspace_bytes(desc)
    moe.set_tma_gather(True)
    try:
        with_gather = moe.workspace_bytes(desc)
    finally:
        moe.set_tma_gather(False)
    assert with_copy - with_gather >= 4096 * 8 * 2048 * 2
