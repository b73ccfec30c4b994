"""The tensor-core path's fused selection + permutation (route_permute_gather,
one cooperative launch after the router GEMM) against the separate launches
it replaces, moe_route and the oracle.  With the x rows copied into expert
order first (the default) the fused kernel also does that copy and replaces
three launches (router_topk, permute, gather_rows); with the expert GEMM
gathering its rows itself (moe_set_tma_gather(1)) it replaces two.

The fused kernel selects with the same code as router_topk_kernel and the
permutation is a stable sort (unique), so logits, ids, weights, counts,
offsets, sorted pairs and their inverse must be bit-identical to the
separate-launch path, and so must the output (the GEMMs then see the same rows).
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
    "T65_E32": (spec(65, 256, 32, 128, 4), {}),
    "T200_E64_bias": (spec(200, 512, 64, 64, 8), dict(bias=True)),
    "T300_E256_no_renorm": (spec(300, 256, 256, 64, 8, renorm=False), {}),
    "T1100_E256_shared_gated": (spec(1100, 1024, 256, 64, 8, shared=32, gated=True), {}),
    "T333_E64_shared_ungated": (spec(333, 512, 64, 256, 8, shared=96), {}),
    "skew_all_to_two": (spec(300, 256, 32, 64, 2), dict(skew=True)),
    # E not dividing 512 (2, 3, 5 count threads per expert) and 16, 8, 4 split-K partial logits
    # (one, two and four experts' parts requested together)
    "T700_E224_16_parts": (spec(700, 1024, 224, 64, 8), {}),
    "T2000_E160_8_parts": (spec(2000, 1024, 160, 64, 6), {}),
    "T3000_E96_4_parts": (spec(3000, 512, 96, 64, 6), {}),
}


def _workload(s, opt, seed):
    bias = None
    if opt.get("bias"):
        bias = np.linspace(2, -2, s.E)
    if opt.get("skew"):
        bias = np.array([50.0, 40.0] + [0.0] * (s.E - 2))
    return make(s, seed=seed, bias_values=bias)


def _run(desc, w, x, fused):
    moe.set_fused_front(fused)
    try:
        out = torch.empty((desc.T, desc.H), dtype=x.dtype, device="cuda")
        ws = torch.zeros(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
        n0 = moe.launch_count()
        moe.layer(desc, x, w, out, ws)
        torch.cuda.synchronize()
        launches = moe.launch_count() - n0
        assert moe.last_device_status() == moe.MOE_OK
    finally:
        moe.set_fused_front(True)
    reg = moe.workspace_regions(desc)
    T, E, K = desc.T, desc.E, desc.top_k
    P = T * K

    def view(name, n, dtype):
        off = reg[name]
        return ws[off:off + 4 * n].view(dtype).clone()

    r = {"logits": view("logits", T * E, torch.float32), "topk_ids": view("topk_ids", P, torch.int32),
         "topk_w": view("topk_w", P, torch.float32), "counts": view("counts", E, torch.int32),
         "offsets": view("offsets", E + 1, torch.int32), "sorted_pairs": view("sorted_pairs", P, torch.int32),
         "pair_pos": view("pair_pos", P, torch.int32)}
    if desc.shared_I and desc.has_shared_gate:
        r["shared_gate"] = view("shared_gate", T, torch.float32)
    return out, r, launches


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


@pytest.mark.parametrize("case", sorted(CASES))
def test_fused_front_matches_three_launches(case):
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=53)
    desc, w, x = _gpu.upload(wl)
    out_f, rf, nf = _run(desc, w, x, True)
    out_s, rs, ns = _run(desc, w, x, False)
    assert ns - nf == 2  # selection, permutation and the row copy: three launches become one
    for k in rs:
        assert torch.equal(_bits(rf[k]), _bits(rs[k])), f"{case}: {k}"
    assert torch.equal(_bits(out_f), _bits(out_s))
    logits, gids, gw, _ = _gpu.run_route(desc, w, x)
    assert torch.equal(_bits(rf["topk_ids"]), _bits(gids.reshape(-1)))
    assert torch.equal(_bits(rf["topk_w"]), _bits(gw.reshape(-1)))
    ids = rf["topk_ids"].cpu().numpy()
    order = np.argsort(ids, kind="stable")
    assert np.array_equal(rf["sorted_pairs"].cpu().numpy(), order)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out_f), exp, s.act_dtype, case)


def test_fused_front_back_to_back():
    s, opt = CASES["T200_E64_bias"]
    wl = _workload(s, opt, seed=59)
    desc, w, x = _gpu.upload(wl)
    ref, _, _ = _run(desc, w, x, True)
    out = torch.empty_like(ref)
    ws = torch.empty(moe.workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    for _ in range(30):
        moe.layer(desc, x, w, out, ws)
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.MOE_OK
    assert torch.equal(_bits(out), _bits(ref))


def test_fused_front_with_gathering_gemm():
    """With the gate/up GEMM gathering its x rows itself (moe_set_tma_gather(1)) the fused kernel writes no
    copy: two launches become one, and the layer has the same bits as with the copied rows."""
    s, opt = CASES["T333_E64_shared_ungated"]
    wl = _workload(s, opt, seed=57)
    desc, w, x = _gpu.upload(wl)
    out_c, _, n_c = _run(desc, w, x, True)
    moe.set_tma_gather(True)
    try:
        out_f, _, nf = _run(desc, w, x, True)
        out_s, _, ns = _run(desc, w, x, False)
    finally:
        moe.set_tma_gather(False)
    assert ns - nf == 1
    assert nf == n_c
    assert torch.equal(out_f.view(torch.int16), out_s.view(torch.int16))
    assert torch.equal(out_f.view(torch.int16), out_c.view(torch.int16))
