"""GPU parity of the CTA-pair expert GEMMs (tcgen05.mma.cta_group::2, 256 x 256 tiles on clusters of two SMs)
that compute-bound launches use for every group's full 256-row tiles, with the rest of each group's rows on the
single-CTA kernel.  Shapes: groups with several full pair tiles and a ragged remainder (one or two 128-row tail
tiles), groups of exactly 256 or 512 rows (no remainder), small groups next to large ones (no pair tile), output
widths that are not multiples of the 256-column tile, and the shared expert as one group of T rows.  Each case
is checked against the oracle, and against the same layer with the pair kernel switched off."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402


def spec(T, H, E, I, K, shared=0, gated=False, act="silu", name="pair"):
    return workloads.Spec(T=T, H=H, E=E, I=I, K=K, act=act, shared_I=shared, shared_gated=gated, name=name)


# (spec, router bias): the bias steers the loads
CASES = {
    # 700 rows per expert on average: two full pair tiles and a remainder per expert
    "remainders": (spec(1400, 256, 4, 256, 2), None),
    # all pairs on two experts: 700 rows each (2 pair tiles + 188 rows: tails of 128 and 60 rows)
    "skew_two_experts": (spec(700, 512, 8, 128, 2), [50.0, 40.0] + [0.0] * 6),
    # every token on both experts: exactly 512 rows each, no remainder
    "exact_tiles": (spec(512, 256, 2, 256, 2), None),
    # I = 160 (dual tiles of 128 features: a ragged last column tile), H = 352 (ragged 256-column tile)
    "ragged_columns": (spec(900, 352, 4, 160, 2, act="gelu_tanh"), None),
    # two large experts (pair tiles and a remainder each) beside six small ones (single-CTA kernel only)
    "mixed_sizes": (spec(900, 256, 8, 128, 2), [4.0, 3.0] + [0.0] * 6),
    # shared expert: one group of T = 600 rows (two pair tiles + 88 rows); routed groups of ~300 rows
    "shared_expert": (spec(600, 256, 8, 64, 4, shared=256, gated=True), None),
}


def _run(s, bias, pair: bool, seed=41):
    wl = workloads.make(s, seed=seed)
    if bias is not None:
        wl.router_bias = np.asarray(bias, np.float32)
    desc, w, x = _gpu.upload(wl)
    moe.set_pair_gemm(pair)
    try:
        out = _gpu.run_layer(desc, w, x)
    finally:
        moe.set_pair_gemm(True)
    assert moe.last_device_status() == moe.MOE_OK
    return wl, desc, w, x, out


@pytest.mark.parametrize("case", sorted(CASES))
def test_pair_layer_matches_oracle(case):
    s, bias = CASES[case]
    wl, desc, w, x, out = _run(s, bias, pair=True)
    logits, ids, _, _ = _gpu.run_route(desc, w, x)
    L = oracle.from_workload(wl)
    exp, flagged = _gpu.expected_layer(L, ids.cpu().numpy(), gpu_logits=logits.cpu().numpy().astype(np.float64))
    err = _gpu.assert_close(_gpu.to_np(out), exp, s.act_dtype, case)
    counts = np.bincount(ids.cpu().numpy().reshape(-1), minlength=s.E)
    print(f"\n{case}: rows per expert {sorted(counts.tolist(), reverse=True)[:4]}, max|gpu-oracle| {err:.3e}, "
          f"{flagged} flagged")


@pytest.mark.parametrize("case", sorted(CASES))
def test_pair_on_off_agree(case):
    s, bias = CASES[case]
    *_, on = _run(s, bias, pair=True)
    *_, off = _run(s, bias, pair=False)
    a, b = _gpu.to_np(on), _gpu.to_np(off)
    same = bool(np.array_equal(on.view(torch.int16).cpu().numpy(), off.view(torch.int16).cpu().numpy()))
    # both are f32 accumulations of the same exact bf16 products: they differ by rounding order at most
    assert np.max(np.abs(a - b)) <= 2e-2 * np.max(np.abs(b))
    print(f"\n{case}: pair vs single-CTA bits identical: {same}, max|diff| {np.max(np.abs(a - b)):.3e}")


def test_pair_expert_ffn_f32_slots():
    """moe_expert_ffn's weighted f32 slot rows through the pair kernel (single mode, f32 epilogue)."""
    s = spec(1200, 256, 4, 128, 2)
    wl = workloads.make(s, seed=43)
    desc, w, x = _gpu.upload(wl)
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
    assert int(counts.min()) >= 256  # every expert has a full pair tile
    y = torch.full((P, s.H), float("nan"), dtype=torch.float32, device="cuda")
    ws = torch.full((moe.workspace_bytes(desc),), 0xFF, dtype=torch.uint8, device="cuda")
    moe.expert_ffn(desc, x, w, offsets, sp, tw, y, ws)
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.MOE_OK
    got = y.cpu().numpy().astype(np.float64)
    exp = np.zeros_like(got)
    for p in range(P):
        t, k = divmod(p, s.K)
        exp[p] = ref["w"][t, k] * oracle.expert(L, t, int(ids[t, k]))
    _gpu.assert_close(got, exp, s.act_dtype, "pair_expert_ffn")
