"""Q4_K / Q6_K expert stacks on the weight-streaming path (ferrum-kernels vnext
MoE: the "q4k" and "q4k_q6k" providers), through the C ABI, against the oracle
reading the GGML blocks.

The split of Q6_K blocks moves bytes only, so it is compared bit for bit with
a numpy restatement of the layout include/moe.h documents.  Layer outputs use
the f32 / bf16 tolerances; routing is shared with the other formats and is
bit-exact (the fused decode kernel against the step-by-step launches too).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402
from mixture_experts_ffn_07_b200.host import split_q6_k  # noqa: E402
from tests.test_gpu_parity import make, spec  # noqa: E402


def _numpy_q6_k_split(blocks, rows, cols):
    nb = cols // 256
    b = blocks.reshape(rows, nb, 210)
    q = b[:, :, :192].copy()
    srow = moe.q6_k_srow_bytes(cols)
    s = np.zeros((rows, srow), np.uint8)
    s[:, :16 * nb] = b[:, :, 192:208].reshape(rows, 16 * nb)
    s[:, 16 * nb:18 * nb] = b[:, :, 208:210].reshape(rows, 2 * nb)
    return q, s


@pytest.mark.parametrize("rows,cols", [(1, 256), (7, 768), (300, 512), (33, 2816 // 256 * 256)])
def test_q6_k_split_moves_bytes(rows, cols):
    blocks = workloads.kquant_blocks(5, 3, (rows, cols), "q6_k")
    q, s = split_q6_k(blocks, rows, cols)
    torch.cuda.synchronize()
    rq, rs = _numpy_q6_k_split(blocks, rows, cols)
    assert np.array_equal(q.cpu().numpy().reshape(rows, cols // 256, 192), rq)
    assert np.array_equal(s.cpu().numpy(), rs)


def kspec(T, H, E, I, K, w_dt="q4_k_q6_k", dt="f32", **kw):
    return spec(T, H, E, I, K, dt=dt, w_dt=w_dt, r_dt="f32" if dt == "f32" else "bf16", **kw)


CASES = {
    "q4k_q6k_T1_K_split": (kspec(1, 2048, 32, 512, 2), {}),        # few pairs: rows split along K
    "q4k_q6k_T16": (kspec(16, 1024, 32, 768, 8), {}),
    "q4k_all_T5_gelu": (kspec(5, 512, 16, 256, 4, w_dt="q4_k", act="gelu_tanh"), {}),
    "q4k_q6k_bf16_x_T40": (kspec(40, 512, 16, 512, 4, dt="bf16"), {}),
    "q4k_q6k_shared_gated_T9": (kspec(9, 768, 16, 256, 2, shared=512, gated=True), {}),
    "q4k_shared_ungated_T3": (kspec(3, 512, 8, 256, 2, w_dt="q4_k", shared=256), {}),
    "q4k_q6k_T80_per_step": (kspec(80, 512, 16, 256, 4), {}),       # above the fused decode range
    "q4k_q6k_T64_bias_no_renorm": (kspec(64, 512, 64, 256, 6, renorm=False), dict(bias=True)),
    "q4k_q6k_skew_all_to_two": (kspec(48, 512, 8, 256, 2), dict(skew=True)),
}


def _workload(s, opt, seed):
    bias = None
    if opt.get("bias"):
        bias = np.linspace(2, -2, s.E)
    if opt.get("skew"):
        bias = np.array([50.0, 40.0] + [0.0] * (s.E - 2))
    return make(s, seed=seed, bias_values=bias)


@pytest.mark.parametrize("case", sorted(CASES))
def test_kquant_layer_matches_oracle(case):
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=61)
    desc, w, x = _gpu.upload(wl)
    out = _gpu.run_layer(desc, w, x)
    _, gids, _, _ = _gpu.run_route(desc, w, x)
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out), exp, s.act_dtype, case)


@pytest.mark.parametrize("case", ["q4k_q6k_T16", "q4k_q6k_shared_gated_T9", "q4k_all_T5_gelu"])
def test_fused_decode_matches_steps(case):
    s, opt = CASES[case]
    wl = _workload(s, opt, seed=67)
    desc, w, x = _gpu.upload(wl)
    outs = []
    for fused in (True, False):
        moe.set_fused_decode(fused)
        try:
            n0 = moe.launch_count()
            outs.append((_gpu.run_layer(desc, w, x), moe.launch_count() - n0))
        finally:
            moe.set_fused_decode(True)
    (a, na), (b, nb_) = outs
    assert na == 1 and nb_ >= 4
    exp, _ = _gpu.expected_layer(oracle.from_workload(wl), _gpu.run_route(desc, w, x)[1].cpu().numpy())
    _gpu.assert_close(_gpu.to_np(a), exp, s.act_dtype, case + " fused")
    _gpu.assert_close(_gpu.to_np(b), exp, s.act_dtype, case + " steps")


def test_kquant_is_deterministic():
    s, opt = CASES["q4k_q6k_T16"]
    wl = _workload(s, opt, seed=71)
    desc, w, x = _gpu.upload(wl)
    a = _gpu.run_layer(desc, w, x)
    b = _gpu.run_layer(desc, w, x)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_kquant_rejects_sizes_that_are_not_whole_blocks():
    s = kspec(4, 512, 8, 256, 2)
    wl = make(s, seed=3)
    desc, w, x = _gpu.upload(wl)
    out = torch.empty((4, 512), device="cuda")
    ws = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    bad = moe.Desc(T=4, H=512, E=8, I=128, top_k=2, act_dtype="f32", w_dtype="q4_k_q6_k", router_dtype="f32")
    with pytest.raises(moe.MoeError) as e:
        moe.layer(bad, x, w, out, ws)
    assert e.value.code == moe.MOE_ERR_UNSUPPORTED
    w.down_scale = None
    with pytest.raises(moe.MoeError) as e:
        moe.layer(desc, x, w, out, ws)
    assert e.value.code == moe.MOE_ERR_INVALID_ARG
