"""Backward of the combine and of act(gate)*up on the GPU, through the C ABI,
against the oracle (mlx-native moe_dispatch.rs, the backward kernels of
moe_weighted_sum_seq and moe_swiglu_seq).

d_y = w * d_out is one f32 product, so it equals the oracle's f64 value
rounded to f32 bit for bit.  d_w is a dot product over H summed in another
order: its error is bounded by H * 2^-24 * sum_h |y d_out| (+ tiny).  The
act * up gradients use the f32 tolerance of the layer (1e-3 * max + 1e-5).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
from tests import _gpu  # noqa: E402

F32_TOL = (1e-3, 1e-5)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def _combine(T, K, H, seed, offset=0):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((T, K, H)).astype(np.float32)
    w = rng.random((T, K)).astype(np.float32)
    d_out = rng.standard_normal((T, H)).astype(np.float32)
    # `offset` floats of padding in front of every device buffer: unaligned views take the scalar kernel
    def dev(a):
        flat = torch.zeros(a.size + offset, dtype=torch.float32, device="cuda")
        flat[offset:] = torch.from_numpy(a.reshape(-1)).cuda()
        return flat[offset:].view(a.shape)

    yd, wd, dd = dev(y), dev(w), dev(d_out)
    d_y = torch.full((T, K, H), float("nan"), device="cuda")
    d_w = torch.full((T, K), float("nan"), device="cuda")
    moe.combine_backward(yd, wd, dd, d_y, d_w)
    torch.cuda.synchronize()
    return y, w, d_out, d_y.cpu().numpy(), d_w.cpu().numpy()


@pytest.mark.parametrize("T,K,H,offset", [
    (3, 4, 7, 0),        # the page's falsifier sizes (scalar path)
    (512, 8, 2048, 0),   # the prefill workload's slots
    (37, 9, 2052, 0),    # two slot groups, ragged last group, H not a multiple of 1024
    (5, 1, 6, 0),        # K = 1, H % 4 != 0
    (64, 32, 256, 0),    # the largest top-K
    (17, 3, 2048, 1),    # unaligned buffers: scalar path
    (1, 8, 7168, 0),     # the skewed workload's hidden size, one token
])
def test_combine_backward_matches_oracle(T, K, H, offset):
    y, w, d_out, d_y, d_w = _combine(T, K, H, seed=T * 31 + K, offset=offset)
    ry, rw = oracle.combine_backward(y, w, d_out)
    assert np.array_equal(d_y, ry.astype(np.float32)), "d_y is one f32 product: bit-exact"
    bound = H * 2.0 ** -24 * np.einsum("tkh,th->tk", np.abs(y).astype(np.float64), np.abs(d_out)) + 1e-30
    assert np.all(np.abs(d_w - rw) <= bound), float(np.max(np.abs(d_w - rw) / bound))


def test_combine_backward_is_deterministic():
    a = _combine(300, 8, 2048, seed=3)
    b = _combine(300, 8, 2048, seed=3)
    assert np.array_equal(a[4].view(np.int32), b[4].view(np.int32))


def _act_up(act, P, I, seed, scale=3.0, offset=0):
    rng = np.random.default_rng(seed)
    gu = (scale * rng.standard_normal((P, 2 * I))).astype(np.float32)
    dh = rng.standard_normal((P, I)).astype(np.float32)

    def dev(a):
        flat = torch.zeros(a.size + offset, dtype=torch.float32, device="cuda")
        flat[offset:] = torch.from_numpy(a.reshape(-1)).cuda()
        return flat[offset:].view(a.shape)

    out = torch.full((P, 2 * I), float("nan"), device="cuda")
    moe.act_up_backward(act, dev(gu), dev(dh), out)
    torch.cuda.synchronize()
    return gu, dh, out.cpu().numpy()


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("P,I,offset", [(6, 5, 0), (4096, 1024, 0), (1000, 516, 0), (33, 7, 0), (129, 256, 3),
                                         (32768, 512, 0)])
def test_act_up_backward_matches_oracle(act, P, I, offset):
    gu, dh, got = _act_up(act, P, I, seed=P + I, offset=offset)
    ref = oracle.act_up_backward(act, gu, dh)
    for half, name in ((slice(0, I), "d_gate"), (slice(I, 2 * I), "d_up")):
        r, g = ref[:, half], got[:, half]
        tol = F32_TOL[0] * np.max(np.abs(r)) + F32_TOL[1]
        assert np.max(np.abs(g - r)) <= tol, (act, name, float(np.max(np.abs(g - r))), tol)


@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
def test_act_up_backward_canonical_points(act):
    """The page's canonical gradient values on the GPU (gate 0, +10, -10)."""
    import json
    import os
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "backward_canonical.json")))
    gu = _dev(np.array([g["gate_up"]]))
    out = torch.zeros_like(gu)
    moe.act_up_backward(act, gu, _dev(np.array([g["d_h"]])), out)
    got = out.cpu().numpy()[0]
    for v, e, tol in zip(got, g["expected_d_gate_up"], g["tol"]):
        assert abs(v - e) <= tol, (act, v, e)


def test_act_up_backward_extreme_gates_stay_finite():
    I = 8
    gu = np.array([[-1e4, -100.0, -20.0, -1e-30, 0.0, 1e-30, 100.0, 1e4] + [1.0] * I], np.float32)
    dh = np.ones((1, I), np.float32)
    for act in ("silu", "gelu_tanh"):
        out = torch.zeros((1, 2 * I), device="cuda")
        moe.act_up_backward(act, _dev(gu), _dev(dh), out)
        got = out.cpu().numpy()
        assert np.all(np.isfinite(got)), (act, got)
        ref = oracle.act_up_backward(act, gu, dh)
        assert np.max(np.abs(got - ref)) <= 1e-3 * np.max(np.abs(ref)) + 1e-5, act


def test_backward_zero_sizes_and_bad_arguments():
    x = torch.zeros(64, device="cuda")
    L = moe._lib.lib()
    s = torch.cuda.current_stream().cuda_stream
    # empty batches: nothing to do
    assert L.moe_combine_backward(0, 8, 16, x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                  s) == moe.MOE_OK
    assert L.moe_act_up_backward(0, 16, 0, x.data_ptr(), x.data_ptr(), x.data_ptr(), s) == moe.MOE_OK
    # an output that aliases an input is rejected before any launch
    y = torch.zeros((2, 2, 4), device="cuda")
    with pytest.raises(moe.MoeError):
        moe.combine_backward(y, torch.zeros((2, 2), device="cuda"), torch.zeros((2, 4), device="cuda"), y,
                             torch.zeros((2, 2), device="cuda"))
    gu = torch.zeros((3, 8), device="cuda")
    with pytest.raises(moe.MoeError):
        moe.act_up_backward("silu", gu, torch.zeros((3, 4), device="cuda"), gu)
    torch.cuda.synchronize()
    assert moe.last_device_status() == moe.MOE_OK
