"""GPU parity: every stage of the C ABI against the f64 oracle on seeded inputs.

Sizes are small enough for the oracle to finish in seconds but span several
tiles and ragged tails (M tiles of 128 rows, N tiles of 128/256 columns,
K blocks of 64).  Integer results (expert ids, permutation) are compared
bit-exactly; floating-point outputs within |gpu - oracle|_inf <= 2e-2 max|oracle|
for bf16 and <= 1e-3 max|oracle| + 1e-5 for f32 activations.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import mixture_experts_ffn_07_b200 as moe  # noqa: E402
import oracle  # noqa: E402
import workloads  # noqa: E402
from tests import _gpu  # noqa: E402


def spec(T, H, E, I, K, act="silu", dt="bf16", w_dt=None, r_dt=None, shared=0, gated=False, bias=None,
         renorm=True, name="case"):
    return workloads.Spec(T=T, H=H, E=E, I=I, K=K, act=act, act_dtype=dt, w_dtype=w_dt or dt,
                          router_dtype=r_dt or dt, shared_I=shared, shared_gated=gated, renormalize=renorm,
                          router_bias=bias, name=name)


def make(s, seed=11, bias_values=None, router_std=None):
    if router_std is not None:
        s.router_std = router_std
    wl = workloads.make(s, seed=seed)
    if bias_values is not None:
        wl.router_bias = np.asarray(bias_values, np.float32)
    return wl


ROUTE_CASES = {
    "f32_simt": (spec(5, 256, 16, 64, 4, dt="f32"), None),
    "bf16_cluster_router": (spec(200, 512, 64, 64, 8), None),
    "bf16_tensor_router_large": (spec(1100, 1024, 256, 64, 8, shared=32, gated=True), "bias"),
    "bf16_simt_router_bias_gated": (spec(130, 256, 48, 64, 6, shared=32, gated=True), "bias"),
    "bf16_tensor_no_renorm_E256": (spec(300, 256, 256, 64, 8, renorm=False), None),
    "K_equals_E": (spec(7, 128, 8, 64, 8, dt="f32"), None),
    "single_expert": (spec(100, 256, 1, 64, 1), None),
    "f32_x_bf16_router": (spec(9, 256, 32, 64, 4, dt="f32", r_dt="bf16"), None),
}


@pytest.mark.parametrize("case", sorted(ROUTE_CASES))
def test_route(case):
    s, bias = ROUTE_CASES[case]
    wl = make(s, bias_values=(np.linspace(-3, 3, s.E)[::-1] if bias else None))
    desc, w, x = _gpu.upload(wl)
    logits, ids, tw, sg = _gpu.run_route(desc, w, x)
    L = oracle.from_workload(wl)
    ref_logits, absmax = oracle.logits(L)
    gl = logits.cpu().numpy().astype(np.float64)
    # logits: f32 accumulation of exact products, error well inside 2^-24 * 64 * sum|x w|
    assert np.all(np.abs(gl - ref_logits) <= 64 * 2.0 ** -24 * absmax[:, None] + 1e-7)
    # selection and weights on the GPU's own logits: ids bit-exact, weights to f32 rounding
    ref_ids, ref_w = oracle.select(gl, s.K, s.renormalize)
    assert np.array_equal(ids.cpu().numpy(), ref_ids)
    assert np.max(np.abs(tw.cpu().numpy() - ref_w)) < 2e-6
    if s.shared_I and s.shared_gated:
        _, gs = oracle.shared(L)
        assert np.max(np.abs(sg.cpu().numpy()[: s.T] - gs)) < 1e-5


PERMUTE_CASES = {
    "uniform": (300, 8, 64, "uniform"),
    "all_to_one": (257, 4, 16, "one"),
    "empty_experts": (100, 2, 256, "few"),
    "tiny": (1, 1, 4, "uniform"),
    "large": (8192, 8, 256, "zipf"),
    "two_ctas": (1250, 8, 64, "uniform"),
    "beyond_cluster": (9000, 8, 256, "zipf"),
    "ragged": (77, 3, 5, "uniform"),
}


def _ids(T, K, E, kind, rng):
    if kind == "one":
        base = np.zeros((T, K), np.int64) + np.arange(K)[None, :]
        return (base % E).astype(np.int32)
    if kind == "few":
        return rng.choice(4, size=(T, K), replace=True).astype(np.int32) * 37 % E
    if kind == "zipf":
        p = 1.0 / np.arange(1, E + 1) ** 1.1
        p /= p.sum()
        return np.stack([rng.choice(E, K, replace=False, p=p) for _ in range(T)]).astype(np.int32)
    return np.stack([rng.choice(E, K, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("case", sorted(PERMUTE_CASES))
def test_permute(case):
    T, K, E, kind = PERMUTE_CASES[case]
    ids = _ids(T, K, E, kind, np.random.default_rng(T + K + E))
    desc = moe.Desc(T=T, H=64, E=E, I=64, top_k=K)
    P = T * K
    d_ids = torch.from_numpy(ids.reshape(-1)).cuda()
    counts = torch.full((E,), -1, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -1, dtype=torch.int32, device="cuda")
    sp = torch.full((P,), -1, dtype=torch.int32, device="cuda")
    pp = torch.full((P,), -1, dtype=torch.int32, device="cuda")
    moe.permute(desc, d_ids, counts, offsets, sp, pp)
    assert moe.last_device_status() == moe.MOE_OK
    rc, ro, rs, rp = oracle.permute(ids, E)
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(sp.cpu().numpy(), rs)
    assert np.array_equal(pp.cpu().numpy(), rp)


def test_permute_reports_out_of_range_ids():
    ids = torch.tensor([0, 1, 5, 2], dtype=torch.int32, device="cuda")   # 5 >= E
    desc = moe.Desc(T=2, H=64, E=4, I=64, top_k=2)
    bufs = [torch.zeros(n, dtype=torch.int32, device="cuda") for n in (4, 5, 4, 4)]
    moe.permute(desc, ids, *bufs)
    assert moe.last_device_status() == moe.MOE_ERR_DEVICE_INDEX
    assert moe.last_device_status() == moe.MOE_OK      # reading clears the word
    assert bufs[0].cpu().tolist() == [1, 1, 1, 0]


FFN_CASES = {
    "tensor_ragged": spec(200, 256, 16, 160, 4),
    "tensor_multi_mtile": spec(300, 384, 8, 128, 2),
    "tensor_two_row_tiles_per_item": spec(520, 384, 8, 128, 2),
    "stream_f32_gelu": spec(6, 256, 16, 96, 4, act="gelu_tanh", dt="f32"),
    "stream_bf16": spec(40, 256, 32, 128, 8),
    "stream_q8": spec(16, 256, 32, 128, 8, dt="f32", w_dt="q8_0", r_dt="f32"),
    "stream_f32x_bf16w": spec(10, 256, 16, 64, 2, dt="f32", w_dt="bf16", r_dt="f32"),
}


@pytest.fixture
def path_for(request):
    """Cases named stream_* run with bf16 batches of up to 64 tokens on the streaming path."""
    case = request.node.callspec.params.get("case", "")
    if case.startswith("stream_"):
        with _gpu.streaming_path():
            yield
    else:
        yield


@pytest.mark.parametrize("case", sorted(FFN_CASES))
def test_expert_ffn(case, path_for):
    s = FFN_CASES[case]
    wl = make(s, seed=5)
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
    _gpu.assert_close(got, exp, s.act_dtype, case)


LAYER_CASES = {
    "stream_f32_gelu_decode": (spec(5, 256, 16, 128, 4, act="gelu_tanh", dt="f32"), {}),
    "tensor_bf16_ragged_I": (spec(200, 256, 16, 160, 4), {}),
    "tensor_bf16_shared_gated": (spec(333, 512, 64, 256, 8, shared=96, gated=True), {}),
    "tensor_bf16_bias_ungated_ragged_H": (spec(257, 352, 32, 64, 2, shared=64), dict(bias=True)),
    "stream_bf16_T64_shared": (spec(64, 256, 16, 128, 4, shared=64, gated=True), {}),
    "tensor_bf16_T65": (spec(65, 256, 16, 128, 4), {}),
    "stream_q8": (spec(16, 256, 32, 128, 8, dt="f32", w_dt="q8_0", r_dt="f32"), {}),
    "stream_q8_shared": (spec(9, 256, 16, 64, 2, dt="f32", w_dt="q8_0", r_dt="f32", shared=64, gated=True), {}),
    "stream_f32x_bf16w": (spec(10, 256, 16, 64, 2, dt="f32", w_dt="bf16", r_dt="f32"), {}),
    "dense_E1_K1": (spec(100, 256, 1, 128, 1), {}),
    "skew_all_to_two": (spec(300, 256, 8, 64, 2), dict(skew=True)),
    "no_renorm_gelu_tensor": (spec(150, 256, 32, 96, 4, act="gelu_tanh", renorm=False), {}),
    "K_equals_E_stream": (spec(3, 128, 4, 64, 4, dt="f32"), {}),
    "stream_f32_wide_H_token_batches": (spec(20, 4096, 4, 64, 2, dt="f32", shared=32), {}),
    # more than 96 rows per expert: items of two row tiles against one weight tile
    "tensor_bf16_two_row_tiles": (spec(700, 256, 8, 128, 2), {}),
    "tensor_bf16_two_row_tiles_odd": (spec(390, 256, 4, 64, 2, act="gelu_tanh"), {}),
    "tensor_bf16_two_row_tiles_skew": (spec(700, 256, 8, 96, 2), dict(skew=True)),
    "tensor_bf16_shared_T150_two_row_tiles": (spec(150, 256, 16, 64, 4, shared=128, gated=True), {}),
    "tensor_bf16_wide_tiles": (spec(600, 256, 4, 64, 2), {}),   # 300 rows per expert: compute-bound, N = 256 tiles
}


@pytest.mark.parametrize("case", sorted(LAYER_CASES))
def test_layer(case, path_for):
    s, opt = LAYER_CASES[case]
    bias = None
    if opt.get("bias"):
        bias = np.linspace(2, -2, s.E)
    if opt.get("skew"):
        bias = np.array([50.0, 40.0] + [0.0] * (s.E - 2))
    wl = make(s, seed=17, bias_values=bias)
    desc, w, x = _gpu.upload(wl)
    out = _gpu.run_layer(desc, w, x)
    _, gids, _, _ = _gpu.run_route(desc, w, x)
    L = oracle.from_workload(wl)
    exp, flagged = _gpu.expected_layer(L, gids.cpu().numpy())
    _gpu.assert_close(_gpu.to_np(out), exp, s.act_dtype, case)


def test_empty_batch():
    s = spec(0, 256, 16, 128, 4)
    desc = moe.Desc(T=0, H=256, E=16, I=128, top_k=4)
    wl = make(spec(1, 256, 16, 128, 4))
    _, w, _ = _gpu.upload(wl)
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    ws = torch.full((max(moe.workspace_bytes(desc), 256),), 0xFF, dtype=torch.uint8, device="cuda")
    n0 = moe.launch_count()
    moe.layer(desc, x, w, out, ws)
    assert moe.launch_count() == n0
    assert s.T == 0


@pytest.mark.parametrize("case", ["tensor_bf16_shared_gated", "stream_q8"])
def test_deterministic(case):
    s, _ = LAYER_CASES[case]
    wl = make(s, seed=23)
    desc, w, x = _gpu.upload(wl)
    a = _gpu.run_layer(desc, w, x)
    b = _gpu.run_layer(desc, w, x)
    assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def test_layer_host_matches_device_call():
    s, _ = LAYER_CASES["tensor_bf16_shared_gated"]
    wl = make(s, seed=29)
    desc, w, x = _gpu.upload(wl)
    ref = _gpu.run_layer(desc, w, x)
    xh = x.cpu().pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    xd = torch.empty_like(x)
    od = torch.empty_like(x)
    ws = torch.full((moe.workspace_bytes(desc),), 0xFF, dtype=torch.uint8, device="cuda")
    moe.layer_host(desc, xh, w, oh, xd, od, ws)
    torch.cuda.synchronize()
    assert torch.equal(oh.view(torch.int16), ref.cpu().view(torch.int16))


def test_token_order_invariance_on_gpu():
    s, _ = LAYER_CASES["tensor_bf16_ragged_I"]
    wl = make(s, seed=31)
    desc, w, x = _gpu.upload(wl)
    out = _gpu.run_layer(desc, w, x)
    perm = torch.randperm(s.T, generator=torch.Generator().manual_seed(0)).cuda()
    out_p = _gpu.run_layer(desc, w, x[perm].contiguous())
    assert torch.equal(out_p.view(torch.int16), out[perm].view(torch.int16))



@pytest.mark.parametrize("case", ["tensor_bf16_shared_gated", "stream_q8_shared"])
def test_two_streams_alternating_host_calls(case):
    """moe_layer_host calls alternating over two streams, each with its own buffers and workspace (the pipelined
    end-to-end benchmark), give the bits of one stream.  Both cooperative kernels (the prefill front and the fused
    decode layer) keep their grid barriers consistent across the streams."""
    s, _ = LAYER_CASES[case]
    wl = make(s, seed=37)
    desc, w, x = _gpu.upload(wl)
    ref = _gpu.run_layer(desc, w, x)
    xh = x.cpu().pin_memory()
    sets = [dict(oh=torch.empty_like(xh).pin_memory(), xd=torch.empty_like(x), od=torch.empty_like(x),
                 ws=torch.full((moe.workspace_bytes(desc),), 0xFF, dtype=torch.uint8, device="cuda"),
                 stream=torch.cuda.Stream()) for _ in range(2)]
    outs = []
    for i in range(8):
        b = sets[i % 2]
        if i >= 2:  # the pinned output of this stream's previous step is read before it is overwritten
            b["stream"].synchronize()
            outs.append(b["oh"].clone())
        moe.layer_host(desc, xh, w, b["oh"], b["xd"], b["od"], b["ws"], stream=b["stream"])
    torch.cuda.synchronize()
    outs += [sets[0]["oh"].clone(), sets[1]["oh"].clone()]
    assert moe.last_device_status() == moe.MOE_OK
    bits = (lambda t: t.view(torch.int16)) if ref.dtype == torch.bfloat16 else (lambda t: t.view(torch.int32))
    for o in outs:
        assert torch.equal(bits(o), bits(ref.cpu()))
