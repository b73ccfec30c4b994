"""The C-ABI library loads and exports every symbol include/moe.h declares, and the
host-side checks reject bad arguments before touching CUDA (CPU only: no compute calls)."""
import ctypes
import os
import re

import pytest

from tests.conftest import ROOT

HEADER = os.path.join(ROOT, "include", "moe.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def L():
    from mixture_experts_ffn_07_b200 import _lib
    return _lib.lib()


def test_exports_every_declared_symbol(L):
    from mixture_experts_ffn_07_b200 import _lib
    names = _declared()
    assert len(names) >= 15
    assert sorted(_lib.EXPORTS) == names
    for n in names:
        assert hasattr(L, n), n


def test_struct_layouts_match_header(L):
    from mixture_experts_ffn_07_b200 import _lib
    src = open(HEADER).read()
    desc_fields = re.search(r"typedef struct moe_desc \{(.*?)\} moe_desc;", src, re.S).group(1)
    desc_fields = re.sub(r"/\*.*?\*/", "", desc_fields, flags=re.S)
    n_desc = sum(len(line.split(";")[0].replace("int32_t", "").split(",")) for line in desc_fields.split("\n")
                 if "int32_t" in line)
    assert ctypes.sizeof(_lib.MoeDesc) == 4 * n_desc
    w_fields = re.search(r"typedef struct moe_weights \{(.*?)\} moe_weights;", src, re.S).group(1)
    assert ctypes.sizeof(_lib.MoeWeights) == 8 * w_fields.count(";")
    assert [f[0] for f in _lib.MoeDesc._fields_] == re.findall(r"([A-Za-z_]+)\s*[,;]", desc_fields)


def test_status_strings_and_version(L):
    import mixture_experts_ffn_07_b200 as moe
    assert moe.status_string(0) == "ok"
    assert "timed out" in moe.status_string(moe.MOE_ERR_TIMEOUT)
    assert "sm_100a" in moe.version()


def test_workspace_bytes_host_only():
    import mixture_experts_ffn_07_b200 as moe
    d = moe.Desc(T=512, H=2048, E=64, I=1024, top_k=8)
    n = moe.workspace_bytes(d)
    P = 512 * 8
    # routing + permutation + slots [P,H] f32 + the x rows in expert order [P,H] bf16 + h [P,I] bf16
    assert n >= P * 2048 * 4 + P * 2048 * 2 + P * 1024 * 2
    assert n % 256 == 0
    # with the gate/up GEMM gathering the x rows itself: no [P,H] bf16 copy
    moe.set_tma_gather(True)
    try:
        assert n - moe.workspace_bytes(d) >= P * 2048 * 2
    finally:
        moe.set_tma_gather(False)
    # affine in T without the tensor-core router; with it, plus at most 20480 * E * 4 bytes of split-K scratch
    # and 256 * E * 4 bytes of per-CTA expert counts (each region 256-byte aligned)
    ts = (1024, 2048, 3072, 4096, 8192)
    plain = [moe.workspace_bytes(moe.Desc(T=t, H=2048, E=64, I=1024, top_k=8, router_dtype="f32")) for t in ts]
    step = (plain[1] - plain[0]) / 1024
    for t, sz in zip(ts, plain):
        assert abs(sz - plain[0] - step * (t - 1024)) <= 256 * 16
    for t, sz in zip(ts, plain):
        extra = moe.workspace_bytes(moe.Desc(T=t, H=2048, E=64, I=1024, top_k=8)) - sz
        assert 0 < extra <= (20480 + 256) * 64 * 4 + 2 * 256
    assert moe.workspace_bytes(moe.Desc(T=1, H=33, E=4, I=32, top_k=1)) == 0   # invalid -> 0


@pytest.mark.parametrize("bad", [dict(E=0), dict(E=257), dict(top_k=0), dict(top_k=33, E=64), dict(top_k=5, E=4),
                                 dict(T=-1), dict(H=0), dict(act=7), dict(renormalize=2), dict(act_dtype=2),
                                 dict(w_dtype=5), dict(T=(1 << 20) + 1), dict(gating=2), dict(n_groups=-1),
                                 dict(n_groups=33, E=66), dict(n_groups=3), dict(n_groups=2, topk_groups=0),
                                 dict(n_groups=2, topk_groups=3), dict(n_groups=4, topk_groups=1, top_k=2)])
def test_invalid_descriptor_rejected_before_cuda(bad):
    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import _lib
    d = _lib.MoeDesc(8, 64, 4, 64, 2, 0, 1, 1, 1, 1, 0, 0, 0)
    for k, v in bad.items():
        setattr(d, k, v)
    w = _lib.MoeWeights()
    rc = _lib.lib().moe_layer(ctypes.byref(d), None, ctypes.byref(w), None, None, 0, None)
    assert rc == moe.MOE_ERR_INVALID_ARG


def test_routing_options_accepted():
    """Valid gating / group settings pass validation (moe_workspace_bytes returns 0 only for invalid descriptors)."""
    from mixture_experts_ffn_07_b200 import _lib
    for gating, n_groups, topk_groups, K in ((1, 0, 0, 2), (0, 1, 7, 2), (1, 2, 1, 2), (0, 4, 2, 2), (1, 4, 4, 4)):
        d = _lib.MoeDesc(8, 64, 4, 64, K, 0, 1, 1, 1, 1, 0, 0, 0, gating, n_groups, topk_groups)
        assert _lib.lib().moe_workspace_bytes(ctypes.byref(d)) > 0, (gating, n_groups, topk_groups, K)


def test_unsupported_sizes_and_bad_pointers():
    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import _lib
    L = _lib.lib()
    d = _lib.MoeDesc(8, 48, 4, 64, 2, 0, 1, 1, 1, 1, 0, 0, 0)           # H not a multiple of 32
    w = _lib.MoeWeights()
    assert L.moe_layer(ctypes.byref(d), None, ctypes.byref(w), None, None, 0, None) == moe.MOE_ERR_UNSUPPORTED
    d.H = 64
    assert L.moe_layer(ctypes.byref(d), None, ctypes.byref(w), None, None, 0, None) == moe.MOE_ERR_INVALID_ARG
    # misaligned x pointer (not 16-byte aligned) is rejected on the host
    w.router = 0x1000
    w.gate = w.up = w.down = 0x2000
    assert L.moe_route(ctypes.byref(d), 0x1001, ctypes.byref(w), 0x3000, 0x4000, 0x5000, None, None, 0, None) == \
        moe.MOE_ERR_INVALID_ARG
    # workspace too small
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, 16, None) == moe.MOE_ERR_WORKSPACE
    # out aliasing x
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x1000, 0x7000, 1 << 30, None) == \
        moe.MOE_ERR_INVALID_ARG
    # Q8_0 without scale planes
    d.w_dtype = moe.MOE_Q8_0
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, 1 << 30, None) == \
        moe.MOE_ERR_INVALID_ARG
    assert L.moe_q8_0_split(None, 4, 48, None, None, None) == moe.MOE_ERR_INVALID_ARG


def test_streaming_path_row_limit():
    """The weight-streaming path stages whole token rows (<= 64 KB) in shared
    memory; larger rows are rejected on the host, the tensor-core path is not."""
    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import _lib
    L = _lib.lib()
    w = _lib.MoeWeights(router=0x1000, gate=0x2000, up=0x2000, down=0x2000)
    big = 1 << 34
    # f32 x with H = 16416 (65664-byte rows) on the streaming path
    d = _lib.MoeDesc(4, 16416, 4, 64, 2, 0, 1, moe.MOE_F32, moe.MOE_F32, moe.MOE_F32, 0, 0, 0)
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, big, None) == \
        moe.MOE_ERR_UNSUPPORTED
    d.H = 16384  # exactly 64 KB passes validation (the call then fails only for want of a device)
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, big, None) != \
        moe.MOE_ERR_UNSUPPORTED
    # hidden rows: I * 4 bytes
    d.H, d.I = 64, 16416
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, big, None) == \
        moe.MOE_ERR_UNSUPPORTED
    # the same sizes in bf16 with T > 64 take the tensor-core path: no row limit
    d = _lib.MoeDesc(100, 16416, 4, 64, 2, 0, 1, moe.MOE_BF16, moe.MOE_BF16, moe.MOE_BF16, 0, 0, 0)
    assert L.moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, big, None) != \
        moe.MOE_ERR_UNSUPPORTED


def test_empty_batch_is_a_no_op_without_cuda():
    import mixture_experts_ffn_07_b200 as moe
    from mixture_experts_ffn_07_b200 import _lib
    d = _lib.MoeDesc(0, 64, 4, 64, 2, 0, 1, 1, 1, 1, 0, 0, 0)
    w = _lib.MoeWeights(router=0x1000, gate=0x2000, up=0x2000, down=0x2000)
    ws = moe.workspace_bytes(moe.Desc(T=0, H=64, E=4, I=64, top_k=2))
    assert _lib.lib().moe_layer(ctypes.byref(d), 0x1000, ctypes.byref(w), 0x6000, 0x7000, max(ws, 256), None) == \
        moe.MOE_OK


def test_workspace_regions_host_only():
    import mixture_experts_ffn_07_b200 as moe
    for d in (moe.Desc(T=1, H=2816, E=128, I=704, top_k=8, act_dtype="f32", w_dtype="f32", router_dtype="f32"),
              moe.Desc(T=512, H=2048, E=64, I=1024, top_k=8),
              moe.Desc(T=16, H=2048, E=128, I=768, top_k=8, act_dtype="f32", w_dtype="q8_0", router_dtype="f32",
                       shared_I=64, has_shared_gate=1)):
        r = moe.workspace_regions(d)
        n = moe.workspace_bytes(d)
        P = d.T * d.top_k
        sizes = {"logits": d.T * d.E * 4, "topk_ids": P * 4, "topk_w": P * 4, "shared_gate": d.T * 4,
                 "counts": d.E * 4, "offsets": (d.E + 1) * 4, "sorted_pairs": P * 4, "pair_pos": P * 4}
        spans = sorted((r[k], r[k] + sizes[k]) for k in sizes)
        for (a0, a1), (b0, _) in zip(spans, spans[1:]):
            assert a1 <= b0  # disjoint
        for k in sizes:
            assert r[k] % 256 == 0 and r[k] + sizes[k] <= n
    with pytest.raises(moe.MoeError):
        moe.workspace_regions(moe.Desc(T=1, H=33, E=4, I=32, top_k=1))


def test_backward_argument_checks_host_only(L):
    """Invalid sizes, null pointers and overlapping outputs are rejected before any CUDA call."""
    from mixture_experts_ffn_07_b200 import _lib as moe
    inv = moe.MOE_ERR_INVALID_ARG
    a, b, c, d, e = 1 << 20, 2 << 20, 3 << 20, 4 << 20, 5 << 20  # disjoint fake addresses, never dereferenced
    assert L.moe_combine_backward(-1, 8, 16, a, b, c, d, e, None) == inv
    assert L.moe_combine_backward(4, 0, 16, a, b, c, d, e, None) == inv
    assert L.moe_combine_backward(4, 8, 0, a, b, c, d, e, None) == inv
    assert L.moe_combine_backward(1 << 31, 1, 1, a, b, c, d, e, None) == inv
    assert L.moe_combine_backward(1 << 20, 1 << 14, 1, a, b, c, d, e, None) == inv  # T*K beyond the grid
    assert L.moe_combine_backward(4, 8, 16, None, b, c, d, e, None) == inv
    assert L.moe_combine_backward(4, 8, 16, a, b, c, a, e, None) == inv  # d_y over y
    assert L.moe_combine_backward(4, 8, 16, a, b, c, d, c + 4, None) == inv  # d_w inside d_out
    assert L.moe_combine_backward(4, 8, 16, a, b, c, d, d + 64, None) == inv  # d_w inside d_y
    assert L.moe_combine_backward(0, 8, 16, None, None, None, None, None, None) == moe.MOE_OK
    assert L.moe_act_up_backward(-1, 16, 0, a, b, c, None) == inv
    assert L.moe_act_up_backward(4, 0, 0, a, b, c, None) == inv
    assert L.moe_act_up_backward(4, 16, 7, a, b, c, None) == inv
    assert L.moe_act_up_backward(4, 16, 0, a, None, c, None) == inv
    assert L.moe_act_up_backward(4, 16, 0, a, b, a + 8, None) == inv  # d_gate_up over gate_up
    assert L.moe_act_up_backward(4, 16, 1, a, b, b, None) == inv  # d_gate_up over d_h
    assert L.moe_act_up_backward(0, 16, 0, None, None, None, None) == moe.MOE_OK
