"""MoE FFN layer for NVIDIA B200 -- Python binding of libmoe.so (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  Tensors are torch CUDA tensors (any object with ``data_ptr()``);
streams default to torch's current stream.  PyTorch provides device memory and
streams; it computes nothing here.

    desc = Desc(T=512, H=2048, E=64, I=1024, top_k=8)
    w = Weights(router=..., gate=..., up=..., down=...)
    ws = torch.empty(workspace_bytes(desc), dtype=torch.uint8, device="cuda")
    layer(desc, x, w, out, ws)
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass, fields

from . import _lib
from ._lib import (MOE_ACT_GELU_TANH, MOE_ACT_SILU, MOE_BF16, MOE_ERR_CUDA, MOE_ERR_DEVICE_INDEX,  # noqa: F401
                   MOE_ERR_INVALID_ARG, MOE_ERR_TIMEOUT, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_F32, MOE_OK,
                   MOE_Q4_K, MOE_Q4_K_Q6_K, MOE_Q8_0, MoeError, check, status_string)

DTYPES = {"f32": MOE_F32, "bf16": MOE_BF16, "q8_0": MOE_Q8_0, "q4_k": MOE_Q4_K, "q4_k_q6_k": MOE_Q4_K_Q6_K}
ACTS = {"silu": MOE_ACT_SILU, "gelu_tanh": MOE_ACT_GELU_TANH}
GATINGS = {"softmax": 0, "sigmoid": 1}  # moe_gating


@dataclass
class Desc:
    T: int
    H: int
    E: int
    I: int
    top_k: int
    act: str = "silu"
    renormalize: bool = True
    act_dtype: str = "bf16"
    w_dtype: str = "bf16"
    router_dtype: str = "bf16"
    has_router_bias: bool = False
    shared_I: int = 0
    has_shared_gate: bool = False
    gating: str = "softmax"
    n_groups: int = 0
    topk_groups: int = 0

    def c(self) -> _lib.MoeDesc:
        return _lib.MoeDesc(self.T, self.H, self.E, self.I, self.top_k, ACTS[self.act], int(self.renormalize),
                            DTYPES[self.act_dtype], DTYPES[self.w_dtype], DTYPES[self.router_dtype],
                            int(self.has_router_bias), self.shared_I, int(self.has_shared_gate),
                            GATINGS[self.gating], self.n_groups, self.topk_groups)

    @property
    def P(self) -> int:
        return self.T * self.top_k


@dataclass
class Weights:
    """Device tensors, out x in.  For Q8_0 the projections are int8 and *_scale hold fp16 block scales."""
    router: object = None
    router_bias: object = None
    gate: object = None
    up: object = None
    down: object = None
    sh_gate: object = None
    sh_up: object = None
    sh_down: object = None
    sh_gate_w: object = None
    gate_scale: object = None
    up_scale: object = None
    down_scale: object = None
    sh_gate_scale: object = None
    sh_up_scale: object = None
    sh_down_scale: object = None

    def c(self) -> _lib.MoeWeights:
        return _lib.MoeWeights(*[_ptr(getattr(self, f.name)) for f in fields(self)])


def _ptr(t):
    return None if t is None else t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def version() -> str:
    return _lib.lib().moe_version().decode()


def workspace_bytes(desc: Desc) -> int:
    d = desc.c()
    return _lib.lib().moe_workspace_bytes(ctypes.byref(d))


def workspace_regions(desc: Desc) -> dict:
    """moe_workspace_regions: byte offsets of the routing results moe_layer leaves in the workspace."""
    d, r = desc.c(), _lib.MoeWsRegions()
    check(_lib.lib().moe_workspace_regions(ctypes.byref(d), ctypes.byref(r)), "moe_workspace_regions")
    return {n: getattr(r, n) for n, _ in _lib.MoeWsRegions._fields_}


def route(desc, x, w, logits, topk_ids, topk_w, shared_gate=None, ws=None, stream=None):
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_route(ctypes.byref(d), _ptr(x), ctypes.byref(cw), _ptr(logits), _ptr(topk_ids),
                               _ptr(topk_w), _ptr(shared_gate), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_route")


def permute(desc, topk_ids, counts, offsets, sorted_pairs, pair_pos, stream=None):
    d = desc.c()
    check(_lib.lib().moe_permute(ctypes.byref(d), _ptr(topk_ids), _ptr(counts), _ptr(offsets), _ptr(sorted_pairs),
                                 _ptr(pair_pos), _stream(stream)), "moe_permute")


def expert_ffn(desc, x, w, offsets, sorted_pairs, topk_w, y_slots, ws, stream=None):
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_expert_ffn(ctypes.byref(d), _ptr(x), ctypes.byref(cw), _ptr(offsets), _ptr(sorted_pairs),
                                    _ptr(topk_w), _ptr(y_slots), _ptr(ws), _nbytes(ws), _stream(stream)),
          "moe_expert_ffn")


def combine(desc, y_slots, x, w, shared_gate, out, ws=None, stream=None):
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_combine(ctypes.byref(d), _ptr(y_slots), _ptr(x), ctypes.byref(cw), _ptr(shared_gate),
                                 _ptr(out), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_combine")


def layer(desc, x, w, out, ws, stream=None):
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_layer(ctypes.byref(d), _ptr(x), ctypes.byref(cw), _ptr(out), _ptr(ws), _nbytes(ws),
                               _stream(stream)), "moe_layer")


def layer_noalloc(desc, x, w, out, stream=None):
    """moe_layer with the library's static 32 MiB device scratch: for callers that cannot allocate.

    Calls that may overlap on the GPU share that scratch and race; the first call on a device
    looks up its address and should come before any stream capture."""
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_layer_noalloc(ctypes.byref(d), _ptr(x), ctypes.byref(cw), _ptr(out), _stream(stream)),
          "moe_layer_noalloc")


def layer_host(desc, x_host, w, out_host, x_dev, out_dev, ws, stream=None):
    """moe_layer with host x/out (pinned torch CPU tensors); copies are enqueued on `stream`."""
    d, cw = desc.c(), w.c()
    check(_lib.lib().moe_layer_host(ctypes.byref(d), _ptr(x_host), ctypes.byref(cw), _ptr(out_host), _ptr(x_dev),
                                    _ptr(out_dev), _ptr(ws), _nbytes(ws), _stream(stream)), "moe_layer_host")


def q8_0_split(blocks, rows, cols, q, scales, stream=None):
    check(_lib.lib().moe_q8_0_split(_ptr(blocks), rows, cols, _ptr(q), _ptr(scales), _stream(stream)),
          "moe_q8_0_split")


def combine_backward(y, w, d_out, d_y, d_w, stream=None):
    """moe_combine_backward: y [T,K,H] (unweighted expert outputs), w [T,K], d_out [T,H] -> d_y, d_w (all f32)."""
    T, K, H = y.shape
    check(_lib.lib().moe_combine_backward(T, K, H, _ptr(y), _ptr(w), _ptr(d_out), _ptr(d_y), _ptr(d_w),
                                          _stream(stream)), "moe_combine_backward")


def act_up_backward(act, gate_up, d_h, d_gate_up, stream=None):
    """moe_act_up_backward: gate_up [P,2I] ([gate | up]), d_h [P,I] -> d_gate_up [P,2I] (all f32)."""
    P, I = d_h.shape
    check(_lib.lib().moe_act_up_backward(P, I, ACTS[act] if isinstance(act, str) else act, _ptr(gate_up), _ptr(d_h),
                                         _ptr(d_gate_up), _stream(stream)), "moe_act_up_backward")


def q6_k_split(blocks, rows, cols, q, scales, stream=None):
    """moe_q6_k_split: GGML Q6_K blocks -> 16-byte aligned quant and scale planes."""
    check(_lib.lib().moe_q6_k_split(_ptr(blocks), rows, cols, _ptr(q), _ptr(scales), _stream(stream)),
          "moe_q6_k_split")


def q6_k_srow_bytes(cols: int) -> int:
    """Bytes of one scale row of the Q6_K split form (include/moe.h)."""
    return (cols // 256 * 18 + 15) // 16 * 16


def last_device_status(stream=None) -> int:
    return _lib.lib().moe_last_device_status(_stream(stream))


def launch_count() -> int:
    return _lib.lib().moe_launch_count()


def trace_enable(on: bool) -> None:
    _lib.lib().moe_trace_enable(int(on))


def trace_read(max_records: int = 4096):
    names = (ctypes.c_char_p * max_records)()
    ms = (ctypes.c_float * max_records)()
    n = _lib.lib().moe_trace_read(names, ms, max_records)
    return [(names[i].decode(), ms[i]) for i in range(min(n, max_records))]


def debug_set_wait_limit(cycles: int) -> None:
    _lib.lib().moe_debug_set_wait_limit(cycles)


def debug_set_skip_stage(enable: bool) -> None:
    _lib.lib().moe_debug_set_skip_stage(int(enable))


def debug_set_barrier_delay(cycles: int) -> None:
    """moe_debug_set_barrier_delay: CTA 0 of the cooperative kernels arrives late at its first grid barrier."""
    _lib.lib().moe_debug_set_barrier_delay(cycles)


def set_fused_front(enable: bool) -> None:
    """moe_set_fused_front: selection + permutation + row gather of the tensor-core
    path as one cooperative kernel (True, default) or three launches (False)."""
    _lib.lib().moe_set_fused_front(int(enable))


def set_pair_gemm(enable: bool) -> None:
    """moe_set_pair_gemm: full 256-row tiles of compute-bound expert GEMMs on CTA pairs
    (tcgen05.mma.cta_group::2, True, default) or every row on single CTAs (False)."""
    _lib.lib().moe_set_pair_gemm(int(enable))


def set_decode_stream(enable: bool) -> None:
    """moe_set_decode_stream: gate/up and down of the cooperative decode kernel for f32 / bf16 / Q8_0 weights
    as one TMA-fed stream of work items (True, default) or two phases with a grid barrier (False)."""
    _lib.lib().moe_set_decode_stream(int(enable))


def set_tma_gather(enable: bool) -> None:
    """moe_set_tma_gather: the routed gate/up GEMM gathers its x rows with the copy engine (True) or
    reads a copy of them in expert order (False, default); size workspaces after changing it."""
    _lib.lib().moe_set_tma_gather(int(enable))


def set_tensor_min_tokens(tokens: int) -> None:
    """moe_set_tensor_min_tokens: bf16 layers of at least `tokens` tokens take the tensor-core path
    (default 16); size workspaces after changing it."""
    _lib.lib().moe_set_tensor_min_tokens(int(tokens))


def set_fused_decode(enable: bool) -> None:
    """moe_set_fused_decode: one cooperative kernel (True, default) or step-by-step
    launches (False) for 1..64 tokens on the weight-streaming path."""
    _lib.lib().moe_set_fused_decode(int(enable))


def _nbytes(t) -> int:
    if t is None:
        return 0
    return t.numel() * t.element_size()
