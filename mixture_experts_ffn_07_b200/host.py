"""Host-side conveniences: move numpy weights/activations to the device in the
layouts include/moe.h expects, and run one call.  Argument marshalling only.

`upload(src)` takes any object with the attributes of a layer invocation
(``spec`` with T, H, E, I, K, act, renormalize, act_dtype, w_dtype,
router_dtype, shared_I; arrays x, router, router_bias, gate, up, down,
sh_gate, sh_up, sh_down, sh_gate_w).  bf16 arrays are uint16 bit patterns;
Q8_0 weights are GGML blocks and are split on the device by moe_q8_0_split;
Q4_K blocks are used in place and Q6_K blocks are split by moe_q6_k_split.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (Desc, Weights, last_device_status, layer, q6_k_split, q6_k_srow_bytes, q8_0_split, route,
               workspace_bytes, MOE_OK)


def to_device(a: np.ndarray, dtype: str) -> torch.Tensor:
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()
    raise ValueError(dtype)


def split_q8_0(blocks: np.ndarray, rows: int, cols: int):
    b = torch.from_numpy(np.ascontiguousarray(blocks).reshape(-1)).cuda()
    q = torch.empty((rows, cols), dtype=torch.int8, device="cuda")
    s = torch.empty((rows, cols // 32), dtype=torch.float16, device="cuda")
    q8_0_split(b, rows, cols, q, s)
    return q, s


def split_q6_k(blocks: np.ndarray, rows: int, cols: int):
    b = torch.from_numpy(np.ascontiguousarray(blocks).reshape(-1)).cuda()
    q = torch.empty((rows, cols // 256, 192), dtype=torch.uint8, device="cuda")
    s = torch.empty((rows, q6_k_srow_bytes(cols)), dtype=torch.uint8, device="cuda")
    q6_k_split(b, rows, cols, q, s)
    return q, s


def upload(src):
    s = src.spec
    desc = Desc(T=s.T, H=s.H, E=s.E, I=s.I, top_k=s.K, act=s.act, renormalize=s.renormalize,
                act_dtype=s.act_dtype, w_dtype=s.w_dtype, router_dtype=s.router_dtype,
                has_router_bias=src.router_bias is not None, shared_I=s.shared_I,
                has_shared_gate=src.sh_gate_w is not None, gating=getattr(s, "gating", "softmax"),
                n_groups=getattr(s, "n_groups", 1), topk_groups=getattr(s, "topk_groups", 1))
    w = Weights(router=to_device(src.router, s.router_dtype))
    if src.router_bias is not None:
        w.router_bias = torch.from_numpy(np.asarray(src.router_bias, np.float32)).cuda()
    mats = [("gate", src.gate, s.E * s.I, s.H), ("up", src.up, s.E * s.I, s.H), ("down", src.down, s.E * s.H, s.I)]
    if s.shared_I:
        mats += [("sh_gate", src.sh_gate, s.shared_I, s.H), ("sh_up", src.sh_up, s.shared_I, s.H),
                 ("sh_down", src.sh_down, s.H, s.shared_I)]
        if src.sh_gate_w is not None:
            w.sh_gate_w = to_device(src.sh_gate_w, s.router_dtype)
    for name, a, rows, cols in mats:
        if s.w_dtype == "q8_0":
            q, sc = split_q8_0(a, rows, cols)
            setattr(w, name, q)
            setattr(w, name + "_scale", sc)
        elif s.w_dtype == "q4_k_q6_k" and name in ("down", "sh_down"):
            q, sc = split_q6_k(a, rows, cols)
            setattr(w, name, q)
            setattr(w, name + "_scale", sc)
        elif s.w_dtype in ("q4_k", "q4_k_q6_k"):
            setattr(w, name, torch.from_numpy(np.ascontiguousarray(a).reshape(-1)).cuda())
        else:
            setattr(w, name, to_device(a, s.w_dtype))
    x = to_device(src.x, s.act_dtype)
    return desc, w, x


def run_layer(desc, w, x):
    """One moe_layer call on fresh buffers; the output starts as NaN and every workspace byte as 0xFF (NaN as
    f32), so a row read before it is written, or an output never written, shows in the result."""
    out = torch.full((desc.T, desc.H), float("nan"), dtype=x.dtype, device="cuda")
    ws = torch.full((max(workspace_bytes(desc), 256),), 0xFF, dtype=torch.uint8, device="cuda")
    layer(desc, x, w, out, ws)
    torch.cuda.synchronize()
    st = last_device_status()
    if st != MOE_OK:
        raise RuntimeError(f"device status {st}")
    return out


def run_route(desc, w, x):
    T, E, K = desc.T, desc.E, desc.top_k
    logits = torch.empty((T, E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, K), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, K), dtype=torch.float32, device="cuda")
    sg = torch.empty((max(T, 1),), dtype=torch.float32, device="cuda")
    ws = torch.empty(max(workspace_bytes(desc), 256), dtype=torch.uint8, device="cuda")
    route(desc, x, w, logits, ids, tw, sg if desc.has_shared_gate and desc.shared_I else None, ws)
    torch.cuda.synchronize()
    return logits, ids, tw, sg
