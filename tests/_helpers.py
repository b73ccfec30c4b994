"""Small numpy helpers shared by the tests (no step of the layer lives here)."""
from __future__ import annotations

import numpy as np


def widen(a: np.ndarray, dtype: str, cols: int | None = None) -> np.ndarray:
    """Stored tensor -> float64 with numpy only (bf16 bit patterns, Q8_0 GGML blocks, f32)."""
    if dtype == "f32":
        return np.asarray(a, np.float32).astype(np.float64)
    if dtype == "bf16":
        return (np.asarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "q8_0":
        b = np.asarray(a, np.uint8)
        lead = b.shape[:-2]
        nb = b.shape[-2]
        d = b[..., 0:2].copy().view(np.float16).astype(np.float64)        # [..., nb, 1]
        q = b[..., 2:34].copy().view(np.int8).astype(np.float64)           # [..., nb, 32]
        return (d * q).reshape(*lead, nb * 32)
    raise ValueError(dtype)


def silu(g):
    return g / (1.0 + np.exp(-g))


def gelu_tanh(g):
    return 0.5 * g * (1.0 + np.tanh(np.sqrt(2.0 / np.pi) * (g + 0.044715 * g ** 3)))


ACTS = {"silu": silu, "gelu_tanh": gelu_tanh}


def numpy_layer(L) -> dict:
    """An independent restatement of the layer with numpy matmuls, for tiny inputs.

    Selection uses Python's stable sort with key (-logit, expert); weights are
    written with math from the definition; the expert FFN uses matrix products
    in the out x in orientation.
    """
    x = widen(L.x, L.act_dtype)
    Wr = widen(L.router, L.router_dtype)
    g = widen(L.gate, L.w_dtype).reshape(L.E, L.I, L.H)
    u = widen(L.up, L.w_dtype).reshape(L.E, L.I, L.H)
    dn = widen(L.down, L.w_dtype).reshape(L.E, L.H, L.I)
    act = ACTS[L.act]
    logits = x @ Wr.T
    if L.bias is not None:
        logits = logits + np.asarray(L.bias, np.float64)[None, :]
    out = np.zeros((L.T, L.H))
    ids = np.zeros((L.T, L.K), np.int32)
    ws = np.zeros((L.T, L.K))
    for t in range(L.T):
        l = logits[t]
        order = sorted(range(L.E), key=lambda e: (-l[e], e))[: L.K]
        p = np.exp(l - l.max())
        p = p / p.sum()
        w = p[order]
        if L.renormalize:
            w = w / w.sum()
        ids[t] = order
        ws[t] = w
        for k, e in enumerate(order):
            a = act(g[e] @ x[t]) * (u[e] @ x[t])
            out[t] += w[k] * (dn[e] @ a)
    if L.shared_I > 0:
        sg = widen(L.sh_gate, L.w_dtype).reshape(L.shared_I, L.H)
        su = widen(L.sh_up, L.w_dtype).reshape(L.shared_I, L.H)
        sd = widen(L.sh_down, L.w_dtype).reshape(L.H, L.shared_I)
        a = act(x @ sg.T) * (x @ su.T)
        y = a @ sd.T
        if L.sh_gate_w is not None:
            s = 1.0 / (1.0 + np.exp(-(x @ widen(L.sh_gate_w, L.router_dtype))))
            y = y * s[:, None]
        out += y
    return dict(out=out, logits=logits, ids=ids, w=ws)
