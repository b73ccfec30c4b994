"""ORACLE for the MoE FFN layer -- test infrastructure only.

A thin ctypes wrapper over ``oracle.c`` (plain C, f64 accumulation, OpenMP over
tokens).  Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU
baseline may import this package; the product library never does.  It imports
nothing from the product package or from the CUDA sources: callers hand it
plain numpy arrays (bf16 as uint16 bit patterns, Q8_0 as GGML blocks).

Every function is pinned by ``tests/test_oracle_pins.py`` against closed forms,
brute force and the worked values the pages print.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "liboracle.so")
_SRC = os.path.join(_HERE, "oracle.c")

DTYPE = {"f32": 0, "bf16": 1, "q8_0": 2, "q4_k": 3, "q4_k_q6_k": 4, "q6_k": 5}
# bytes of one stored block and the values it holds, for the block formats
BLOCK = {"q8_0": (34, 32), "q4_k": (144, 256), "q6_k": (210, 256)}
ACT = {"silu": 0, "gelu_tanh": 1}


def build(force: bool = False) -> str:
    """Compile oracle.c (gcc -O2, strict IEEE: no -ffast-math, so sums keep loop order)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class _Desc(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("H", ctypes.c_int64), ("E", ctypes.c_int64), ("I", ctypes.c_int64),
                ("K", ctypes.c_int64), ("act", ctypes.c_int32), ("renormalize", ctypes.c_int32),
                ("act_dtype", ctypes.c_int32), ("w_dtype", ctypes.c_int32), ("router_dtype", ctypes.c_int32),
                ("has_router_bias", ctypes.c_int32), ("shared_I", ctypes.c_int64),
                ("has_shared_gate", ctypes.c_int32), ("gating", ctypes.c_int32), ("n_groups", ctypes.c_int64),
                ("topk_groups", ctypes.c_int64)]


class _Route(ctypes.Structure):
    _fields_ = [("E", ctypes.c_int64), ("K", ctypes.c_int64), ("renorm", ctypes.c_int), ("gating", ctypes.c_int),
                ("n_groups", ctypes.c_int64), ("topk_groups", ctypes.c_int64)]


GATING = {"softmax": 0, "sigmoid": 1}


class _Tensors(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("x", "router", "bias", "gate", "up", "down", "sh_gate", "sh_up", "sh_down", "sh_gate_w")]


_lib_handle = None


def bind(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    lib.ora_fp16_to_double.argtypes = [ctypes.c_uint16]
    lib.ora_fp16_to_double.restype = ctypes.c_double
    lib.ora_act.argtypes = [i32, ctypes.c_double]
    lib.ora_act.restype = ctypes.c_double
    lib.ora_sigmoid.argtypes = [ctypes.c_double]
    lib.ora_sigmoid.restype = ctypes.c_double
    lib.ora_select.argtypes = [p, i64, p, p, p]
    lib.ora_weights_for.argtypes = [p, i64, p, p, p]
    lib.ora_permute.argtypes = [p, i64, i64, p, p, p, p]
    lib.ora_permute.restype = i32
    lib.ora_expert.argtypes = [p, p, i64, i64, p]
    lib.ora_layer.argtypes = [p, p, p, i64, p, p, p, p, p, p, p]
    lib.ora_logits.argtypes = [p, p, p, i64, p, p]
    lib.ora_shared.argtypes = [p, p, p, i64, p, p]
    lib.ora_load_rows.argtypes = [p, i32, i64, i64, i64, p]
    lib.ora_act_array.argtypes = [i32, p, i64, p]
    lib.ora_act_grad.argtypes = [i32, ctypes.c_double]
    lib.ora_act_grad.restype = ctypes.c_double
    lib.ora_combine_backward.argtypes = [p, p, p, i64, i64, i64, p, p]
    lib.ora_act_up_backward.argtypes = [i32, p, p, i64, i64, p]
    lib.ora_threads.restype = i32
    lib.ora_set_threads.argtypes = [i32]
    for f in (lib.ora_select, lib.ora_weights_for, lib.ora_expert, lib.ora_layer, lib.ora_logits,
              lib.ora_shared, lib.ora_load_rows, lib.ora_act_array, lib.ora_set_threads, lib.ora_combine_backward,
              lib.ora_act_up_backward):
        f.restype = None
    return lib


def _lib():
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = bind(ctypes.CDLL(build()))
    return _lib_handle


@dataclass
class Layer:
    """Sizes, formats and host tensors of one layer invocation, as the oracle reads them."""
    T: int
    H: int
    E: int
    I: int
    K: int
    act: str
    renormalize: bool
    act_dtype: str
    w_dtype: str
    router_dtype: str
    x: np.ndarray
    router: np.ndarray
    gate: np.ndarray
    up: np.ndarray
    down: np.ndarray
    bias: np.ndarray | None = None
    shared_I: int = 0
    sh_gate: np.ndarray | None = None
    sh_up: np.ndarray | None = None
    sh_down: np.ndarray | None = None
    sh_gate_w: np.ndarray | None = None
    gating: str = "softmax"
    n_groups: int = 1
    topk_groups: int = 1

    def _c(self):
        d = _Desc(self.T, self.H, self.E, self.I, self.K, ACT[self.act], int(self.renormalize),
                  DTYPE[self.act_dtype], DTYPE[self.w_dtype], DTYPE[self.router_dtype],
                  int(self.bias is not None), self.shared_I, int(self.sh_gate_w is not None), GATING[self.gating],
                  self.n_groups, self.topk_groups)
        keep = []

        def ptr(a, dt=None):
            if a is None:
                return None
            a = np.ascontiguousarray(a if dt is None else a.astype(dt))
            keep.append(a)
            return a.ctypes.data

        t = _Tensors(ptr(self.x), ptr(self.router), ptr(self.bias, np.float32), ptr(self.gate), ptr(self.up),
                     ptr(self.down), ptr(self.sh_gate), ptr(self.sh_up), ptr(self.sh_down), ptr(self.sh_gate_w))
        return d, t, keep


def from_workload(wl) -> Layer:
    """Adapter from a ``workloads.Workload`` (plain arrays + sizes) to the oracle's own record."""
    s = wl.spec
    return Layer(T=s.T, H=s.H, E=s.E, I=s.I, K=s.K, act=s.act, renormalize=s.renormalize, act_dtype=s.act_dtype,
                 w_dtype=s.w_dtype, router_dtype=s.router_dtype, x=wl.x, router=wl.router, gate=wl.gate, up=wl.up,
                 down=wl.down, bias=wl.router_bias, shared_I=s.shared_I, sh_gate=wl.sh_gate, sh_up=wl.sh_up,
                 sh_down=wl.sh_down, sh_gate_w=wl.sh_gate_w, gating=getattr(s, "gating", "softmax"),
                 n_groups=getattr(s, "n_groups", 1), topk_groups=getattr(s, "topk_groups", 1))


def _tok(tokens, n_default):
    if tokens is None:
        return None, n_default
    tk = np.ascontiguousarray(tokens, np.int64)
    return tk, len(tk)


def layer(L: Layer, tokens=None, force_ids=None):
    """Full layer on a token list. Returns dict(out[n,H], logits[n,E], ids[n,K], w[n,K], gate_s[n], absmax[n])."""
    tk, n = _tok(tokens, L.T)
    d, t, keep = L._c()
    out = np.zeros((n, L.H), np.float64)
    logits = np.zeros((n, L.E), np.float64)
    ids = np.zeros((n, L.K), np.int32)
    w = np.zeros((n, L.K), np.float64)
    gs = np.zeros((n,), np.float64)
    am = np.zeros((n,), np.float64)
    fi = None
    if force_ids is not None:
        fi = np.ascontiguousarray(force_ids, np.int32).reshape(n, L.K)
    _lib().ora_layer(ctypes.byref(d), ctypes.byref(t), None if tk is None else tk.ctypes.data, n,
                     None if fi is None else fi.ctypes.data, out.ctypes.data, logits.ctypes.data, ids.ctypes.data,
                     w.ctypes.data, gs.ctypes.data, am.ctypes.data)
    return dict(out=out, logits=logits, ids=ids, w=w, gate_s=gs, absmax=am)


def logits(L: Layer, tokens=None):
    tk, n = _tok(tokens, L.T)
    d, t, keep = L._c()
    out = np.zeros((n, L.E), np.float64)
    am = np.zeros((n,), np.float64)
    _lib().ora_logits(ctypes.byref(d), ctypes.byref(t), None if tk is None else tk.ctypes.data, n,
                      out.ctypes.data, am.ctypes.data)
    return out, am


def select(logit_rows: np.ndarray, K: int, renormalize: bool = True, gating: str = "softmax", n_groups: int = 1,
           topk_groups: int = 1):
    """Selection (l desc, e asc; first K, among the topk_groups best of n_groups groups) and weights from given
    logits [n,E] (any float dtype, widened exactly)."""
    l = np.ascontiguousarray(logit_rows, np.float64)
    n, E = l.shape
    ids = np.zeros((n, K), np.int32)
    w = np.zeros((n, K), np.float64)
    r = _Route(E, K, int(renormalize), GATING[gating], n_groups, topk_groups)
    _lib().ora_select(l.ctypes.data, n, ctypes.byref(r), ids.ctypes.data, w.ctypes.data)
    return ids, w


def weights_for(logit_rows: np.ndarray, ids: np.ndarray, renormalize: bool = True, gating: str = "softmax"):
    l = np.ascontiguousarray(logit_rows, np.float64)
    n, E = l.shape
    ids = np.ascontiguousarray(ids, np.int32)
    K = ids.shape[1]
    w = np.zeros((n, K), np.float64)
    r = _Route(E, K, int(renormalize), GATING[gating], 1, 1)
    _lib().ora_weights_for(l.ctypes.data, n, ctypes.byref(r), ids.ctypes.data, w.ctypes.data)
    return w


def permute(ids: np.ndarray, E: int):
    """Counting-sort permutation of pair ids by expert: counts[E], offsets[E+1], sorted_pairs[P], pair_pos[P]."""
    f = np.ascontiguousarray(ids, np.int32).reshape(-1)
    P = f.size
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    sp = np.zeros(P, np.int32)
    pp = np.zeros(P, np.int32)
    rc = _lib().ora_permute(f.ctypes.data, P, E, counts.ctypes.data, offsets.ctypes.data, sp.ctypes.data,
                            pp.ctypes.data)
    if rc != 0:
        raise ValueError("expert id out of range")
    return counts, offsets, sp, pp


def expert(L: Layer, t: int, e: int) -> np.ndarray:
    d, tt, keep = L._c()
    y = np.zeros(L.H, np.float64)
    _lib().ora_expert(ctypes.byref(d), ctypes.byref(tt), t, e, y.ctypes.data)
    return y


def shared(L: Layer, tokens=None):
    """Shared expert alone (already scaled by its sigmoid gate when gated): y[n,H], gate_s[n]."""
    tk, n = _tok(tokens, L.T)
    d, t, keep = L._c()
    y = np.zeros((n, L.H), np.float64)
    gs = np.zeros((n,), np.float64)
    _lib().ora_shared(ctypes.byref(d), ctypes.byref(t), None if tk is None else tk.ctypes.data, n, y.ctypes.data,
                      gs.ctypes.data)
    return y, gs


def load_rows(a: np.ndarray, dtype: str, cols: int, r0: int = 0, n: int | None = None) -> np.ndarray:
    """Rows of a stored matrix widened to f64 (dequantising Q8_0, Q4_K or Q6_K blocks)."""
    a = np.ascontiguousarray(a)
    if n is None:
        if dtype in BLOCK:
            nb, nv = BLOCK[dtype]
            n = a.nbytes // (cols // nv * nb)
        else:
            n = a.size // cols
    out = np.zeros((n, cols), np.float64)
    _lib().ora_load_rows(a.ctypes.data, DTYPE[dtype], r0, n, cols, out.ctypes.data)
    return out


def act(name: str, g) -> np.ndarray:
    g = np.ascontiguousarray(np.atleast_1d(g), np.float64)
    out = np.zeros_like(g)
    _lib().ora_act_array(ACT[name], g.ctypes.data, g.size, out.ctypes.data)
    return out


def act_grad(name: str, g: float) -> float:
    """Derivative of the activation at g (backward of act * up)."""
    return _lib().ora_act_grad(ACT[name], g)


def combine_backward(y: np.ndarray, w: np.ndarray, d_out: np.ndarray):
    """Backward of out[t] = sum_k w[t,k] y[t,k]: y[T,K,H], w[T,K], d_out[T,H] (f32) -> d_y[T,K,H], d_w[T,K] (f64)."""
    y = np.ascontiguousarray(y, np.float32)
    w = np.ascontiguousarray(w, np.float32)
    d_out = np.ascontiguousarray(d_out, np.float32)
    T, K, H = y.shape
    assert w.shape == (T, K) and d_out.shape == (T, H)
    d_y = np.zeros((T, K, H), np.float64)
    d_w = np.zeros((T, K), np.float64)
    _lib().ora_combine_backward(y.ctypes.data, w.ctypes.data, d_out.ctypes.data, T, K, H, d_y.ctypes.data,
                                d_w.ctypes.data)
    return d_y, d_w


def act_up_backward(act_name: str, gate_up: np.ndarray, d_h: np.ndarray) -> np.ndarray:
    """Backward of h = act(gate) * up: gate_up[P, 2I] ([gate | up]), d_h[P, I] (f32) -> d_gate_up[P, 2I] (f64)."""
    gu = np.ascontiguousarray(gate_up, np.float32)
    dh = np.ascontiguousarray(d_h, np.float32)
    P, I2 = gu.shape
    I = I2 // 2
    assert I2 == 2 * I and dh.shape == (P, I)
    out = np.zeros((P, 2 * I), np.float64)
    _lib().ora_act_up_backward(ACT[act_name], gu.ctypes.data, dh.ctypes.data, P, I, out.ctypes.data)
    return out


def sigmoid(z: float) -> float:
    return _lib().ora_sigmoid(z)


def fp16_to_double(bits: int) -> float:
    return _lib().ora_fp16_to_double(bits)


def threads() -> int:
    return _lib().ora_threads()


def set_threads(n: int) -> None:
    _lib().ora_set_threads(n)
