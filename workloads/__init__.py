"""Seeded synthetic workloads for the MoE FFN layer.

The arrays made here are the only thing the CUDA path and the f64 oracle
share.  Nothing in this package computes any step of the layer: it draws
numbers (``gen.c``: splitmix64 + Box-Muller, counter based) and rounds them to
the storage formats the layer reads.

Named configurations follow the five workloads the layer is measured on:

=====================  =====  ====  ===  ====  =  =========  =====  ===========
name                   T      H     E    I     K  act        dtype  shared
=====================  =====  ====  ===  ====  =  =========  =====  ===========
decode_f32_t1          1      2816  128  704   8  gelu_tanh  f32    none
prefill_bf16_t512      512    2048  64   1024  8  silu       bf16   none
routed_shared_t4096    4096   2048  256  512   8  silu       bf16   512, gated
skewed_zipf_t8192      8192   7168  256  2048  8  silu       bf16   2048, ungated
q8_0_decode_t16        16     2048  128  768   8  silu       Q8_0   none
=====================  =====  ====  ===  ====  =  =========  =====  ===========

Distributions: x ~ N(0,1); router W and the shared-gate vector w_s ~ N(0,0.02)
(second parameter = standard deviation); expert and shared projections
~ N(0, 1/sqrt(fan_in)); Q8_0 blocks q ~ U{-127..127}, d ~ U[0.001,0.01] rounded
to fp16; Q4_K / Q6_K blocks with every quant, scale and min byte uniform over
0..255 and fp16 d ~ U[1e-4, 2e-4], dmin ~ U[7.5e-4, 1.5e-3] (Q4_K) or
d ~ U[2e-5, 4e-5] (Q6_K, fp16 subnormals included); bf16 tensors are rounded to nearest-even from the f32 samples.  The
skewed workload adds a per-expert router bias b_e = 2 ln p_r with Zipf(s=1.1)
rank r = e + 1 over the 256 experts.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "libmoegen.so")
_SRC = os.path.join(_HERE, "gen.c")

F32, BF16, Q8_0 = "f32", "bf16", "q8_0"
Q4_K, Q4_K_Q6_K = "q4_k", "q4_k_q6_k"   # all projections Q4_K; gate/up Q4_K with down Q6_K
SILU, GELU_TANH = "silu", "gelu_tanh"


def build(force: bool = False) -> str:
    """Compile gen.c into libmoegen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


_lib_handle = None


def _lib():
    global _lib_handle
    if _lib_handle is None:
        lib = ctypes.CDLL(build())
        u64, i64, d, p = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.gen_normal_f32.argtypes = [u64, u64, d, d, i64, p]
        lib.gen_normal_bf16.argtypes = [u64, u64, d, d, i64, p]
        lib.gen_uniform_f32.argtypes = [u64, u64, d, d, i64, p]
        lib.gen_q8_0_blocks.argtypes = [u64, u64, i64, i64, ctypes.c_int, ctypes.c_int, d, d, p]
        lib.round_f32_to_bf16.argtypes = [p, i64, p]
        for f in (lib.gen_normal_f32, lib.gen_normal_bf16, lib.gen_uniform_f32, lib.gen_q8_0_blocks,
                  lib.round_f32_to_bf16):
            f.restype = None
        _lib_handle = lib
    return _lib_handle


def normal(seed: int, stream: int, shape, std: float, dtype: str, mean: float = 0.0) -> np.ndarray:
    n = int(np.prod(shape))
    if dtype == F32:
        out = np.empty(n, np.float32)
        _lib().gen_normal_f32(seed, stream, mean, std, n, out.ctypes.data)
    elif dtype == BF16:
        out = np.empty(n, np.uint16)
        _lib().gen_normal_bf16(seed, stream, mean, std, n, out.ctypes.data)
    else:
        raise ValueError(dtype)
    return out.reshape(shape)


def uniform(seed: int, stream: int, shape, lo: float, hi: float) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, np.float32)
    _lib().gen_uniform_f32(seed, stream, lo, hi, n, out.ctypes.data)
    return out.reshape(shape)


def q8_0_blocks(seed: int, stream: int, shape, q_lo=-127, q_hi=127, d_lo=0.001, d_hi=0.01) -> np.ndarray:
    """GGML Q8_0 blocks for a weight of logical shape (..., rows, cols): uint8 [..., rows, cols/32, 34]."""
    *lead, rows, cols = shape
    assert cols % 32 == 0
    nrows = int(np.prod(lead, dtype=np.int64)) * rows
    out = np.empty((nrows * (cols // 32) * 34,), np.uint8)
    _lib().gen_q8_0_blocks(seed, stream, nrows, cols, q_lo, q_hi, d_lo, d_hi, out.ctypes.data)
    return out.reshape(*lead, rows, cols // 32, 34)


def _bytes(seed, stream, n):
    u = uniform(seed, stream, (n,), 0.0, 256.0)
    return np.minimum(np.floor(u), 255).astype(np.uint8)


def _fp16_bits(seed, stream, n, lo, hi):
    return uniform(seed, stream, (n,), lo, hi).astype(np.float16).view(np.uint8).reshape(n, 2)


def kquant_blocks(seed: int, stream: int, shape, fmt: str, d=(1e-4, 2e-4), dmin=(7.5e-4, 1.5e-3)) -> np.ndarray:
    """GGML Q4_K (144-byte) or Q6_K (210-byte) blocks of 256 values for a weight of logical shape
    (..., rows, cols): uint8 [..., rows, cols/256, nbytes].  Every quant, scale and min byte is uniform
    over 0..255; the fp16 super-block scale d (and Q4_K's dmin) are uniform over the given ranges."""
    *lead, rows, cols = shape
    assert cols % 256 == 0
    nblk = int(np.prod(lead, dtype=np.int64)) * rows * (cols // 256)
    if fmt == Q4_K:
        b = np.empty((nblk, 144), np.uint8)
        b[:, 0:2] = _fp16_bits(seed, stream | 1 << 8, nblk, *d)
        b[:, 2:4] = _fp16_bits(seed, stream | 2 << 8, nblk, *dmin)
        b[:, 4:] = _bytes(seed, stream | 3 << 8, nblk * 140).reshape(nblk, 140)
    elif fmt == "q6_k":
        b = np.empty((nblk, 210), np.uint8)
        b[:, :208] = _bytes(seed, stream | 3 << 8, nblk * 208).reshape(nblk, 208)
        b[:, 208:210] = _fp16_bits(seed, stream | 1 << 8, nblk, *d)
    else:
        raise ValueError(fmt)
    return b.reshape(*lead, rows, cols // 256, b.shape[1])


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    _lib().round_f32_to_bf16(a.ctypes.data, a.size, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(a, np.uint16).astype(np.uint32) << 16).view(np.float32)


def zipf_log_bias(E: int, s: float = 1.1, scale: float = 2.0) -> np.ndarray:
    """b_e = scale * ln p_r, p_r = r^-s / sum_j j^-s, r = e + 1 (input recipe of the skewed workload)."""
    r = np.arange(1, E + 1, dtype=np.float64)
    w = r ** (-s)
    return (scale * np.log(w / w.sum())).astype(np.float32)


@dataclass
class Spec:
    """Sizes and formats of one MoE layer invocation."""
    T: int
    H: int
    E: int
    I: int
    K: int
    act: str = SILU
    act_dtype: str = BF16
    w_dtype: str = BF16
    router_dtype: str = BF16
    renormalize: bool = True
    shared_I: int = 0
    shared_gated: bool = False
    router_bias: str | None = None     # None | "zipf1.1"
    router_std: float = 0.02
    name: str = "custom"
    gating: str = "softmax"            # "softmax" | "sigmoid"
    n_groups: int = 1                  # group-limited selection when > 1
    topk_groups: int = 1

    @property
    def P(self) -> int:
        return self.T * self.K


CONFIGS = {
    "decode_f32_t1": Spec(T=1, H=2816, E=128, I=704, K=8, act=GELU_TANH, act_dtype=F32, w_dtype=F32,
                          router_dtype=F32, name="decode_f32_t1"),
    "prefill_bf16_t512": Spec(T=512, H=2048, E=64, I=1024, K=8, name="prefill_bf16_t512"),
    "routed_shared_t4096": Spec(T=4096, H=2048, E=256, I=512, K=8, shared_I=512, shared_gated=True,
                                name="routed_shared_t4096"),
    "skewed_zipf_t8192": Spec(T=8192, H=7168, E=256, I=2048, K=8, shared_I=2048, shared_gated=False,
                              router_bias="zipf1.1", name="skewed_zipf_t8192"),
    "q8_0_decode_t16": Spec(T=16, H=2048, E=128, I=768, K=8, act_dtype=F32, w_dtype=Q8_0, router_dtype=F32,
                            name="q8_0_decode_t16"),
    # routing variants on the prefill shapes: sigmoid gating, 8 groups of 8 experts, 4 groups kept
    "grouped_sigmoid_t512": Spec(T=512, H=2048, E=64, I=1024, K=8, gating="sigmoid", n_groups=8, topk_groups=4,
                                 name="grouped_sigmoid_t512"),
    # Q8_0-decode shapes with the k-quant stacks of the Metal MoE providers: gate/up Q4_K, down Q6_K
    "q4k_q6k_decode_t16": Spec(T=16, H=2048, E=128, I=768, K=8, act_dtype=F32, w_dtype=Q4_K_Q6_K, router_dtype=F32,
                               name="q4k_q6k_decode_t16"),
    # the skewed layer's expert shapes (H=7168, I=2048) with every token on all 8 experts: 2048 rows per expert,
    # a few GB on the device, for profiling the expert GEMMs where they are tensor bound
    "gemm_h7168_i2048_e8_t2048": Spec(T=2048, H=7168, E=8, I=2048, K=8, name="gemm_h7168_i2048_e8_t2048"),
}
CONFIG_ORDER = list(CONFIGS)
BASE_SEED = 0xB2000000


def config_seed(name: str) -> int:
    return BASE_SEED + CONFIG_ORDER.index(name) if name in CONFIG_ORDER else BASE_SEED + 0x100


@dataclass
class Workload:
    spec: Spec
    seed: int
    x: np.ndarray
    router: np.ndarray
    router_bias: np.ndarray | None
    gate: np.ndarray
    up: np.ndarray
    down: np.ndarray
    sh_gate: np.ndarray | None = None
    sh_up: np.ndarray | None = None
    sh_down: np.ndarray | None = None
    sh_gate_w: np.ndarray | None = None
    extra: dict = field(default_factory=dict)


# stream ids of the tensors of one workload
S_X, S_ROUTER, S_GATE, S_UP, S_DOWN, S_SH_GATE, S_SH_UP, S_SH_DOWN, S_SH_GATE_W = range(1, 10)
S_X_ALT = 64  # streams S_X_ALT + i: further token batches of a config


def _weight(seed, stream, shape, fan_in, w_dtype, down=False):
    if w_dtype == Q8_0:
        return q8_0_blocks(seed, stream, shape)
    if w_dtype in (Q4_K, Q4_K_Q6_K):
        if down and w_dtype == Q4_K_Q6_K:  # |d sc (q - 32)| ~ d * 74 * 18.5: about 1/sqrt(I) for I = 768
            return kquant_blocks(seed, stream, shape, "q6_k", d=(2e-5, 4e-5))
        return kquant_blocks(seed, stream, shape, Q4_K)
    return normal(seed, stream, shape, 1.0 / math.sqrt(fan_in), w_dtype)


def token_batch(spec: Spec, i: int, seed: int | None = None, x_std: float = 1.0) -> np.ndarray:
    """Token batch i of a config: 0 is the workload's own x, i > 0 further batches of the same
    distribution (benchmarks rotate over them so that consecutive steps route differently)."""
    if seed is None:
        seed = config_seed(spec.name)
    return normal(seed, S_X if i == 0 else S_X_ALT + i, (spec.T, spec.H), x_std, spec.act_dtype)


def make(spec: Spec, seed: int | None = None, x_std: float = 1.0) -> Workload:
    """Draw every input tensor of one layer invocation (host numpy arrays).

    bf16 tensors are returned as uint16 bit patterns; Q8_0 weights as uint8
    GGML blocks of shape [..., rows, cols/32, 34].
    """
    if seed is None:
        seed = config_seed(spec.name)
    T, H, E, I, Is = spec.T, spec.H, spec.E, spec.I, spec.shared_I
    x = token_batch(spec, 0, seed, x_std)
    router = normal(seed, S_ROUTER, (E, H), spec.router_std, spec.router_dtype)
    bias = zipf_log_bias(E) if spec.router_bias == "zipf1.1" else None
    gate = _weight(seed, S_GATE, (E, I, H), H, spec.w_dtype)
    up = _weight(seed, S_UP, (E, I, H), H, spec.w_dtype)
    down = _weight(seed, S_DOWN, (E, H, I), I, spec.w_dtype, down=True)
    wl = Workload(spec, seed, x, router, bias, gate, up, down)
    if Is > 0:
        wl.sh_gate = _weight(seed, S_SH_GATE, (Is, H), H, spec.w_dtype)
        wl.sh_up = _weight(seed, S_SH_UP, (Is, H), H, spec.w_dtype)
        wl.sh_down = _weight(seed, S_SH_DOWN, (H, Is), Is, spec.w_dtype, down=True)
        if spec.shared_gated:
            wl.sh_gate_w = normal(seed, S_SH_GATE_W, (H,), 0.02, spec.router_dtype)
    return wl
