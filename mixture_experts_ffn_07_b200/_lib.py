"""ctypes declarations of libmoe.so (include/moe.h).  Argument marshalling only.

Importing this module loads the library; it raises if ``libmoe.so`` has not
been built -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

# enums (include/moe.h)
MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_TIMEOUT, \
    MOE_ERR_DEVICE_INDEX = range(7)
MOE_F32, MOE_BF16, MOE_Q8_0, MOE_Q4_K, MOE_Q4_K_Q6_K = 0, 1, 2, 3, 4
MOE_NOALLOC_SCRATCH_BYTES = 32 << 20
MOE_ACT_SILU, MOE_ACT_GELU_TANH = 0, 1

# every symbol include/moe.h declares
EXPORTS = ("moe_status_string", "moe_version", "moe_workspace_bytes", "moe_route", "moe_permute", "moe_expert_ffn",
           "moe_combine", "moe_layer", "moe_layer_host", "moe_layer_noalloc", "moe_q8_0_split",
           "moe_last_device_status", "moe_launch_count", "moe_trace_enable", "moe_trace_read",
           "moe_debug_set_wait_limit", "moe_debug_set_skip_stage", "moe_set_fused_decode",
           "moe_workspace_regions", "moe_set_fused_front", "moe_set_pair_gemm", "moe_set_decode_stream", "moe_set_tma_gather", "moe_set_tensor_min_tokens", "moe_combine_backward", "moe_act_up_backward",
           "moe_q6_k_split", "moe_debug_set_barrier_delay")


class MoeDesc(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "H", "E", "I", "top_k", "act", "renormalize", "act_dtype", "w_dtype", "router_dtype",
                 "has_router_bias", "shared_I", "has_shared_gate", "gating", "n_groups", "topk_groups")]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("router", "router_bias", "gate", "up", "down", "sh_gate", "sh_up", "sh_down", "sh_gate_w",
                 "gate_scale", "up_scale", "down_scale", "sh_gate_scale", "sh_up_scale", "sh_down_scale")]


class MoeWsRegions(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in
                ("logits", "topk_ids", "topk_w", "shared_gate", "counts", "offsets", "sorted_pairs", "pair_pos")]


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} ({code})")


_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libmoe.so is not built ({LIB_PATH}); run mixture_experts_ffn_07_b200/build.py")
        L = ctypes.CDLL(LIB_PATH)
        P, S, DP, WP, I32, I64 = (ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(MoeDesc),
                                  ctypes.POINTER(MoeWeights), ctypes.c_int, ctypes.c_int64)
        L.moe_status_string.argtypes = [I32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_version.restype = ctypes.c_char_p
        L.moe_workspace_bytes.argtypes = [DP]
        L.moe_workspace_bytes.restype = S
        L.moe_route.argtypes = [DP, P, WP, P, P, P, P, P, S, P]
        L.moe_permute.argtypes = [DP, P, P, P, P, P, P]
        L.moe_expert_ffn.argtypes = [DP, P, WP, P, P, P, P, P, S, P]
        L.moe_combine.argtypes = [DP, P, P, WP, P, P, P, S, P]
        L.moe_layer.argtypes = [DP, P, WP, P, P, S, P]
        L.moe_layer_host.argtypes = [DP, P, WP, P, P, P, P, S, P]
        L.moe_layer_noalloc.argtypes = [DP, P, WP, P, P]
        L.moe_q8_0_split.argtypes = [P, I64, I64, P, P, P]
        L.moe_q6_k_split.argtypes = [P, I64, I64, P, P, P]
        L.moe_last_device_status.argtypes = [P]
        L.moe_combine_backward.argtypes = [I64, I64, I64, P, P, P, P, P, P]
        L.moe_act_up_backward.argtypes = [I64, I64, I32, P, P, P, P]
        for f in (L.moe_route, L.moe_permute, L.moe_expert_ffn, L.moe_combine, L.moe_layer, L.moe_layer_host,
                  L.moe_layer_noalloc, L.moe_q8_0_split, L.moe_last_device_status, L.moe_combine_backward,
                  L.moe_act_up_backward, L.moe_q6_k_split):
            f.restype = I32
        L.moe_launch_count.restype = ctypes.c_uint64
        L.moe_trace_enable.argtypes = [I32]
        L.moe_trace_enable.restype = None
        L.moe_trace_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_float), I32]
        L.moe_trace_read.restype = I32
        L.moe_debug_set_wait_limit.argtypes = [I64]
        L.moe_debug_set_wait_limit.restype = None
        L.moe_debug_set_skip_stage.argtypes = [I32]
        L.moe_debug_set_skip_stage.restype = None
        L.moe_debug_set_barrier_delay.argtypes = [I64]
        L.moe_debug_set_barrier_delay.restype = None
        L.moe_set_fused_decode.argtypes = [I32]
        L.moe_set_fused_decode.restype = None
        L.moe_set_fused_front.argtypes = [I32]
        L.moe_set_fused_front.restype = None
        L.moe_set_pair_gemm.argtypes = [I32]
        L.moe_set_pair_gemm.restype = None
        L.moe_set_decode_stream.argtypes = [I32]
        L.moe_set_decode_stream.restype = None
        L.moe_set_tma_gather.argtypes = [I32]
        L.moe_set_tma_gather.restype = None
        L.moe_set_tensor_min_tokens.argtypes = [I32]
        L.moe_set_tensor_min_tokens.restype = None
        L.moe_workspace_regions.argtypes = [DP, ctypes.POINTER(MoeWsRegions)]
        L.moe_workspace_regions.restype = I32
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


def check(code: int, where: str) -> None:
    if code != MOE_OK:
        raise MoeError(code, where)
