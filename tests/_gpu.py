"""Helpers for the GPU parity tests: upload a seeded workload, run the C ABI,
and compare with the oracle under the near-tie protocol."""
from __future__ import annotations

import numpy as np
import torch

import mixture_experts_ffn_07_b200 as moe
import oracle

BF16_TOL = 2e-2          # |gpu - oracle|_inf <= 2e-2 * max|oracle|          (bf16 weights, f32 accumulate)
F32_TOL = (1e-3, 1e-5)   # |gpu - oracle|_inf <= 1e-3 * max|oracle| + 1e-5   (f32 activations)


from mixture_experts_ffn_07_b200.host import run_layer, run_route, split_q8_0 as q8_split, to_device as dev, upload  # noqa: E402,F401


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64) if t.is_floating_point() else t.cpu().numpy()


def tolerance(ref: np.ndarray, act_dtype: str) -> float:
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if act_dtype == "bf16":
        return BF16_TOL * scale
    return F32_TOL[0] * scale + F32_TOL[1]


def near_tie(logits_row: np.ndarray, K: int, absmax: float) -> bool:
    """True when two of the K+1 largest logits are closer than 64 f32 rounding units of the logit's scale."""
    s = -np.sort(-logits_row)[: K + 1]
    delta = 64 * 2.0 ** -24 * absmax
    return bool(np.any(np.diff(-s) < delta)) if len(s) > 1 else False


def expected_layer(L: oracle.Layer, gpu_ids: np.ndarray, tokens=None):
    """Oracle output for `tokens`; tokens whose GPU selection differs from the oracle's are
    accepted only at a near-tie and then recomputed with the GPU's selection.  Returns (out, n_flagged)."""
    ref = oracle.layer(L, tokens)
    ids = ref["ids"]
    g = gpu_ids if tokens is None else gpu_ids[np.asarray(tokens)]
    diff = np.where(np.any(ids != g, axis=1))[0]
    for i in diff:
        assert near_tie(ref["logits"][i], L.K, ref["absmax"][i]), \
            f"token {i}: GPU ids {g[i]} vs oracle {ids[i]} without a near-tie"
    out = ref["out"]
    if len(diff):
        tk = np.arange(L.T) if tokens is None else np.asarray(tokens)
        forced = oracle.layer(L, tk[diff], force_ids=g[diff])
        out = out.copy()
        out[diff] = forced["out"]
    return out, len(diff)


def assert_close(gpu: np.ndarray, ref: np.ndarray, act_dtype: str, what: str = ""):
    err = float(np.max(np.abs(gpu - ref))) if ref.size else 0.0
    tol = tolerance(ref, act_dtype)
    assert err <= tol, f"{what}: max|gpu-oracle| = {err:.3e} > tol {tol:.3e} (max|oracle| {np.max(np.abs(ref)):.3e})"
    return err
