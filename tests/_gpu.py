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


DEFAULT_TENSOR_MIN_TOKENS = 16  # moe_set_tensor_min_tokens' default


class streaming_path:
    """Within the block, bf16 layers of up to 64 tokens take the weight-streaming path (the tensor-core path
    starts at 65 tokens instead of the default 16), for tests of that path."""

    def __enter__(self):
        moe.set_tensor_min_tokens(65)
        return self

    def __exit__(self, *exc):
        moe.set_tensor_min_tokens(DEFAULT_TENSOR_MIN_TOKENS)
        return False


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64) if t.is_floating_point() else t.cpu().numpy()


def tolerance(ref: np.ndarray, act_dtype: str) -> float:
    scale = float(np.max(np.abs(ref))) if ref.size else 0.0
    if act_dtype == "bf16":
        return BF16_TOL * scale
    return F32_TOL[0] * scale + F32_TOL[1]


def tie_delta(absmax: float) -> float:
    """delta_t = 64 * 2^-24 * max_e (sum_h |x_h W_r[e,h]| + |b_e|): the gap below which f32 and f64 logits may
    order two experts differently."""
    return 64 * 2.0 ** -24 * absmax


def near_tie(logits_row: np.ndarray, K: int, absmax: float) -> bool:
    """True when the K-th and (K+1)-th largest logits are closer than delta_t."""
    if len(logits_row) <= K:
        return False
    s = -np.sort(-logits_row)[: K + 1]
    return bool(s[K - 1] - s[K] < tie_delta(absmax))


def valid_near_tie_selection(logits_row: np.ndarray, sel, absmax: float) -> bool:
    """The GPU's ordered selection `sel` is a top-K of the oracle's logits up to delta_t: no unselected expert is
    more than delta_t above a selected one (so a set change needs a K-th vs (K+1)-th near-tie), and consecutive
    slots are in descending order up to delta_t (an order change needs an adjacent near-tie)."""
    d = tie_delta(absmax)
    sel = np.asarray(sel)
    ls = logits_row[sel]
    rest = np.setdiff1d(np.arange(len(logits_row)), sel)
    if len(set(sel.tolist())) != len(sel):
        return False
    if len(rest) and ls.min() < logits_row[rest].max() - d:
        return False
    return bool(np.all(ls[:-1] >= ls[1:] - d))


def expected_layer(L: oracle.Layer, gpu_ids: np.ndarray, tokens=None, gpu_logits: np.ndarray | None = None):
    """Oracle output for `tokens`; a token whose GPU selection differs from the oracle's is flagged and accepted
    only at a near-tie, then recomputed with the GPU's selection.  Near-tie: with the GPU's own f32 logits given
    (whose selection the caller checks bit-exactly), every GPU logit lies within delta_t of the oracle's f64 logit,
    so the GPU's selection is the exact selection of logits inside the rounding bound; without them (plain
    softmax/sigmoid top-K only), the selection is a top-K of the oracle's logits up to delta_t.
    Returns (out, n_flagged)."""
    ref = oracle.layer(L, tokens)
    ids = ref["ids"]
    tk = np.arange(L.T) if tokens is None else np.asarray(tokens)
    g = gpu_ids[tk]
    diff = np.where(np.any(ids != g, axis=1))[0]
    for i in diff:
        if gpu_logits is not None:
            err = float(np.max(np.abs(gpu_logits[tk[i]] - ref["logits"][i])))
            ok = err <= tie_delta(ref["absmax"][i])
        else:
            ok = L.n_groups <= 1 and valid_near_tie_selection(ref["logits"][i], g[i], ref["absmax"][i])
        assert ok, f"token {tk[i]}: GPU ids {g[i]} vs oracle {ids[i]} without a near-tie"
    out = ref["out"]
    if len(diff):
        forced = oracle.layer(L, tk[diff], force_ids=g[diff])
        out = out.copy()
        out[diff] = forced["out"]
    return out, len(diff)


def tile_cover_tokens(ids: np.ndarray, E: int, tile: int = 128) -> list[int]:
    """Tokens such that every (expert, `tile`-row tile) block of the grouped GEMMs holds at least one of their
    pairs, plus the last token.  The GEMM rows of expert e are its pairs t*K + k in ascending order (the stable
    permutation), so tile j of e holds the pairs at ranks [j*tile, (j+1)*tile) of e.  Greedy: blocks of the most
    loaded experts first; for an uncovered block, the token of the block whose K pairs cover most uncovered
    blocks."""
    T, K = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offs = np.concatenate([[0], np.cumsum(counts)])
    rank = np.empty_like(order)
    rank[order] = np.arange(len(order))
    block = flat * (T * K + 1) + (rank - offs[flat]) // tile
    uniq, inv = np.unique(block, return_inverse=True)
    tok_blocks = inv.reshape(T, K)
    covered = np.zeros(len(uniq), bool)
    chosen = {T - 1}
    covered[tok_blocks[T - 1]] = True
    for u in np.argsort(-counts[uniq // (T * K + 1)], kind="stable"):
        if covered[u]:
            continue
        e, j = int(uniq[u] // (T * K + 1)), int(uniq[u] % (T * K + 1))
        cand = order[offs[e] + j * tile: offs[e] + min((j + 1) * tile, int(counts[e]))] // K
        t = int(cand[np.argmax((~covered[tok_blocks[cand]]).sum(axis=1))])
        chosen.add(t)
        covered[tok_blocks[t]] = True
    assert covered.all()
    return sorted(chosen)


def assert_close(gpu: np.ndarray, ref: np.ndarray, act_dtype: str, what: str = ""):
    err = float(np.max(np.abs(gpu - ref))) if ref.size else 0.0
    tol = tolerance(ref, act_dtype)
    assert err <= tol, f"{what}: max|gpu-oracle| = {err:.3e} > tol {tol:.3e} (max|oracle| {np.max(np.abs(ref)):.3e})"
    return err
