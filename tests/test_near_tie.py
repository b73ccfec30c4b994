"""The GPU tests' near-tie acceptance rule and tile-covering token sample, on hand-made cases (CPU only)."""
import numpy as np

from tests import _gpu


def test_near_tie_is_the_kth_vs_next_gap():
    d = _gpu.tie_delta(1.0)
    row = np.array([5.0, 4.0, 3.0, 3.0 - d / 2, 1.0])
    assert _gpu.near_tie(row, 3, 1.0)        # 3rd and 4th within delta
    assert not _gpu.near_tie(row, 2, 1.0)    # 2nd and 3rd are 1 apart
    row2 = np.array([5.0, 5.0 - d / 2, 3.0, 1.0])
    assert not _gpu.near_tie(row2, 3, 1.0)   # a near-tie inside the top K is not a K-th vs (K+1)-th tie


def test_valid_selection_rules():
    d = _gpu.tie_delta(1.0)
    row = np.array([5.0, 4.0, 3.0, 3.0 - d / 2, 1.0])
    assert _gpu.valid_near_tie_selection(row, [0, 1, 2], 1.0)       # the exact top-3
    assert _gpu.valid_near_tie_selection(row, [0, 1, 3], 1.0)       # swaps the tied 3rd/4th
    assert not _gpu.valid_near_tie_selection(row, [0, 1, 4], 1.0)   # expert 4 is far below
    assert not _gpu.valid_near_tie_selection(row, [1, 0, 2], 1.0)   # order change without a tie
    row2 = np.array([5.0, 5.0 - d / 2, 3.0, 1.0])
    assert _gpu.valid_near_tie_selection(row2, [1, 0, 2], 1.0)      # adjacent tie: either order
    assert not _gpu.valid_near_tie_selection(row2, [0, 0, 2], 1.0)  # repeated expert


def test_tile_cover_brute_force():
    rng = np.random.default_rng(3)
    T, E, K, tile = 300, 6, 2, 16
    # skewed routing: expert 0 gets most first choices
    ids = np.stack([rng.choice(E, size=K, replace=False, p=[.5, .2, .1, .1, .05, .05]) for _ in range(T)])
    tokens = _gpu.tile_cover_tokens(ids, E, tile)
    assert T - 1 in tokens
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")
    counts = np.bincount(flat, minlength=E)
    offs = np.concatenate([[0], np.cumsum(counts)])
    chosen = set(tokens)
    for e in range(E):
        for j in range((counts[e] + tile - 1) // tile):
            rows = order[offs[e] + j * tile: offs[e] + min((j + 1) * tile, counts[e])]
            assert any(p // K in chosen for p in rows), (e, j)
    assert len(tokens) < T // 2
