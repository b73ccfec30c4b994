"""Pins of the f64 oracle to facts outside itself (CPU only).

Each pin comes from the pages (worked values, printed tolerances), a closed form,
brute force on tiny inputs, an invariant, or a special case that reduces to a
textbook formula.  Together they are chosen so that a plausible slip in the
oracle (dropped term, flipped tie-break, transposed weight, wrong constant,
missing renormalisation, wrong shared-gate scale, wrong dequantisation) fails
at least one of them; ``test_oracle_mutants.py`` checks exactly that by
planting such slips in a copy of the oracle.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import workloads
from tests._helpers import ACTS, numpy_layer, widen


def _tiny(T=5, H=64, E=6, I=96, K=2, act="silu", act_dtype="f32", w_dtype="f32", router_dtype="f32",
          shared_I=0, gated=False, bias=None, seed=7, renorm=True, router_std=0.5):
    spec = workloads.Spec(T=T, H=H, E=E, I=I, K=K, act=act, act_dtype=act_dtype, w_dtype=w_dtype,
                          router_dtype=router_dtype, shared_I=shared_I, shared_gated=gated, renormalize=renorm,
                          router_std=router_std)
    wl = workloads.make(spec, seed=seed)
    if bias is not None:
        wl.router_bias = np.asarray(bias, np.float32)
    return oracle.from_workload(wl)


# ---------------------------------------------------------------- activations

def test_silu_known_values(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "silu_known_values.json")))
    gate = np.array(g["gate"])
    up = np.array(g["up"])
    got = oracle.act("silu", gate) * up
    printed = g["silu_of_gate_printed"]
    for i, (gv, uv) in enumerate(zip(gate, up)):
        key = repr(float(gv))
        if key in printed:
            assert abs(got[i] - printed[key] * uv) < g["tolerance"] * max(1.0, abs(uv))
    # the fourth element is the page's own formula 2/(1+e^-2) * 0.5
    assert abs(got[3] - (2.0 / (1.0 + math.exp(-2.0))) * 0.5) < 1e-15


def test_silu_closed_form_and_symmetry():
    g = np.linspace(-20, 20, 4001)
    s = oracle.act("silu", g)
    assert np.allclose(s, g / (1.0 + np.exp(-g)), rtol=0, atol=1e-15)
    # silu(g) - silu(-g) = g  (sigma(g) + sigma(-g) = 1)
    assert np.allclose(s - oracle.act("silu", -g), g, atol=1e-12)


def test_gelu_asymptotics(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "gelu_asymptotics.json")))
    for pt in g["points"]:
        assert abs(oracle.act("gelu_tanh", pt["g"])[0] - pt["gelu"]) <= pt["tol"]
    h = 1e-5
    fd = (oracle.act("gelu_tanh", h)[0] - oracle.act("gelu_tanh", -h)[0]) / (2 * h)
    assert abs(fd - g["derivative_at_zero"]) < g["derivative_tol"]
    # the page's literal constant differs from sqrt(2/pi) by ~3e-11: same function to 1e-9
    c = g["page_constant_sqrt_2_over_pi"]
    xs = np.linspace(-8, 8, 1601)
    page = 0.5 * xs * (1.0 + np.tanh(c * (xs + 0.044715 * xs ** 3)))
    assert np.max(np.abs(oracle.act("gelu_tanh", xs) - page)) < 1e-9


def test_gelu_cubic_term_matters():
    # gelu(g) - g*Phi_tanh(g) with the cubic term: at g=2 the tanh argument is sqrt(2/pi)*(2+0.35772)
    v = oracle.act("gelu_tanh", 2.0)[0]
    assert abs(v - 0.5 * 2.0 * (1 + math.tanh(math.sqrt(2 / math.pi) * (2.0 + 0.044715 * 8.0)))) < 1e-15


# ---------------------------------------------------------------- routing

def test_topk_worked_example(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "topk_worked_example.json")))
    ids, w = oracle.select(np.array([g["logits"]]), g["top_k"], True)
    assert ids[0, 0] == g["first_id"]
    assert ids[0, 1] == 1  # lower index wins the three-way tie
    assert abs(w.sum() - g["weight_sum"]) < g["weight_sum_tolerance"]
    # closed form: renormalised over {0,1}: w0 = e^9/(e^9+1)
    assert abs(w[0, 0] - math.exp(9) / (math.exp(9) + 1)) < 1e-15
    assert w[0, 0] > 100 * w[0, 1]


@pytest.mark.parametrize("E,K", [(1, 1), (2, 1), (4, 2), (7, 3), (12, 12), (16, 5), (64, 8), (256, 8)])
def test_selection_matches_brute_force_sort(E, K):
    rng = np.random.default_rng(E * 100 + K)
    # coarse grid -> many exact ties, which is where a tie-break slip shows
    l = np.round(rng.normal(size=(40, E)) * 2) / 2
    ids, _ = oracle.select(l, K, True)
    for t in range(l.shape[0]):
        ref = sorted(range(E), key=lambda e: (-l[t, e], e))[:K]
        assert list(ids[t]) == ref


def test_weights_closed_form_renorm_and_not():
    rng = np.random.default_rng(3)
    l = rng.normal(size=(30, 9)) * 3
    for renorm in (True, False):
        ids, w = oracle.select(l, 4, renorm)
        for t in range(30):
            den = sum(math.exp(v - l[t].max()) for v in l[t])
            p = [math.exp(l[t, e] - l[t].max()) / den for e in ids[t]]
            if renorm:
                s = sum(p)
                p = [v / s for v in p]
            assert np.allclose(w[t], p, rtol=1e-14, atol=0)


def test_renormalised_weights_sum_to_one():
    rng = np.random.default_rng(11)
    l = rng.normal(size=(200, 128)) * 4
    _, w = oracle.select(l, 8, True)
    assert np.max(np.abs(w.sum(1) - 1.0)) < 1e-12
    # without renormalisation, K = E gives the full softmax, which also sums to 1
    _, w2 = oracle.select(l[:, :16], 16, False)
    assert np.max(np.abs(w2.sum(1) - 1.0)) < 1e-12


def test_softmax_shift_invariance_and_extremes():
    l = np.array([[1000.0, 999.0, -1000.0, 0.0]])
    ids, w = oracle.select(l, 2, True)
    assert list(ids[0]) == [0, 1]
    assert abs(w[0, 0] - 1 / (1 + math.exp(-1))) < 1e-15
    ids2, w2 = oracle.select(l - 12345.0, 2, True)
    assert (ids2 == ids).all() and np.allclose(w2, w, rtol=1e-13)


def test_single_expert_weight_is_exactly_one():
    # ferrox-models decoder.rs, is_dense_layer: top-1 of one expert has weight exactly 1.0
    l = np.random.default_rng(1).normal(size=(10, 1))
    ids, w = oracle.select(l, 1, True)
    assert (ids == 0).all() and (w == 1.0).all()
    ids, w = oracle.select(l, 1, False)
    assert (w == 1.0).all()


def test_router_logits_and_bias():
    L = _tiny(T=6, E=5, bias=[0.0, 0.0, 0.0, 0.0, 50.0])
    lg, am = oracle.logits(L)
    x = widen(L.x, "f32")
    Wr = widen(L.router, "f32")
    assert np.allclose(lg, x @ Wr.T + np.array(L.bias, np.float64), rtol=1e-12, atol=1e-12)
    assert np.allclose(am, (np.abs(x[:, None, :] * Wr[None]).sum(-1) + np.abs(L.bias)).max(1), rtol=1e-12)
    r = oracle.layer(L)
    assert (r["ids"][:, 0] == 4).all()   # the +50 bias wins every token's first slot


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("T,K,E", [(1, 1, 1), (3, 2, 4), (50, 8, 16), (200, 8, 256), (97, 3, 5)])
def test_permutation_properties(T, K, E):
    rng = np.random.default_rng(T * K + E)
    # K distinct experts per token, skewed towards low ids
    ids = np.stack([rng.choice(E, size=K, replace=False, p=None) for _ in range(T)]).astype(np.int32)
    counts, offsets, sp, pp = oracle.permute(ids, E)
    P = T * K
    assert counts.sum() == P
    assert offsets[0] == 0 and offsets[-1] == P and (np.diff(offsets) == counts).all()
    assert sorted(sp.tolist()) == list(range(P))
    assert (sp[pp] == np.arange(P)).all()
    flat = ids.reshape(-1)
    assert sp.tolist() == sorted(range(P), key=lambda p: (flat[p], p))   # stable counting sort
    for e in range(E):
        assert (flat[sp[offsets[e]:offsets[e + 1]]] == e).all()


def test_permutation_rejects_out_of_range():
    with pytest.raises(ValueError):
        oracle.permute(np.array([[0, 5]], np.int32), 4)


# ---------------------------------------------------------------- formats

def test_fp16_decode_all_finite_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    fin = np.isfinite(ref)
    got = np.array([oracle.fp16_to_double(int(b)) for b in bits[fin][::7]])
    assert np.array_equal(got, ref[fin][::7])
    for b in (0x0001, 0x03FF, 0x0400, 0x3C00, 0x7BFF, 0x8001, 0xFBFF):
        assert oracle.fp16_to_double(b) == float(np.array([b], np.uint16).view(np.float16)[0])


def test_q8_0_and_bf16_loads():
    blk = workloads.q8_0_blocks(5, 1, (3, 64))
    got = oracle.load_rows(blk, "q8_0", 64)
    assert np.array_equal(got, widen(blk, "q8_0"))
    # fp16 scale times int8 fits exactly in f32 (11 + 8 significant bits)
    assert np.array_equal(got.astype(np.float32).astype(np.float64), got)
    b = workloads.normal(5, 2, (4, 32), 1.0, "bf16")
    assert np.array_equal(oracle.load_rows(b, "bf16", 32), widen(b, "bf16"))


# ---------------------------------------------------------------- the layer

@pytest.mark.parametrize("act", ["silu", "gelu_tanh"])
@pytest.mark.parametrize("dt", ["f32", "bf16", "q8_0"])
def test_dense_special_case(act, dt):
    """E=1, K=1, no shared expert: the weight is exactly 1 and the layer is a dense gated FFN."""
    L = _tiny(T=4, H=64, E=1, I=96, K=1, act=act, w_dtype=dt, act_dtype="bf16" if dt == "bf16" else "f32",
              router_dtype="bf16" if dt == "bf16" else "f32")
    r = oracle.layer(L)
    assert (r["w"] == 1.0).all() and (r["ids"] == 0).all()
    x = widen(L.x, L.act_dtype)
    g = widen(L.gate, dt).reshape(96, 64)
    u = widen(L.up, dt).reshape(96, 64)
    d = widen(L.down, dt).reshape(64, 96)
    dense = (ACTS[act](x @ g.T) * (x @ u.T)) @ d.T
    assert np.max(np.abs(r["out"] - dense)) <= 1e-12 * np.max(np.abs(dense))


@pytest.mark.parametrize("shared,gated", [(0, False), (48, True), (48, False)])
@pytest.mark.parametrize("renorm", [True, False])
def test_layer_matches_numpy_restatement(shared, gated, renorm):
    L = _tiny(T=7, H=64, E=6, I=32, K=3, shared_I=shared, gated=gated, renorm=renorm, act="gelu_tanh")
    r = oracle.layer(L)
    ref = numpy_layer(L)
    assert (r["ids"] == ref["ids"]).all()
    assert np.allclose(r["w"], ref["w"], rtol=1e-13, atol=0)
    assert np.allclose(r["logits"], ref["logits"], rtol=1e-12, atol=1e-12)
    assert np.max(np.abs(r["out"] - ref["out"])) <= 1e-12 * np.max(np.abs(ref["out"]))


def test_layer_bf16_and_q8_0_match_numpy_restatement():
    for w_dtype, a_dtype in (("bf16", "bf16"), ("q8_0", "f32")):
        L = _tiny(T=5, H=64, E=5, I=64, K=2, act_dtype=a_dtype, w_dtype=w_dtype, router_dtype=a_dtype,
                  shared_I=32, gated=True)
        r = oracle.layer(L)
        ref = numpy_layer(L)
        assert (r["ids"] == ref["ids"]).all()
        assert np.max(np.abs(r["out"] - ref["out"])) <= 1e-12 * np.max(np.abs(ref["out"]))


def test_token_order_invariance():
    L = _tiny(T=9, E=8, K=3, shared_I=32, gated=True)
    base = oracle.layer(L)["out"]
    perm = np.random.default_rng(0).permutation(9)
    L.x = np.ascontiguousarray(L.x[perm])
    got = oracle.layer(L)["out"]
    assert np.array_equal(got, base[perm])      # bit-exact: tokens are independent


def test_token_subset_equals_full():
    L = _tiny(T=9, E=8, K=3)
    full = oracle.layer(L)
    sub = oracle.layer(L, tokens=[8, 0, 3])
    assert np.array_equal(sub["out"], full["out"][[8, 0, 3]])
    assert np.array_equal(sub["ids"], full["ids"][[8, 0, 3]])


def test_forced_selection_reproduces_own_selection():
    L = _tiny(T=6, E=8, K=3)
    full = oracle.layer(L)
    forced = oracle.layer(L, force_ids=full["ids"])
    assert np.array_equal(forced["out"], full["out"])


def test_routed_sum_is_weighted_expert_sum():
    """out[t] = sum_k w_k * expert(t, id_k), summed in k order (the combine)."""
    L = _tiny(T=3, E=5, K=3)
    r = oracle.layer(L)
    for t in range(3):
        acc = np.zeros(L.H)
        for k in range(3):
            acc += r["w"][t, k] * oracle.expert(L, t, int(r["ids"][t, k]))
        assert np.array_equal(acc, r["out"][t])


def test_shared_gate_linearity(golden_dir):
    g = json.load(open(os.path.join(golden_dir, "shared_gate_linearity.json")))
    L = _tiny(T=1, H=g["hidden"], E=g["experts"], K=g["top_k"], I=g["intermediate"],
              shared_I=g["shared_intermediate"], gated=True)
    L.H = g["hidden"]
    outs = []
    for v in g["gate_weight_values"]:
        L.sh_gate_w = np.full(L.H, v, np.float32)
        outs.append(oracle.layer(L)["out"][0])
    mid, a, b = outs
    assert np.max(np.abs(mid - 0.5 * (a + b))) < 1e-12 * np.max(np.abs(mid))
    # with a saturating gate weight, off and on differ by exactly the ungated shared term
    sat = []
    for v in (-1e9, 1e9):
        L.sh_gate_w = np.full(L.H, v, np.float32)
        sat.append(oracle.layer(L)["out"][0])
    a, b = sat
    L.sh_gate_w = None
    y_s, s = oracle.shared(L)
    assert (s == 1.0).all()
    assert np.max(np.abs(np.abs(a - b) - np.abs(y_s[0]))) < 1e-12 * np.max(np.abs(y_s))


def test_ungated_shared_is_added_with_scale_one():
    L = _tiny(T=4, E=4, K=2, shared_I=32, gated=False)
    full = oracle.layer(L)["out"]
    y_s, s = oracle.shared(L)
    Ls = _tiny(T=4, E=4, K=2, shared_I=0)
    routed = oracle.layer(Ls)["out"]
    assert np.max(np.abs(full - (routed + y_s))) < 1e-13 * np.max(np.abs(full))


# ---------------------------------------------------------------- routing variants (SURVEY next rows f-1, f-2)
def test_sigmoid_gating_known_values():
    """sigma(0) = 1/2 exactly; equal logits renormalise to exactly 1/K."""
    _, w = oracle.select(np.zeros((1, 4)), 1, False, gating="sigmoid")
    assert w[0, 0] == 0.5
    _, w = oracle.select(np.full((1, 6), 0.37), 3, True, gating="sigmoid")
    assert np.all(np.abs(w - 1.0 / 3.0) < 1e-15)


def test_sigmoid_gating_equals_two_way_softmax():
    """sigma(a) = e^a / (e^a + e^0): the sigmoid weight of a logit equals the softmax
    weight of the same logit against a single zero logit (an identity, not the formula)."""
    rng = np.random.default_rng(7)
    for a in rng.normal(0, 4, 20):
        _, ws = oracle.select(np.array([[a, -50.0, -60.0]]), 1, False, gating="sigmoid")
        _, wm = oracle.select(np.array([[a, 0.0]]), 2, False, gating="softmax")
        p_a = wm[0, 0] if a >= 0 else wm[0, 1]  # slot of logit a in the softmax selection
        assert abs(ws[0, 0] - p_a) < 1e-14


def test_sigmoid_gating_selects_like_softmax():
    """sigmoid is increasing: the chosen experts and their order are the softmax ones;
    renormalised weights sum to 1 and follow the logit order."""
    rng = np.random.default_rng(8)
    l = rng.normal(0, 2, (40, 32))
    l[:, 5] = l[:, 6]  # ties keep the lower index
    ids_m, _ = oracle.select(l, 6, True)
    ids_s, w_s = oracle.select(l, 6, True, gating="sigmoid")
    assert np.array_equal(ids_m, ids_s)
    assert np.all(np.abs(w_s.sum(axis=1) - 1.0) < 1e-12)
    assert np.all(np.diff(w_s, axis=1) <= 0)
    _, w_n = oracle.select(l, 6, False, gating="sigmoid")
    assert np.all((w_n > 0) & (w_n < 1)) and np.all(np.diff(w_n, axis=1) <= 0)


def _grouped_brute(l, K, n_groups, topk_groups):
    """Independent statement: group maxima by reshape, groups ranked by (max desc, index asc),
    eligible experts ranked by (logit desc, index asc)."""
    E = l.size
    gs = E // n_groups
    gmax = l.reshape(n_groups, gs).max(axis=1)
    order_g = sorted(range(n_groups), key=lambda g: (-gmax[g], g))[:topk_groups]
    elig = [e for e in range(E) if e // gs in order_g]
    return sorted(elig, key=lambda e: (-l[e], e))[:K]


def test_grouped_worked_example():
    """E=8 in 4 groups of 2, 2 groups kept: group maxima (10, 6, 4, 9) keep groups 0 and 3,
    so the third expert is the weak partner of the best one, not the 6 of group 1."""
    l = np.array([[10.0, -5.0, 6.0, 5.0, 4.0, 4.0, 9.0, -9.0]])
    ids, _ = oracle.select(l, 3, True, n_groups=4, topk_groups=2)
    assert ids[0].tolist() == [0, 6, 1]
    ids, _ = oracle.select(l, 3, True)
    assert ids[0].tolist() == [0, 6, 2]


def test_grouped_special_cases_and_brute_force():
    rng = np.random.default_rng(9)
    l = rng.normal(0, 1, (60, 16))
    base, _ = oracle.select(l, 4, True)
    one, _ = oracle.select(l, 4, True, n_groups=1, topk_groups=1)     # one group: plain top-K
    assert np.array_equal(base, one)
    each, _ = oracle.select(l, 4, True, n_groups=16, topk_groups=4)  # a group per expert, K groups: plain top-K
    assert np.array_equal(base, each)
    ties = np.round(rng.normal(0, 1, (60, 16)) * 2) / 2               # many equal logits and equal group maxima
    for n_groups, topk_groups, K in ((4, 2, 3), (8, 3, 5), (2, 1, 8), (4, 4, 6)):
        for rows in (l, ties):
            ids, w = oracle.select(rows, K, True, n_groups=n_groups, topk_groups=topk_groups)
            for t in range(rows.shape[0]):
                assert ids[t].tolist() == _grouped_brute(rows[t], K, n_groups, topk_groups)
            assert np.all(np.abs(w.sum(axis=1) - 1.0) < 1e-12)


# ---------------------------------------------------------------- backward (act * up, combine)
# Inputs of the finite-difference falsifiers on the page (mlx-native
# moe_dispatch.rs, backward_*_finite_difference_falsifier tests).

def _page_seq(n, a, b, c, fn):
    i = np.arange(n, dtype=np.float32)
    return (np.float32(a) + i * np.float32(b) - fn(i * np.float32(c))).astype(np.float32)


def _act_up_forward(act, gu, I):
    g, u = gu[:, :I].astype(np.float64), gu[:, I:].astype(np.float64)
    return oracle.act(act, g.reshape(-1)).reshape(g.shape) * u


@pytest.mark.parametrize("act", ["gelu_tanh", "silu"])
def test_backward_canonical_values(act, golden_dir):
    g = json.load(open(os.path.join(golden_dir, "backward_canonical.json")))
    gu = np.array([g["gate_up"]], np.float32)
    d = oracle.act_up_backward(act, gu, np.array([g["d_h"]], np.float32))[0]
    for v, e, tol in zip(d, g["expected_d_gate_up"], g["tol"]):
        assert abs(v - e) <= tol, (act, v, e)


@pytest.mark.parametrize("act", ["gelu_tanh", "silu"])
def test_act_grad_matches_finite_difference(act):
    h = 1e-5
    for g in np.linspace(-9, 9, 721):
        fd = (oracle.act(act, g + h)[0] - oracle.act(act, g - h)[0]) / (2 * h)
        assert abs(oracle.act_grad(act, g) - fd) < 1e-8, (act, g)


@pytest.mark.parametrize("act", ["gelu_tanh", "silu"])
def test_act_up_backward_finite_difference(act):
    T, K, I = 2, 3, 5
    P = T * K
    gu = _page_seq(P * 2 * I, 0.5, 0.07, 0.013, np.sin).reshape(P, 2 * I)
    seed = _page_seq(P * I, 0.3, 0.05, 0.011, np.cos).reshape(P, I)
    d = oracle.act_up_backward(act, gu, seed)
    base = gu.astype(np.float64)
    h = 1e-4
    for idx in range(base.size):
        r, c = divmod(idx, 2 * I)
        gp, gm = base.copy(), base.copy()
        gp[r, c] += h
        gm[r, c] -= h
        fd = (np.sum(_act_up_forward(act, gp, I) * seed) - np.sum(_act_up_forward(act, gm, I) * seed)) / (2 * h)
        assert abs(d[r, c] - fd) < 1e-7 * max(1.0, abs(fd)), (act, idx)


def test_combine_backward_finite_difference():
    T, K, H = 3, 4, 7
    y = _page_seq(T * K * H, 0.1, 0.013, 0.004, np.sin).reshape(T, K, H)
    w = (np.float32(0.2) + np.arange(T * K, dtype=np.float32) * np.float32(0.07)).reshape(T, K)
    seed = _page_seq(T * H, 0.3, 0.05, 0.011, np.cos).reshape(T, H)
    d_y, d_w = oracle.combine_backward(y, w, seed)

    def loss(yy, ww):
        out = np.einsum("tkd,tk->td", yy, ww)
        return np.sum(out * seed)

    Y, W = y.astype(np.float64), w.astype(np.float64)
    h = 1e-3
    for idx in np.ndindex(T, K, H):
        yp, ym = Y.copy(), Y.copy()
        yp[idx] += h
        ym[idx] -= h
        fd = (loss(yp, W) - loss(ym, W)) / (2 * h)
        assert abs(d_y[idx] - fd) < 1e-9 * max(1.0, abs(fd)), idx
    for idx in np.ndindex(T, K):
        wp, wm = W.copy(), W.copy()
        wp[idx] += h
        wm[idx] -= h
        fd = (loss(Y, wp) - loss(Y, wm)) / (2 * h)
        assert abs(d_w[idx] - fd) < 1e-9 * max(1.0, abs(fd)), idx


def test_combine_backward_special_cases():
    rng = np.random.default_rng(5)
    T, K, H = 4, 3, 6
    y = rng.standard_normal((T, K, H)).astype(np.float32)
    w = rng.random((T, K)).astype(np.float32)
    d_y, d_w = oracle.combine_backward(y, w, np.zeros((T, H), np.float32))
    assert not d_y.any() and not d_w.any()
    # one-hot d_out picks out single elements: d_w[t,k] = y[t,k,j], d_y[t,k,:] = w[t,k] e_j
    for t, j in [(0, 0), (2, 5), (3, 2)]:
        dout = np.zeros((T, H), np.float32)
        dout[t, j] = 1.0
        d_y, d_w = oracle.combine_backward(y, w, dout)
        for k in range(K):
            assert d_w[t, k] == y[t, k, j]
            assert d_y[t, k, j] == w[t, k] and np.count_nonzero(d_y[t, k]) == (w[t, k] != 0)
        assert not np.delete(d_w, t, axis=0).any()


# ---------------------------------------------------------------- k-quant stacks (Q4_K, Q6_K)
# ferrum-kernels vnext MoE names Q4_K and Q6_K blocks of 256 values in 144 and
# 210 bytes; the byte layout is GGML's.  The gguf package's numpy dequantiser
# (a library routine, independent of the oracle) pins the decoding.

def _kq_blocks(fmt, nblocks, seed, d=0.01, dmin=0.02):
    rng = np.random.default_rng(seed)
    nb = oracle.BLOCK[fmt][0]
    b = rng.integers(0, 256, (nblocks, nb), dtype=np.uint8)
    if fmt == "q4_k":
        b[:, 0:2] = np.frombuffer(np.full(nblocks, d, np.float16).tobytes(), np.uint8).reshape(-1, 2)
        b[:, 2:4] = np.frombuffer(np.full(nblocks, dmin, np.float16).tobytes(), np.uint8).reshape(-1, 2)
    else:
        b[:, 208:210] = np.frombuffer(np.full(nblocks, d, np.float16).tobytes(), np.uint8).reshape(-1, 2)
    return b


def test_kquant_block_sizes_from_the_pages():
    gguf = pytest.importorskip("gguf")
    T = gguf.constants.GGMLQuantizationType
    assert oracle.BLOCK["q4_k"] == (144, 256) == gguf.constants.GGML_QUANT_SIZES[T.Q4_K][::-1]
    assert oracle.BLOCK["q6_k"] == (210, 256) == gguf.constants.GGML_QUANT_SIZES[T.Q6_K][::-1]


@pytest.mark.parametrize("fmt", ["q4_k", "q6_k"])
def test_kquant_rows_match_gguf(fmt):
    gguf = pytest.importorskip("gguf")
    qt = {"q4_k": gguf.constants.GGMLQuantizationType.Q4_K, "q6_k": gguf.constants.GGMLQuantizationType.Q6_K}[fmt]
    for seed, (d, dmin) in enumerate([(0.01, 0.02), (1.5e-4, 1e-3), (3e-5, 2e-5), (-0.5, 0.25), (7.0, -3.0)]):
        rows, cols = 3, 768
        b = _kq_blocks(fmt, rows * cols // 256, seed, d, dmin)
        ref = gguf.quants.dequantize(b.reshape(-1), qt).reshape(rows, cols)
        got = oracle.load_rows(b.reshape(rows, -1), fmt, cols)
        # every term is exact in f64 and gguf rounds once to f32
        assert np.array_equal(got.astype(np.float32), ref), (fmt, seed)


def test_q4_k_single_sub_block_probes():
    """One sub-block scale (or min) at a time: only that sub-block's 32 values move."""
    for j in range(8):
        b = np.zeros(144, np.uint8)
        b[0:2] = np.frombuffer(np.float16(0.5).tobytes(), np.uint8)
        b[2:4] = np.frombuffer(np.float16(0.25).tobytes(), np.uint8)
        b[16:] = (np.arange(128) * 37 % 256).astype(np.uint8)  # varied nibbles
        # 6-bit scale 5 and min 3 for sub-block j only
        if j < 4:
            b[4 + j] = 5
            b[8 + j] = 3
        else:
            b[8 + j] = 5 | (3 << 4)
        v = oracle.load_rows(b.reshape(1, -1), "q4_k", 256)[0]
        qs = b[16:]
        for jj in range(8):
            byte = qs[32 * (jj // 2):32 * (jj // 2) + 32]
            q = (byte & 15) if jj % 2 == 0 else (byte >> 4)
            exp = 0.5 * 5 * q - 0.25 * 3 if jj == j else np.zeros(32)
            assert np.array_equal(v[32 * jj:32 * jj + 32], exp), (j, jj)
    # the high bits of scales[j-4] and scales[j] extend sub-block j >= 4 to 6 bits
    b = np.zeros(144, np.uint8)
    b[0:2] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    b[2:4] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    b[4 + 1] = 0xC0  # high bits of scales[1]: scale of sub-block 5 gets 48
    b[4 + 5] = 0x80  # high bits of scales[5]: min of sub-block 5 gets 32
    b[16:] = 0x11
    v = oracle.load_rows(b.reshape(1, -1), "q4_k", 256)[0]
    assert np.all(v[160:192] == 48 * 1 - 32)
    assert np.all(v[32:64] == 0) and np.all(v[64:96] == 0)


def test_q6_k_single_scale_probes():
    rng = np.random.default_rng(9)
    for k in range(16):
        b = np.zeros(210, np.uint8)
        b[:192] = rng.integers(0, 256, 192, dtype=np.uint8)
        b[192 + k] = np.uint8(np.int8(-3).view(np.uint8))
        b[208:210] = np.frombuffer(np.float16(0.125).tobytes(), np.uint8)
        v = oracle.load_rows(b.reshape(1, -1), "q6_k", 256)[0]
        nz = np.nonzero(np.arange(256) // 16 == k)[0]
        assert not np.delete(v, nz).any()
        # brute force of value 16k + l: 6-bit code from ql/qh, centred at 32
        for idx in nz:
            n, j = divmod(idx, 128)
            i, l = divmod(j, 32)
            lowb = b[64 * n + l + 32 * (i & 1)]
            q = (lowb & 15 if i < 2 else lowb >> 4) | (((b[128 + 32 * n + l] >> (2 * i)) & 3) << 4)
            assert v[idx] == 0.125 * -3 * (int(q) - 32)
    # q = 32 everywhere decodes to zero whatever the scales
    b = np.zeros(210, np.uint8)
    b[128:192] = 0xAA  # high bits 2 in every pair -> q = 32
    b[192:208] = 7
    b[208:210] = np.frombuffer(np.float16(1.0).tobytes(), np.uint8)
    assert not oracle.load_rows(b.reshape(1, -1), "q6_k", 256).any()


@pytest.mark.parametrize("w_dtype", ["q4_k", "q4_k_q6_k"])
def test_kquant_dense_special_case(w_dtype):
    """E = 1, K = 1: the layer is the dense FFN on gguf-dequantised weights (numpy matmuls)."""
    gguf = pytest.importorskip("gguf")
    Q = gguf.constants.GGMLQuantizationType
    T, H, I = 5, 512, 256
    rng = np.random.default_rng(3)
    x = rng.standard_normal((T, H)).astype(np.float32)
    g = _kq_blocks("q4_k", I * H // 256, 1, 1e-3, 5e-3)
    u = _kq_blocks("q4_k", I * H // 256, 2, 1e-3, 5e-3)
    dfmt = "q6_k" if w_dtype == "q4_k_q6_k" else "q4_k"
    dq = _kq_blocks(dfmt, H * I // 256, 3, 2e-4, 5e-3)
    L = oracle.Layer(T=T, H=H, E=1, I=I, K=1, act="silu", renormalize=True, act_dtype="f32", w_dtype=w_dtype,
                     router_dtype="f32", x=x, router=np.zeros((1, H), np.float32), gate=g.reshape(1, I, -1),
                     up=u.reshape(1, I, -1), down=dq.reshape(1, H, -1))
    out = oracle.layer(L)["out"]
    G = gguf.quants.dequantize(g.reshape(-1), Q.Q4_K).reshape(I, H).astype(np.float64)
    U = gguf.quants.dequantize(u.reshape(-1), Q.Q4_K).reshape(I, H).astype(np.float64)
    D = gguf.quants.dequantize(dq.reshape(-1), Q.Q6_K if dfmt == "q6_k" else Q.Q4_K).reshape(H, I).astype(np.float64)
    a = x.astype(np.float64) @ G.T
    ref = ((a / (1 + np.exp(-a))) * (x.astype(np.float64) @ U.T)) @ D.T
    assert np.allclose(out, ref, rtol=1e-9, atol=1e-9 * np.max(np.abs(ref)))
