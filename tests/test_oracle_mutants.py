"""Planted mistakes in a copy of the oracle must each fail a pin (CPU only).

Each mutant is oracle.c with one plausible slip applied as a text substitution,
compiled to a temporary library and bound in place of the real one while a
battery of the pin tests runs.  A mutant that passes every pin would mean the
pins leave that part of the oracle unchecked.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = {
    "tie_break_flipped": ("return (a->e > b->e) - (a->e < b->e);", "return (a->e < b->e) - (a->e > b->e);"),
    "renorm_dropped": ("double inv = sum_sel > 1e-20 ? 1.0 / sum_sel : 1.0 / (double)K;", "double inv = 1.0;"),
    "gelu_cubic_coefficient": ("0.044715 * g * g * g", "0.44715 * g * g * g"),
    "silu_sign": ("return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));"),
    "down_row_base": ("load_row(Wd, df, drow0 + j, F, row);", "load_row(Wd, df, row0 + j, F, row);"),
    "shared_gate_ignored": ("for (int64_t j = 0; j < H; ++j) o[j] += s * y[j];",
                            "for (int64_t j = 0; j < H; ++j) o[j] += y[j];"),
    "router_bias_dropped": ("s += (double)w->bias[e];", "s += 0.0;"),
    "permutation_unstable": ("int32_t pos = offsets[e] + fill[e]++;", "int32_t pos = offsets[e + 1] - 1 - fill[e]++;"),
    "q8_unsigned": ("d * (double)(int8_t)p[b * 34 + 2 + j]", "d * (double)(uint8_t)p[b * 34 + 2 + j]"),
    "slot_weight_index": ("o[j] += wk[k] * y[j];", "o[j] += wk[0] * y[j];"),
    "up_reads_gate": ("load_row(Wu, gf, row0 + i, Hin, row);", "load_row(Wg, gf, row0 + i, Hin, row);"),
    "fp16_exponent_bias": ("ldexp(1024.0 + man, ex - 25)", "ldexp(1024.0 + man, ex - 24)"),
    "sigmoid_gating_ignored": ("if (gating == ORA_GATING_SIGMOID) {", "if (0) {"),
    "sigmoid_sign": ("for (int64_t e = 0; e < E; ++e) p[e] = 1.0 / (1.0 + exp(-l[e]));",
                     "for (int64_t e = 0; e < E; ++e) p[e] = 1.0 / (1.0 + exp(l[e]));"),
    "group_score_min": ("if (l[e] > m) m = l[e];\n      gkeys", "if (m == -INFINITY || l[e] < m) m = l[e];\n      gkeys"),
    "groups_kept_off_by_one": ("for (int64_t i = 0; i < r->topk_groups; ++i) keep[gkeys[i].e] = 1;",
                               "for (int64_t i = 0; i <= r->topk_groups && i < r->n_groups; ++i) keep[gkeys[i].e] = 1;"),
    "groups_ignored": ("if (r->n_groups > 1) {", "if (0) {"),
    "gelu_grad_tanh_term_dropped": (" + 0.5 * g * (1.0 - th * th) * c * (1.0 + 3.0 * a * g * g);", ";"),
    "silu_grad_sign": ("return s * (1.0 + g * (1.0 - s));", "return s * (1.0 - g * (1.0 - s));"),
    "d_up_uses_gate": ("d_gate_up[p * 2 * I + I + i] = dh * ora_act(act, g);", "d_gate_up[p * 2 * I + I + i] = dh * g;"),
    "d_gate_drops_up": ("d_gate_up[p * 2 * I + i] = dh * u * ora_act_grad(act, g);",
                        "d_gate_up[p * 2 * I + i] = dh * ora_act_grad(act, g);"),
    "d_w_slots_transposed": ("s += (double)y[p * H + d] * (double)d_out[t * H + d];",
                             "s += (double)y[(k * T + t) * H + d] * (double)d_out[t * H + d];"),
    "q4_k_nibbles_swapped": ("const int q = (j % 2 == 0) ? (byte & 15) : (byte >> 4);",
                             "const int q = (j % 2 == 0) ? (byte >> 4) : (byte & 15);"),
    "q4_k_high_scale_bits": ("s = (sc[j + 4] & 15) | ((sc[j - 4] >> 6) << 4);", "s = (sc[j + 4] & 15) | ((sc[j] >> 6) << 4);"),
    "q4_k_min_added": ("out[b * 256 + 32 * j + l] = d * s * q - dmin * m;", "out[b * 256 + 32 * j + l] = d * s * q + dmin * m;"),
    "q6_k_not_centred": ("out[b * 256 + 128 * n + j] = d * sc[8 * n + j / 16] * (q - 32);",
                         "out[b * 256 + 128 * n + j] = d * sc[8 * n + j / 16] * q;"),
    "q6_k_high_bits_shift": ("const int hi = (qh[32 * n + l] >> (2 * i)) & 3;", "const int hi = (qh[32 * n + l] >> i) & 3;"),
    "q6_k_scale_group": ("d * sc[8 * n + j / 16]", "d * sc[8 * n + j / 32]"),
    "q6_down_read_as_q4": ("static int down_format(int w_dtype) { return w_dtype == ORA_Q4_K_Q6_K ? ORA_Q6_K : w_dtype; }",
                           "static int down_format(int w_dtype) { return w_dtype == ORA_Q4_K_Q6_K ? ORA_Q4_K : w_dtype; }"),
    "d_y_first_slot_weight": ("d_y[p * H + d] = (double)w[p] * (double)d_out[t * H + d];",
                              "d_y[p * H + d] = (double)w[t * K] * (double)d_out[t * H + d];"),
}

BATTERY = [
    pins.test_silu_known_values, pins.test_gelu_asymptotics, pins.test_topk_worked_example,
    lambda g: pins.test_selection_matches_brute_force_sort(16, 5), lambda g: pins.test_renormalised_weights_sum_to_one(),
    lambda g: pins.test_weights_closed_form_renorm_and_not(), lambda g: pins.test_router_logits_and_bias(),
    lambda g: pins.test_permutation_properties(50, 8, 16), lambda g: pins.test_q8_0_and_bf16_loads(),
    lambda g: pins.test_fp16_decode_all_finite_patterns(),
    lambda g: pins.test_dense_special_case("silu", "f32"),
    lambda g: pins.test_layer_matches_numpy_restatement(48, True, True),
    pins.test_shared_gate_linearity,
    lambda g: pins.test_sigmoid_gating_known_values(), lambda g: pins.test_sigmoid_gating_equals_two_way_softmax(),
    lambda g: pins.test_sigmoid_gating_selects_like_softmax(), lambda g: pins.test_grouped_worked_example(),
    lambda g: pins.test_grouped_special_cases_and_brute_force(),
    lambda g: pins.test_backward_canonical_values("gelu_tanh", g), lambda g: pins.test_backward_canonical_values("silu", g),
    lambda g: pins.test_act_grad_matches_finite_difference("gelu_tanh"),
    lambda g: pins.test_act_grad_matches_finite_difference("silu"),
    lambda g: pins.test_act_up_backward_finite_difference("gelu_tanh"),
    lambda g: pins.test_combine_backward_finite_difference(), lambda g: pins.test_combine_backward_special_cases(),
    lambda g: pins.test_kquant_rows_match_gguf("q4_k"), lambda g: pins.test_kquant_rows_match_gguf("q6_k"),
    lambda g: pins.test_q4_k_single_sub_block_probes(), lambda g: pins.test_q6_k_single_scale_probes(),
    lambda g: pins.test_kquant_dense_special_case("q4_k_q6_k"),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, golden_dir):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor not found once: {old}"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-o", str(so), str(path), "-lm"])
    saved = oracle._lib_handle
    oracle._lib_handle = oracle.bind(ctypes.CDLL(str(so)))
    caught = []
    try:
        for check in BATTERY:
            try:
                check(golden_dir)
            except AssertionError:
                caught.append(getattr(check, "__name__", "lambda"))
    finally:
        oracle._lib_handle = saved
    assert caught, f"mutant {name} passed every pin"
