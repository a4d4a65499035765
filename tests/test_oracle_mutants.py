"""Plant plausible mistakes in copies of the oracle and check that the pins catch every one.

Each mutant is the oracle's C source with one textual change, compiled to a temporary library
and swapped in for the real one; at least one pin of test_oracle_pins.py must then fail.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_fp8 as fp8
from tests import test_oracle_mx8act as mx8
from tests import test_oracle_w4a4 as w4a4
from tests import test_oracle_nvfp4 as nv4
from tests import test_oracle_norm_residual as nr
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "beam_oracle.c")

MUTANTS = {
    "group_score_top1": ("for (int r = 0; r < group_topn; ++r) {", "for (int r = 0; r < 1; ++r) {"),
    "no_group_limit": ("if (r < topk_groups) group_kept[g] = 1;", "group_kept[g] = 1;"),
    "weights_use_bias": ("for (int j = 0; j < topk; ++j) den += s[id32[j]];",
                         "for (int j = 0; j < topk; ++j) den += sel[id32[j]];"),
    "ties_to_higher_index": ("if (best < 0 || v[i] > v[best]) best = i;", "if (best < 0 || v[i] >= v[best]) best = i;"),
    "sigmoid_sign": ("score[t * E + e] = 1.0 / (1.0 + exp(-acc[r]));",
                     "score[t * E + e] = 1.0 / (1.0 + exp(acc[r]));"),
    "silu_sign": ("double silu = g[r] / (1.0 + exp(-g[r]));", "double silu = g[r] / (1.0 + exp(g[r]));"),
    "silu_missing": ("hb[(b * I + i) * RB + r] = silu * u[r];", "hb[(b * I + i) * RB + r] = g[r] * u[r];"),
    "down_transposed": ("wdr[i] = bf16_bits_to_double(wd[(int64_t)o * I + i]);",
                        "wdr[i] = bf16_bits_to_double(wd[(int64_t)i * H + o]);"),
    "gate_up_swapped_role": ("double silu = g[r] / (1.0 + exp(-g[r]));", "double silu = u[r] / (1.0 + exp(-u[r]));"),
    "no_routed_scale": ("y[t * H + h] = routed_scale * acc;", "y[t * H + h] = acc;"),
    "permute_tokens_descending": ("for (int64_t q = 0; q < n; ++q)\n            if (ids[q] == e) {",
                                  "for (int64_t q = n - 1; q >= 0; --q)\n            if (ids[q] == e) {"),
    "offsets_inclusive": ("offsets[e + 1] = offsets[e] + counts[e];",
                          "offsets[e + 1] = offsets[e] + counts[e] + (e == 0);"),
    "rmsnorm_sum_not_mean": ("const double inv = 1.0 / sqrt(ss / H + eps);",
                             "const double inv = 1.0 / sqrt(ss + eps);"),
    "rmsnorm_eps_outside_sqrt": ("const double inv = 1.0 / sqrt(ss / H + eps);",
                                 "const double inv = 1.0 / (sqrt(ss / H) + eps);"),
    "residual_weights_swapped": ("keep = sqrt((double)(k - 1) / (double)k), add = 1.0 / sqrt((double)k);",
                                 "add = sqrt((double)(k - 1) / (double)k), keep = 1.0 / sqrt((double)k);"),
    "residual_step_off_by_one": ("keep = sqrt((double)(k - 1) / (double)k), add = 1.0 / sqrt((double)k);",
                                 "keep = sqrt((double)k / (double)(k + 1)), add = 1.0 / sqrt((double)(k + 1));"),
    "e4m3_bias_8": ("ldexp(1.0 + m / 8.0, e - 7)", "ldexp(1.0 + m / 8.0, e - 8)"),
    "e4m3_subnormal_exponent": ("ldexp((double)m, -9)", "ldexp((double)m, -10)"),
    "mxfp8_scale_row_major": ("scale[(int64_t)(k / 32) * rows + r]", "scale[r * (K / 32) + k / 32]"),
    "e2m1_subnormal_quarter": ("e == 0 ? 0.5 * m :", "e == 0 ? 0.25 * m :"),
    "e2m1_bias_0": ("ldexp(1.0 + m / 2.0, e - 1)", "ldexp(1.0 + m / 2.0, e)"),
    "nvfp4_nibbles_swapped": ("(k & 1) ? (byte >> 4) : (byte & 15)", "(k & 1) ? (byte & 15) : (byte >> 4)"),
    "nvfp4_scale_row_major": ("scale[(int64_t)(k / 16) * rows + r]", "scale[r * (K / 16) + k / 16]"),
    "nvfp4_global_dropped": ("e2m1_value(nib) * sv * global", "e2m1_value(nib) * sv"),
    "e4m3_round_truncate": ("const double r = nearbyint(m / quantum) * quantum;",
                            "const double r = floor(m / quantum) * quantum;"),
    "mx_scale_too_small": ("if (amax > ldexp(448.0, e)) e += 1;", "if (amax > ldexp(480.0, e)) e += 1;"),
    "mx8_h_not_quantised": ("hb[(b * I + i) * RB + r] = b * RB + r < n ? hq[(b * RB + r) * I + i] : 0.0;",
                            "hb[(b * I + i) * RB + r] = b * RB + r < n ? hd[(b * RB + r) * I + i] : 0.0;"),
    "mx8_silu_missing": ("hd[(b * RB + r) * I + i] = silu_g * u[r];", "hd[(b * RB + r) * I + i] = g[r] * u[r];"),
    "mx8_x_not_quantised": ("xb[(b * H + h) * RB + r] = b * RB + r < n ? xq[(b * RB + r) * H + h] : 0.0;",
                            "xb[(b * H + h) * RB + r] = b * RB + r < n ? xd[(b * RB + r) * H + h] : 0.0;"),
    "e2m1_round_truncate": ("const double rounded = nearbyint(m / quantum) * quantum;",
                            "const double rounded = floor(m / quantum) * quantum;"),
    "nvfp4_act_scale_without_6": ("double a = amax / (6.0 * g);", "double a = amax / g;"),
    "w4a4_h_row_scale": ("oracle_quant_nvfp4_rows_alt(n, I, hd, 0,", "oracle_quant_nvfp4_rows_alt(n, I, hd, 1,"),
    "w4a4_silu_missing": ("hd[(b * RB + r) * I + i] = silu4 * u[r];", "hd[(b * RB + r) * I + i] = g[r] * u[r];"),
    "expert_f64_silu_missing": ("const double act = g[r] / (1.0 + exp(-g[r]));", "const double act = g[r];"),
    "alt_code_window_missing": ("lo = e2m1_round(fmax(0.0, m - 6.0 * eps)), hi = e2m1_round(m + 6.0 * eps);",
                                "lo = e2m1_round(fmax(0.0, m)), hi = e2m1_round(m);"),
    "alt_other_scale_ignored": ("if (cand[c] == s) continue;", "continue;"),
    "alt_other_scale_code_fixed": ("w2 = 6.0 * eps * fmax(s, a) / cand[c];", "w2 = 0.0 * eps * fmax(s, a) / cand[c];"),
    "group_margin_wrong_ranks": ("gs_sorted[topk_groups - 1] - gs_sorted[topk_groups] : INFINITY;",
                                 "gs_sorted[0] - gs_sorted[topk_groups] : INFINITY;"),
    "expert_margin_wrong_ranks": ("sel_sorted[topk - 1] - sel_sorted[topk] : INFINITY;",
                                  "sel_sorted[topk - 1] - sel_sorted[nk - 1] : INFINITY;"),
    "order_margin_skips_last_pair": ("for (int j = 0; j + 1 < topk; ++j) {", "for (int j = 0; j + 2 < topk; ++j) {"),
    "env_signed_down_weights": ("wabs[i] = fabs(wd[(int64_t)o * I + i]);", "wabs[i] = wd[(int64_t)o * I + i];"),
}

PINS = [
    lambda: pins.test_bruteforce_tiny(False),
    lambda: pins.test_bruteforce_tiny(True),
    pins.test_hand_cases,
    lambda: pins.test_margins_are_the_smallest_chosen_minus_unchosen_gaps(True),
    pins.test_invariants_beam_groups,
    pins.test_all_groups_kept_is_plain_topk,
    pins.test_single_expert_matches_torch_float64,
    pins.test_k1_is_scaled_single_expert,
    pins.test_forward_matches_torch_float64_composition,
    pins.test_permute_matches_stable_argsort,
    nr.test_rmsnorm_matches_torch_float64,
    nr.test_rmsnorm_closed_forms,
    nr.test_residual_weights_are_unit_norm,
    nr.test_every_addition_carries_equal_weight_after_104_steps,
    fp8.test_e4m3_decoder_matches_torch_for_all_codes,
    fp8.test_scale_is_a_power_of_two_per_32_block,
    nv4.test_e2m1_decoder_all_codes_both_nibbles,
    nv4.test_even_element_is_the_low_nibble,
    nv4.test_block_scale_per_16_and_global_scale,
    nv4.test_expert_mlp_f64_matches_torch_float64,
    mx8.test_quantised_rows_match_torch_e4m3_cast_and_scale_rule,
    mx8.test_ties_round_to_even_code,
    mx8.test_expert_mx8_matches_torch_float64_composition,
    w4a4.test_nvfp4_rows_match_exhaustive_search_and_torch_e4m3,
    w4a4.test_codes_decode_to_the_dequantised_values,
    w4a4.test_expert_w4a4_matches_torch_float64_composition,
    w4a4.test_alternative_quantisation_envelope,
    w4a4.test_envelope_bounds_every_perturbed_quantisation,
    w4a4.test_expert_envelope_bounds_a_perturbed_h,
]


@contextlib.contextmanager
def mutant_lib(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutant {name}: snippet not found exactly once in the oracle"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(path), "-lm"],
                   check=True)
    saved = oracle.lib()
    oracle._lib = None
    import oracle.build as ob
    real_build = ob.build
    ob.build = lambda *a, **k: str(so)
    try:
        oracle.lib()
        yield
    finally:
        ob.build = real_build
        oracle._lib = saved


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(tmp_path, name):
    old, new = MUTANTS[name]
    caught = []
    with mutant_lib(tmp_path, name, old, new):
        for pin in PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(pin)
    assert caught, f"no pin caught the planted mistake '{name}'"


def test_unmutated_copy_passes(tmp_path):
    with mutant_lib(tmp_path, "identity", "int oracle_num_threads(void)", "int oracle_num_threads(void)"):
        for pin in PINS:
            pin()
