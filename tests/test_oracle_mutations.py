"""Planted mistakes in the oracle must fail its pins.

Each mutant is a copy of moe_oracle.c with one plausible mistake (a swapped operand, a
dropped term, an off-by-one, a wrong tie rule ...), compiled on the CPU into a temporary
library. The pins of test_oracle_pins.py run against it, and at least one must fail.
"""
import os
import subprocess

import pytest

from oracle import oracle
import test_oracle_pins as pins  # noqa: E402

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = {
    "silu_on_gate": ("a[d] = (u / (1.0 + exp(-u))) * g;", "a[d] = (g / (1.0 + exp(-g))) * u;"),
    "no_shared_term": ("for (int64_t h = 0; h < H; ++h) o[h] += y[h];",
                       "for (int64_t h = 0; h < H; ++h) o[h] += 0.0 * y[h];"),
    "unweighted_combine": ("o[h] += topk_w[s] * y[h];", "o[h] += y[h];"),
    "tie_to_higher_index": ("v[e] > v[best]) best = e;", "v[e] >= v[best]) best = e;"),
    "no_renormalise": ("topk_w[t * k + j] = p[topk_ids[t * k + j]] / s;",
                       "topk_w[t * k + j] = p[topk_ids[t * k + j]];"),
    "capacity_off_by_one": ("(rank < capacity)", "(rank <= capacity)"),
    "bias_sign": ("if (bias) s += (double)bias[e];", "if (bias) s -= (double)bias[e];"),
    "down_transposed": ("s += bf16_to_double(rd[d]) * a[d];",
                        "s += bf16_to_double(w_down[d * H + h]) * a[d];"),
    "segment_not_padded": ("int64_t padded = (kept_n[e] + block_m - 1) / block_m * block_m;",
                           "int64_t padded = kept_n[e];"),
    "unstable_segment_order": ("sorted_ids[offset[e] + fill[e]++] = (int32_t)s;",
                               "sorted_ids[offset[e] + kept_n[e] - 1 - fill[e]++] = (int32_t)s;"),
    "router_row_index": ("const double *w = wr + e * H;", "const double *w = wr + (E - 1 - e) * H;"),
    "combine_skips_first_row": ("for (int64_t j = 0; j < m; ++j) {", "for (int64_t j = 1; j < m; ++j) {"),
    "down_weight_dropped": ("yi[c] = wts[i] * yi[c];", "yi[c] = yi[c];"),
    "shared_up_gate_swapped": ("swiglu_row(xt, ws_up, ws_gate, H, Ds, h + i * ld,",
                               "swiglu_row(xt, ws_gate, ws_up, H, Ds, h + i * ld,"),
    "up_projection_reported_as_gate": ("if (uo) uo[d] = u;", "if (uo) uo[d] = g;"),
}

PIN_TESTS = [
    lambda: pins.test_hand_worked_golden("hand_worked_layer.json"),
    lambda: pins.test_hand_worked_golden("hand_worked_capacity.json"),
    lambda: pins.test_router_logits_match_matmul(),
    lambda: pins.test_topk_softmax_matches_sort_definition(64, 2, True),
    lambda: pins.test_topk_exact_ties_prefer_lower_index(),
    lambda: pins.test_align_matches_argsort_definition("random", 48, 1.0),
    lambda: pins.test_capacity_keeps_first_slots_in_token_order(),
    lambda: pins.test_brute_force_tiny_workload(),
    lambda: pins.test_brute_force_with_capacity_and_shared(),
    lambda: pins.test_brute_force_with_bias(),
    lambda: pins.test_top_k_equals_E_is_dense_softmax_mixture(),
    lambda: pins.test_expert_h_is_swiglu_of_two_matmuls(),
    lambda: pins.test_expert_down_is_weighted_matmul(),
    lambda: pins.test_combine_sums_listed_rows_in_order(),
    lambda: pins.test_stages_compose_to_the_layer(),
]


# first line of the oracle's MXFP8 section
MX_SECTION = " * MXFP8 experts."

# planted mistakes in the MXFP8 arithmetic, checked against the pins of test_oracle_mx_pins.py
MX_MUTANTS = {
    "mx_ties_away_from_zero": ("if (frac > 0.5 || (frac == 0.5 && fmod(n, 2.0) != 0.0)) n += 1.0;",
                               "if (frac >= 0.5) n += 1.0;"),
    "mx_emax_7": ("s = (ex - 1) - 8;", "s = (ex - 1) - 7;"),
    "mx_no_saturation": ("if (a > 448.0) a = 448.0;", "if (a > 1e300) a = 448.0;"),
    "mx_h_not_quantised": ("mx_round_trip(a + l * Dt, Dt, scratch);", "(void)scratch;"),
    "mx_x_not_quantised": ("mx_round_trip(xq + i * H, H, scratch);", "(void)scratch;"),
    "mx_amax_over_16": ("for (int i = 0; i < 32; ++i) if (fabs(blk[i]) > amax)",
                        "for (int i = 0; i < 16; ++i) if (fabs(blk[i]) > amax)"),
    "mx_scale_applied_inverted": ("moe_oracle_e4m3_encode(ldexp(blk[i], -s))",
                                  "moe_oracle_e4m3_encode(ldexp(blk[i], s))"),
    "mx_subnormal_step": ("if (e == 0) v = ldexp((double)m, -9);", "if (e == 0) v = ldexp((double)m, -10);"),
    "mx_exponent_bias": ("else v = ldexp(1.0 + m / 8.0, e - 7);", "else v = ldexp(1.0 + m / 8.0, e - 8);"),
    "mx_down_weights_not_quantised": ("mx_round_trip(wd, Dt, scratch);", "(void)wd;"),
}


def _mx_pin_tests():
    import test_oracle_mx_pins as mx
    return [
        lambda: mx.test_hand_worked_mx_layer(),
        lambda: mx.test_e4m3_every_finite_code_round_trips(),
        lambda: mx.test_e4m3_ties_go_to_the_even_code(),
        lambda: mx.test_e4m3_saturates_at_448(),
        lambda: mx.test_e4m3_matches_torch_float8_conversion(),
        lambda: [mx.test_e4m3_decode_table(c, v) for c, v in ((0x01, 2.0 ** -9), (0x38, 1.0), (0x7E, 448.0))],
        lambda: [mx.test_scale_code_is_floor_log2_amax_minus_8(j, p) for j in (-7, 0, 5) for p in (0, 31)],
        lambda: mx.test_small_element_under_a_large_maximum(),
        lambda: mx.test_rounding_error_bound(),
    ]


def _compile_and_count_failures(src, tmp_path, pin_tests):
    mut = tmp_path / "mut.c"
    mut.write_text(src)
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-fopenmp", str(mut),
                           "-o", str(so), "-lm"])
    failed = 0
    oracle.use_library(str(so))
    try:
        for pin in pin_tests:
            try:
                pin()
            except AssertionError:
                failed += 1
    finally:
        oracle.use_library(None)
    return failed


@pytest.mark.parametrize("name", sorted(MX_MUTANTS))
def test_planted_mx_mistake_fails_a_pin(name, tmp_path):
    old, new = MX_MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old}"
    failed = _compile_and_count_failures(src.replace(old, new), tmp_path, _mx_pin_tests())
    assert failed > 0, f"mutant {name} passed every pin"


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_fails_a_pin(name, tmp_path):
    """The bf16 mutants change the code before the MXFP8 section (the MX layer repeats some of
    the same lines, which its own mutants cover)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    head, tail = src.split(MX_SECTION, 1)
    assert head.count(old) == 1, f"mutation anchor not unique: {old}"
    failed = _compile_and_count_failures(head.replace(old, new) + MX_SECTION + tail, tmp_path, PIN_TESTS)
    assert failed > 0, f"mutant {name} passed every pin"
