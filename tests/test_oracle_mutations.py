"""Planted mistakes in the oracle must fail its pins.

Each case copies the oracle's C source, plants one plausible mistake (a dropped term, a wrong
sign, a swapped or transposed operand, a wrong tie-break, an unstable order), compiles the copy
on the CPU, loads it in place of the real oracle and runs the pin that should catch it. The
real oracle source is never modified.
"""
import ctypes
import pathlib
import subprocess

import pytest

import oracle
from oracle import build as oracle_build
import tests.test_oracle_fp8 as fp8pins
import tests.test_oracle_pins as pins

MUTATIONS = [
    ("gate and up projections swapped",
     "G += xd[k] * bf16_to_double(wg[j * d + k]);\n                U += xd[k] * bf16_to_double(wu[j * d + k]);",
     "G += xd[k] * bf16_to_double(wu[j * d + k]);\n                U += xd[k] * bf16_to_double(wg[j * d + k]);",
     pins.test_expert_rows_match_textbook_swiglu),
    ("silu factor G dropped",
     "double act = G / (1.0 + exp(-G));",
     "double act = 1.0 / (1.0 + exp(-G));",
     pins.test_expert_rows_match_textbook_swiglu),
    ("bias subtracted instead of added",
     "key[i] = s[i] + bias[i];",
     "key[i] = s[i] - bias[i];",
     pins.test_bias_is_added_to_scores_with_the_right_sign),
    ("gates taken from the biased keys",
     "gate[t * K + r] = s[idx[t * K + r]] / Q;",
     "gate[t * K + r] = key[idx[t * K + r]] / Q;",
     pins.test_gates_are_unbiased_scores_renormalised_over_the_chosen),
    ("ties to the higher index",
     "if (best < 0 || key[i] > key[best]) best = i;",
     "if (best < 0 || key[i] >= key[best]) best = i;",
     pins.test_ties_go_to_the_lower_index),
    ("identity term of zero experts dropped",
     "for (int64_t c = 0; c < d; ++c) acc[c] += g * bf16_to_double(x[t * d + c]);",
     "(void)g;",
     pins.test_all_zero_expert_picks_return_the_input_exactly),
    ("router weight transposed",
     "acc += bf16_to_double(x[t * d + j]) * bf16_to_double(wr[i * d + j]);",
     "acc += bf16_to_double(x[t * d + j]) * bf16_to_double(wr[(j % E) * d + (i + j) % d]);",
     pins.test_router_logits_exact_on_grid_inputs),
    ("bias update sign flipped",
     "const float diff = a - c;",
     "const float diff = c - a;",
     pins.test_bias_update_matches_exact_rational_value_and_sign),
    ("bias target over N+Z instead of N",
     "const float kn = (float)K * (float)N;",
     "const float kn = (float)K * (float)E;",
     pins.test_bias_update_is_zero_at_the_target_load),
    ("grouping not stable in token order",
     "        for (int64_t t = 0; t < T; ++t)\n            for (int64_t r = 0; r < K; ++r)\n                if (idx[t * K + r] == e) {",
     "        for (int64_t t = T - 1; t >= 0; --t)\n            for (int64_t r = 0; r < K; ++r)\n                if (idx[t * K + r] == e) {",
     pins.test_permute_is_a_stable_sort_of_ffn_picks_by_expert),
    ("ln 2 tail dropped from the exp reduction",
     "r = fmaf(-n, K.ln2_lo, r);",
     "(void)K.ln2_lo;",
     pins.test_exp_spec_within_two_ulp_of_exp),
    ("last value dropped from the sum",
     "for (int64_t j = l; j < E; j += 32) acc = acc + v[j];",
     "for (int64_t j = l; j < E - (l == 0); j += 32) acc = acc + v[j];",
     pins.test_sum_spec_error_bound_and_small_cases),
    ("combine uses the first gate for every pick",
     "double g = (double)gate[t * K + r];\n                double v = (idx[t * K + r] < N)",
     "double g = (double)gate[t * K + 0];\n                double v = (idx[t * K + r] < N)",
     pins.test_combine_weights_rows_and_identity_terms),
    ("down projection weight transposed",
     "for (int64_t j = 0; j < I; ++j) acc += hd[j] * bf16_to_double(wd[i * I + j]);",
     "for (int64_t j = 0; j < I; ++j) acc += hd[j] * bf16_to_double(wd[(j * d + i) % (d * I)]);",
     pins.test_expert_down_matches_textbook_and_the_full_expert),
    ("softmax denominator off by one term",
     "float S = oracle_sum_spec(e, E);",
     "float S = oracle_sum_spec(e, E - 1);",
     pins.test_scores_are_the_softmax_over_all_experts),
    ("FP8: up projection scaled with the gate row's scale",
     "U += xd[k] * ((double)su[j] * oracle_e4m3_to_double(wu[j * d + k]));",
     "U += xd[k] * ((double)sg[j] * oracle_e4m3_to_double(wu[j * d + k]));",
     fp8pins.test_fp8_experts_reduce_to_the_bf16_oracle_on_exact_inputs),
    ("FP8: down projection scaled by the wrong weight row",
     "acc += hd[j] * ((double)w2s[i] * oracle_e4m3_to_double(w2q[i * I + j]));",
     "acc += hd[j] * ((double)w2s[(i + 1) % d] * oracle_e4m3_to_double(w2q[i * I + j]));",
     fp8pins.test_fp8_down_projection_reduces_to_the_bf16_one_on_exact_inputs),
    ("FP8: H not quantised before the down projection",
     "for (int64_t j = 0; j < I; ++j) hd[j] = (double)sh * oracle_e4m3_to_double(hq[j]);",
     "for (int64_t j = 0; j < I; ++j) hd[j] = bf16_to_double(hrow[j]) * (sh > 0.0f ? 1.0 : 1.0);",
     fp8pins.test_fp8_down_projection_quantises_each_h_row),
    ("FP8: E4M3 exponent bias 8 instead of 7",
     "ldexp(1.0 + m / 8.0, e - 7);",
     "ldexp(1.0 + m / 8.0, e - 8);",
     fp8pins.test_code_table_matches_the_format_definition),
    ("FP8: ties rounded away from zero",
     "double q = nearbyint(ldexp(a, 3 - e));",
     "double q = round(ldexp(a, 3 - e));",
     fp8pins.test_ties_go_to_the_even_code_and_large_values_saturate),
    ("FP8: row scale for a largest code of 240",
     "const float s = (amax > 0.0f) ? amax / 448.0f : 1.0f;",
     "const float s = (amax > 0.0f) ? amax / 240.0f : 1.0f;",
     fp8pins.test_row_quantisation_scale_and_error_bound),
    ("FP8: no saturation at 448",
     "if (a >= 448.0) return sign | 0x7E;",
     "if (a >= 480.0) return sign | 0x7F;",
     fp8pins.test_ties_go_to_the_even_code_and_large_values_saturate),
]


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_fails_its_pin(tmp_path, monkeypatch, name, old, new, pin):
    src = oracle_build.SRC.read_text()
    assert src.count(old) == 1, f"mutation anchor not found exactly once: {name}"
    mutated = tmp_path / "moe_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", *oracle_build.CFLAGS, "-o", str(so), str(mutated), "-lm"], check=True)
    monkeypatch.setattr(oracle, "_LIB", oracle.configure(ctypes.CDLL(str(so))))
    with pytest.raises(AssertionError):
        pin()


def test_unmutated_oracle_passes_the_same_pins():
    for *_, pin in MUTATIONS:
        pin()
