"""The pins catch plausible mistakes in the oracle (CPU only).

Each case plants one mistake -- a wrong constant, a dropped term, a swapped
operand or branch, an off-by-one -- in a temporary copy of the oracle's C
source, builds it, routes the oracle through it, and requires at least one of
the pins to fail.  The product library is not involved.
"""
import os

import pytest

import oracle
import test_oracle_bf16 as BF
import test_oracle_tensor_list as D
import test_oracle_nf4 as N
import test_oracle_philox as P
import test_oracle_update as U
import test_oracle_variants as V
import test_oracle_zeeden as E
import test_oracle_zipsr as Z


def pins(golden):
    return [
        ("philox known answers", lambda: P.test_known_answer_vectors(golden)),
        ("philox keying", P.test_draw_is_word_e_mod_4_of_one_call),
        ("philox library", P.test_matches_the_curand_library_generator),
        ("uniform", P.test_uniform_range_and_granularity),
        ("nf4 quantiles", N.test_levels_match_library_quantiles),
        ("nf4 structure", N.test_level_structure),
        ("nf4 nearest", N.test_rtn_is_nearest_level),
        ("nf4 ties", N.test_rtn_threshold_ties_go_low),
        ("state-space SR", lambda: [N.test_state_space_sr_unbiased_by_enumeration(x)
                                    for x in (-0.3, 0.02, 0.65)]),
        ("worked example", lambda: Z.test_worked_example_near_zero_cell(golden)),
        ("ZIP-SR expectation", lambda: [Z.test_exact_expectation_of_h(*c) for c in Z.CASES[::7]]),
        ("ZIP-SR ends", Z.test_zero_and_top_are_deterministic),
        ("ZIP-SR bracket", Z.test_bracket_at_and_below_code_points),
        ("ZIP-SR 32-bit expectation", lambda: [Z.test_u32_decision_exact_expectation(*c)
                                               for c in Z.CASES[::9]]),
        ("ZIP-SR zero-cell bias", lambda: [Z.test_zero_cell_has_no_23_bit_bias(v)
                                           for v in (1e-2, 1e-3)]),
        ("ZIP-SR block decisions", Z.test_block_decisions_follow_the_page_probability_on_the_word),
        ("uniform32", P.test_uniform32_rounds_the_whole_word),
        ("ZE-EDEN codes", E.test_codes_are_nearest_zero_excluded_points),
        ("ZE-EDEN hand", E.test_factor_hand_computed_two_elements),
        ("ZE-EDEN grid", E.test_factor_is_one_on_the_grid),
        ("ZE-EDEN page formula", lambda: E.test_block_scale_equals_page_formula(128)),
        ("scalars", U.test_step_scalars_closed_form),
        ("final 10%", lambda: [U.test_final_ten_percent_phase(t, T, on) for t, T, on in
                               [(90, 100, False), (91, 100, True), (900, 1000, False),
                                (901, 1000, True)]]),
        ("torch AdamW", U.test_fp32_state_path_matches_torch_adamw),
        ("first step", U.test_update_elem_values),
        ("ordering", U.test_weights_updated_before_quantising),
        ("nibble layout", D.test_nibble_layout_of_the_codes),
        ("k/15 nearest", V.test_zi_rtn_is_nearest_code_point),
        ("k/15 state-space SR", lambda: [V.test_zi_sr_unbiased_by_enumeration(x)
                                         for x in (0.01, 0.2, 0.77)]),
        ("worked example, state space", lambda: V.test_worked_example_state_space_rounding(golden)),
        ("floor code", V.test_ze_floor_is_nearest_zero_excluded_without_rescale),
        ("bf16 library", BF.test_round_matches_the_library_conversion),
        ("bf16 nearest", BF.test_round_is_the_nearest_bf16_by_brute_force),
    ]


MUTANTS = [
    ("Philox multiplier", "#define PHILOX_M0 0xD2511F53u", "#define PHILOX_M0 0xD2511F55u"),
    ("Philox key bumped before the first round", "if (round > 0) {", "if (round >= 0) {"),
    ("Philox word from the wrong product", "uint32_t y0 = hi1 ^ x1 ^ k0;",
     "uint32_t y0 = hi0 ^ x1 ^ k0;"),
    ("draw counter words swapped", "(uint32_t)t,\n                       tensor_id * 2u + stream}",
     "tensor_id * 2u + stream,\n                       (uint32_t)t}"),
    ("uniform takes 24 bits", "(float)(word & 0x7FFFFFu) * 0x1p-23f",
     "(float)(word & 0xFFFFFFu) * 0x1p-23f"),
    ("ZIP-SR uniform scaled by 2^-31", "return (float)word * 0x1p-32f;",
     "return (float)word * 0x1p-31f;"),
    ("ZIP-SR uniform from the low 23 bits", "return (float)word * 0x1p-32f;",
     "return (float)(word & 0x7FFFFFu) * 0x1p-23f;"),
    ("ZIP-SR block step on the 23-bit uniform",
     "oracle_zipsr_decide(x, den[i], R, s->eps, oracle_uniform32(w))",
     "oracle_zipsr_decide(x, den[i], R, s->eps, oracle_uniform(w))"),
    ("NF4 offset", "const double offset = 0.9677083;", "const double offset = 0.96;"),
    ("NF4 negatives not normalised", "out[i] = neg[i] / top;", "out[i] = neg[i] / (top * 1.0001);"),
    ("first bias correction dropped", "s->step_size = (float)((double)lr / bc1);",
     "s->step_size = lr;"),
    ("second bias correction inverted", "s->rs_bc2 = (float)(1.0 / sqrt(bc2));",
     "s->rs_bc2 = (float)sqrt(bc2);"),
    ("eps inside the root", "float den = fmaf(sqrtf(v1), s->rs_bc2, s->eps);",
     "float den = sqrtf(fmaf(v1, s->rs_bc2 * s->rs_bc2, s->eps));"),
    ("gradient not squared", "s->omb2 * (g * g)", "s->omb2 * g"),
    ("beta1 weights swapped", "fmaf(s->b1, m0, s->omb1 * g)", "fmaf(s->omb1, m0, s->b1 * g)"),
    ("weight decay dropped", "float w1 = *w * decay;", "float w1 = *w;"),
    ("update sign", "*w = fmaf(-s->step_size, m1 / den, w1);",
     "*w = fmaf(s->step_size, m1 / den, w1);"),
    ("NF4 ties go high", "if (x > g_nf4_mid[j]) ++c;", "if (x >= g_nf4_mid[j]) ++c;"),
    ("state-space SR sides swapped", "return lower ? j : j + 1;", "return lower ? j + 1 : j;"),
    ("ZIP-SR sides swapped", "return lower ? k : k + 1;\n}\n\n/* ZE-EDEN",
     "return lower ? k + 1 : k;\n}\n\n/* ZE-EDEN"),
    ("k/15 state-space SR sides swapped",
     "(g_vz[k + 1] - x);\n    return lower ? k : k + 1;",
     "(g_vz[k + 1] - x);\n    return lower ? k + 1 : k;"),
    ("k/15 nearest ties go high", "if (x > g_vz_mid[k]) ++c;", "if (x >= g_vz_mid[k]) ++c;"),
    ("floor code rescaled", "oracle_zeeden_code(v1[i] * inv));\n        *vscale = av;",
     "oracle_zeeden_code(v1[i] * inv));\n        *vscale = av * 1.01f;"),
    ("ZIP-SR a and b swapped",
     "float da = fmaf(g_vz_sqrt[k], R, eps);\n    float db = fmaf(g_vz_sqrt[k + 1], R, eps);"
     "\n    int lower;",
     "float db = fmaf(g_vz_sqrt[k], R, eps);\n    float da = fmaf(g_vz_sqrt[k + 1], R, eps);"
     "\n    int lower;"),
    ("ZIP-SR probability in state space",
     "float lhs = u * ((db - da) * dv);\n        float rhs = (db - dv) * da;",
     "float lhs = u * (g_vz[k + 1] - g_vz[k]);\n        float rhs = g_vz[k + 1] - x;"),
    ("32-bit draw scaled by 2^-31", "double u = (double)w * 0x1p-32;",
     "double u = (double)w * 0x1p-31;"),
    ("32-bit decision sides swapped", "lower = u * (double)B < (double)rhs;",
     "lower = u * (double)B >= (double)rhs;"),
    ("ZIP-SR bracket excludes its lower end", "if (g_vz[i] <= x) k = i;",
     "if (g_vz[i] < x) k = i;"),
    ("ZE-EDEN code includes zero", "int k = (int)c - 1;", "int k = (int)c;"),
    ("ZE-EDEN factor inverted", "return sxx / fmaxf(sxq, 1e-12f);",
     "return sxq / fmaxf(sxx, 1e-12f);"),
    ("final 10% off by one", "(10 * t > 9 * total_steps)", "(10 * t >= 9 * total_steps)"),
    ("bf16 ties rounded up", "b += 0x7FFFu + ((b >> 16) & 1u);", "b += 0x8000u;"),
    ("bf16 truncated", "b += 0x7FFFu + ((b >> 16) & 1u);", "b += 0u;"),
    ("nibble order swapped",
     "return (i & 1) ? (codes[i >> 1] >> 4) : (codes[i >> 1] & 15);",
     "return (i & 1) ? (codes[i >> 1] & 15) : (codes[i >> 1] >> 4);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, old, new, tmp_path, golden_dir):
    src = oracle.source()
    assert src.count(old) == 1, f"mutation site not found once: {old!r}"
    path = oracle.build_variant(src.replace(old, new), str(tmp_path / "mutant.so"))
    failed = []
    with oracle.use_library(path):
        for pname, fn in pins(golden_dir):
            try:
                fn()
            except AssertionError:
                failed.append(pname)
    assert failed, f"no pin fails when the oracle has: {name}"


def test_unmutated_oracle_passes_every_pin(tmp_path, golden_dir):
    path = oracle.build_variant(oracle.source(), str(tmp_path / "same.so"))
    with oracle.use_library(path):
        for pname, fn in pins(golden_dir):
            fn()
