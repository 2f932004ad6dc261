"""Plant plausible mistakes in a COPY of the oracle source and check that the
pins of test_oracle.py catch every one of them (the oracle itself is never
edited; each mutant is compiled into a temporary library)."""
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dsa_oracle.c")

# (name, text in the oracle, mistaken replacement)
MUTANTS = [
    ("no_relu_gate", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    ("tie_break_reversed", "return (a->pos > b->pos) - (a->pos < b->pos);",
     "return (a->pos < b->pos) - (a->pos > b->pos);"),
    ("head_weight_transposed", "acc += (double)a->w[(int64_t)t * H + h] * relu;",
     "acc += (double)a->w[(int64_t)t * H + (H - 1 - h)] * relu;"),
    ("scale_group_swapped", "double sc = (double)a->k_scale[row * (a->D_I / 64) + d / 64];",
     "double sc = (double)a->k_scale[row * (a->D_I / 64) + (a->D_I / 64 - 1 - d / 64)];"),
    ("key_without_rope", "for (int d = 0; d < ORACLE_DQK; d++) dot += bf16_to_f64(qg[d])",
     "for (int d = 0; d < ORACLE_DV; d++) dot += bf16_to_f64(qg[d])"),
    ("lse_without_log", "out_lse[(int64_t)i * a->H + g] = m + log(den);",
     "out_lse[(int64_t)i * a->H + g] = m + den;"),
    ("causal_off_by_one", "for (int64_t s = 0; s <= pos; s++) {", "for (int64_t s = 0; s < pos; s++) {"),
    ("pad_with_zero", "out_idx[o] = j < nk ? (int32_t)keep[j] : -1;",
     "out_idx[o] = j < nk ? (int32_t)keep[j] : 0;"),
    ("e4m3_bias_8", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("pair_score_without_relu", "acc += (double)a->w[(int64_t)t * a->H_I + h] * (dot > 0.0 ? dot : 0.0);",
     "acc += (double)a->w[(int64_t)t * a->H_I + h] * dot;"),
    ("pair_score_weight_transposed", "acc += (double)a->w[(int64_t)t * a->H_I + h] * (dot > 0.0 ? dot : 0.0);",
     "acc += (double)a->w[(int64_t)t * a->H_I + (a->H_I - 1 - h)] * (dot > 0.0 ? dot : 0.0);"),
    ("pair_score_causal_edge", "if (s < 0 || s > pos) { out[i] = NAN; continue; }",
     "if (s < 0 || s >= pos) { out[i] = NAN; continue; }"),
    ("softmax_value_from_rope", "for (int d = 0; d < ORACLE_DV; d++) o[d] += p * kv_elem(a, rows[j], d);",
     "for (int d = 0; d < ORACLE_DV; d++) o[d] += p * kv_elem(a, rows[j], d + 64);"),
    ("mx_key_group_of_64", "oracle_e8m0_to_f64(e[row * (a->D_I / 32) + d / 32]);",
     "oracle_e8m0_to_f64(e[row * (a->D_I / 32) + d / 64]);"),
    ("mx_query_group_of_64", "oracle_e8m0_to_f64(a->q_scale[((int64_t)t * a->H_I + h) * (a->D_I / 32) + d / 32]);",
     "oracle_e8m0_to_f64(a->q_scale[((int64_t)t * a->H_I + h) * (a->D_I / 32) + d / 64]);"),
    ("e8m0_bias_126", "return ldexp(1.0, (int)e - 127);", "return ldexp(1.0, (int)e - 126);"),
    ("prolog_rms_sum_not_mean", "ms /= (double)a->D_I;", "ms /= 1.0;"),
    ("prolog_eps_outside_sqrt", "double r = 1.0 / sqrt(ms + a->eps);", "double r = 1.0 / (sqrt(ms) + a->eps);"),
    ("prolog_gamma_reversed", "k_out[(int64_t)t * a->D_I + i] = p[HD + i] * r * (double)a->gamma[i];",
     "k_out[(int64_t)t * a->D_I + i] = p[HD + i] * r * (double)a->gamma[a->D_I - 1 - i];"),
    ("prolog_weight_rows_shifted", "w_out[(int64_t)t * a->H_I + h] = p[HD + a->D_I + h];",
     "w_out[(int64_t)t * a->H_I + h] = p[HD + h];"),
    ("prolog_x_transposed", "acc += bf16_to_f64(a->x[(int64_t)t * a->d + c])",
     "acc += bf16_to_f64(a->x[(int64_t)(a->T - 1 - t) * a->d + c])"),
    ("e4m3_ties_away", "if (d < bd || (d == bd && (c & 1) == 0 && (best & 1) == 1))", "if (d <= bd)"),
    ("mx_scale_minus_7", "e = ex - 1 - 8;", "e = ex - 1 - 7;"),
    ("mx_zero_group_scale", "int e = 0;\n        if (amax > 0.0) {", "int e = -127;\n        if (amax > 0.0) {"),
    ("kv_fp8_tile_shifted", "* (double)a->kv_scale[row * 5 + d / 128];",
     "* (double)a->kv_scale[row * 5 + (d / 128 + 1) % 5];"),
    ("kv_fp8_scale_row_stride", "* (double)a->kv_scale[row * 5 + d / 128];", "* (double)a->kv_scale[row * 4 + d / 128];"),
    ("fp8_group_scale_over_240", "float sc = amax > 0.0 ? (float)(amax / 448.0) : 1.0f;",
     "float sc = amax > 0.0 ? (float)(amax / 240.0) : 1.0f;"),
]

PINS = [pins.test_hand_indexer_relu_gate_weights_and_tie, pins.test_hand_fp8_scale_groups,
        pins.test_hand_score_pairs, lambda: pins.test_score_pairs_match_full_score_rows(dict(key_dtype="bf16")),
        pins.test_hand_softmax_two_rows, pins.test_e4m3_decode_all_codes_vs_torch,
        pins.test_single_head_unit_weight_is_relu_dot_lexsort,
        pins.test_k_at_least_context_equals_dense_causal_attention, pins.test_hand_mxfp8_groups,
        pins.test_e8m0_decode_all_exponents_vs_torch, pins.test_hand_indexer_prolog,
        pins.test_prolog_projection_matches_numpy_matmul, pins.test_prolog_key_matches_torch_rms_norm,
        pins.test_hand_mx_encode_group, pins.test_e4m3_encode_matches_torch_cast_including_ties_and_saturation,
        pins.test_mx_encode_scale_rule_and_error_bound, pins.test_fp8_group_encode_scale_is_amax_over_448,
        pins.test_hand_fp8_latent_rows, pins.test_fp8_latent_rows_equal_the_bf16_rows_they_encode]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(mutant_c), "-lm"])
    caught = []
    with oracle.swapped_library(str(so)):
        for pin in PINS:
            try:
                pin()
            except AssertionError:
                caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"no pin caught the planted mistake {name}"
