"""The pins are strong enough: plausible mistakes planted in a copy of the
oracle (compiled on the CPU, never run on a GPU) each fail at least one pin."""
import os

import pytest

import oracle
from oracle_pins import ALL_CHECKS

# (name, text in oracle.c, replacement): each is a mistake someone could make.
# "ReLU keeps -0" (">= 0" in place of "> 0") is not listed: a sum that starts
# at +0 and rounds to nearest can never be -0 (x + (-x) is +0), so that change
# computes the same function.
MUTANTS = [
    ("transposed_B", "acc[j] = acc[j] + a * brow[j];", "acc[j] = acc[j] + a * Bf[j * K + k];"),
    ("transposed_A", "oracle_f16_to_f32(A[i * K + k])", "oracle_f16_to_f32(A[k * M + i])"),
    ("dropped_last_k", "for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = 0; k + 1 < K; ++k) {"),
    ("relu_missing", "acc[j] > 0.0f ? acc[j] : 0.0f", "acc[j]"),
    ("truncate_not_round", "if (r > 0.5 || (r == 0.5 && fmod(qi, 2.0) != 0.0))", "if (0)"),
    ("ties_away_from_zero", "(r == 0.5 && fmod(qi, 2.0) != 0.0)", "(r == 0.5)"),
    ("wrong_subnormal_quantum", "subnormal ? -24 : e - 10", "subnormal ? -25 : e - 10"),
    ("wrong_f16_bias", "ldexpf((float)(1024 + frac), expo - 25)", "ldexpf((float)(1024 + frac), expo - 24)"),
    ("no_overflow_to_inf", "if (e > 15)", "if (e > 16)"),
    ("ex_weight_layout_ignored", "b_nk ? B[j * ldb + k] : B[k * ldb + j]", "B[k * ldb + j]"),
    ("ex_bias_dropped", "bias ? acc[j] + oracle_f16_to_f32(bias[j]) : acc[j]", "acc[j]"),
    ("ex_bias_after_relu", "const float v = y > 0.0f ? y : 0.0f;",
     "const float v = (acc[j] > 0.0f ? acc[j] : 0.0f) + (bias ? oracle_f16_to_f32(bias[j]) : 0.0f);"),
    ("ex_transposed_a_ignored", "a_km ? A[k * lda + i] : A[i * lda + k]", "A[i * lda + k]"),
    ("ex_ldc_ignored", "C[i * ldc + j] = oracle_f32_to_f16_rne(v);", "C[i * N + j] = oracle_f32_to_f16_rne(v);"),
    ("e4m3_nan_as_number", "if (e == 15 && m == 7)", "if (0)"),
    ("e4m3_wrong_bias", "ldexp((double)(8 + m), e - 10)", "ldexp((double)(8 + m), e - 9)"),
    ("e5m2_wrong_subnormal", "ldexp((double)m, -16)", "ldexp((double)m, -15)"),
    ("ue8m0_wrong_bias", "ldexp(1.0, (int)e - 127)", "ldexp(1.0, (int)e - 128)"),
    ("bf16_wrong_quantum", "subnormal ? -133 : e - 7", "subnormal ? -133 : e - 8"),
    ("bf16_no_overflow", "if (e > 127)", "if (e > 128)"),
    ("mx_block_index_ignored", "SFA[r * S + k / 32]", "SFA[r * S]"),
    ("mx_b_not_transposed", "B[brow * K + k]", "B[(int64_t)g * N * K + k * N + j]"),
    ("mx_group_ignored", "const int64_t brow = (int64_t)g * N + j;", "const int64_t brow = j;"),
    ("mx_relu_ignored", "relu ? (acc > 0.0 ? acc : 0.0) : acc", "acc"),
    ("mx_scale_b_dropped", "* oracle_ue8m0_to_f64(SFB[brow * S + k / 32])", ""),
    ("e2m1_wrong_bias", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e - 2)"),
    ("e2m1_no_subnormal_half", "e == 0 ? 0.5 * m :", "e == 0 ? 1.0 * m :"),
    ("nvf4_nibbles_swapped", "hi ? (uint8_t)(abyte >> 4) : (uint8_t)(abyte & 0xf)",
     "hi ? (uint8_t)(abyte & 0xf) : (uint8_t)(abyte >> 4)"),
    ("nvf4_block_32", "oracle_ue4m3_to_f64(SFA[r * S + k / 16])", "oracle_ue4m3_to_f64(SFA[r * S + k / 32])"),
    ("nvf4_alpha_ignored", "const double y = alpha * acc;", "const double y = acc;"),
    ("nvf4_scale_b_dropped", "oracle_ue4m3_to_f64(SFB[brow * S + k / 16])", "1.0"),
    ("nvf4_group_ignored", "const int64_t brow = (int64_t)g * N + j;\n                double acc = 0.0;\n                for (int64_t k = 0; k < K; ++k) {\n                    const int hi",
     "const int64_t brow = j;\n                double acc = 0.0;\n                for (int64_t k = 0; k < K; ++k) {\n                    const int hi"),
    ("w4_zero_point_7", "(float)(q - 8) * scale", "(float)(q - 7) * scale"),
    ("w4_nibbles_swapped", "const int q = (k & 1) ? (byte >> 4) : (byte & 0xf);",
     "const int q = (k & 1) ? (byte & 0xf) : (byte >> 4);"),
    ("w4_group_index", "S[n * G + k / group]", "S[n * G + k / (2 * group)]"),
    ("w4_scale_row_ignored", "S[n * G + k / group]", "S[k / group]"),
    ("fp64_accumulator", "float *acc = (float *)malloc((size_t)N * sizeof(float));",
     "double *acc = (double *)malloc((size_t)N * sizeof(double));"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    src = oracle.source_text()
    # Mutate the first occurrence: the base function comes first in the file;
    # mutations of the general-layout function use text found only there.
    assert old in src, f"mutation site for {name} not found"
    lib = oracle.load_library(oracle.compile_variant(src.replace(old, new, 1),
                                                     os.path.join(tmp_path, f"lib{name}.so")))
    failed = []
    for check in ALL_CHECKS:
        try:
            check(lib)
        except AssertionError:
            failed.append(check.__name__)
    assert failed, f"no pin catches the planted mistake {name}"
