"""The pins must catch plausible slips in the oracle.

Each case copies the oracle's C source to a temporary directory, plants one mistake by a
text substitution, builds that copy with gcc and runs the pin tests against it: at least
one pin has to fail.  The committed oracle is never modified and no GPU is involved.
"""
import os
import shutil
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lora_oracle.c")

MUTATIONS = {
    "transposed_A": ("acc += xrow[j] * widen(A[i], dtype, (int64_t)k * h + j)",
                     "acc += xrow[j] * widen(A[i], dtype, (int64_t)j * r + k)"),
    "transposed_B": ("widen(B[i], dtype, n * r + k) * v[k];\n                yr[n] += scales[i] * acc;",
                     "widen(B[i], dtype, (int64_t)k * o + n) * v[k];\n                yr[n] += scales[i] * acc;"),
    "dropped_y0": ("yr[n] = widen(y0, dtype, t * ldy + y_offset + n);\n            int32_t i = ids[t];\n"
                   "            if (i < 0)\n                continue;\n            int32_t r = ranks[i];\n"
                   "            if (r > vcap)",
                   "yr[n] = 0.0;\n            int32_t i = ids[t];\n"
                   "            if (i < 0)\n                continue;\n            int32_t r = ranks[i];\n"
                   "            if (r > vcap)"),
    "scale_squared": ("yr[n] += scales[i] * acc;\n            }\n        }\n        free(v);",
                      "yr[n] += scales[i] * scales[i] * acc;\n            }\n        }\n        free(v);"),
    "scale_dropped": ("yr[n] += scales[i] * acc;\n            }\n        }\n        free(v);",
                      "yr[n] += acc;\n            }\n        }\n        free(v);"),
    "neighbour_id": ("int32_t i = ids[t];\n            if (i < 0)\n                continue;\n"
                     "            int32_t r = ranks[i];\n            if (r > vcap)",
                     "int32_t i = ids[(t + 1) % T];\n            if (i < 0)\n                continue;\n"
                     "            int32_t r = ranks[i];\n            if (r > vcap)"),
    "rank_off_by_one": ("for (int32_t k = 0; k < r; ++k) {\n                double acc = 0.0;\n                for (int64_t j = 0; j < h; ++j)\n                    acc += xrow[j]",
                        "for (int32_t k = 0; k < r - 1; ++k) {\n                double acc = 0.0;\n                for (int64_t j = 0; j < h; ++j)\n                    acc += xrow[j]"),
    "unstable_segments": ("for (int64_t t = 0; t < T; ++t)\n        if (ids[t] >= 0)\n            perm[next[ids[t]]++]",
                          "for (int64_t t = T - 1; t >= 0; --t)\n        if (ids[t] >= 0)\n            perm[next[ids[t]]++]"),
    "offset_ignored": ("widen(y0, dtype, t * ldy + y_offset + n);\n            int32_t i = ids[t];\n"
                       "            if (i < 0)\n                continue;\n            int32_t r = ranks[i];\n"
                       "            if (r > vcap)",
                       "widen(y0, dtype, t * ldy + n);\n            int32_t i = ids[t];\n"
                       "            if (i < 0)\n                continue;\n            int32_t r = ranks[i];\n"
                       "            if (r > vcap)"),
    "merge_weight_dropped": ("yr[n] += wt * (scales[i] * acc);", "yr[n] += scales[i] * acc;"),
    "merge_first_slot_only": ("for (int32_t j = 0; j < K; ++j) {\n                int32_t i = ids[t * K + j];",
                              "for (int32_t j = 0; j < 1; ++j) {\n                int32_t i = ids[t * K + j];"),
    "merge_wrong_weight": ("double wt = (double)w[t * K + j];", "double wt = (double)w[t * K];"),
    "sigma_transposed": ("acc += (double)S[(int64_t)k * r + m] * u[m];", "acc += (double)S[(int64_t)m * r + k] * u[m];"),
    "sigma_full_skipped": ("            w[k] = acc;\n        } else if", "            w[k] = u[k];\n        } else if"),
    "sigma_diag_skipped": ("w[k] = (double)S[k] * u[k];", "w[k] = u[k];"),
    "sigma_scale_dropped": ("yr[n] += scales[i] * acc;\n            }\n        }\n        free(u);",
                            "yr[n] += acc;\n            }\n        }\n        free(u);"),
    "base_W_transposed": ("acc += widen(W, dtype, n * ldw + j) * xr[j];",
                          "acc += widen(W, dtype, j * o + n) * xr[j];"),
    "base_A_transposed": ("su += xr[j] * widen(A[i], dtype, (int64_t)m * h + j);",
                          "su += xr[j] * widen(A[i], dtype, (int64_t)j * ri + m);"),
    "base_delta_scale_dropped": ("yr[n] += scales[i] * sd;", "yr[n] += sd;"),
    "base_term_dropped": ("                yr[n] += acc;\n            }\n            int32_t i = ids[t];",
                          "                (void)acc;\n            }\n            int32_t i = ids[t];"),
    "base_accumulate_ignored": ("yr[n] = accumulate ? widen(y0, dtype, t * ldy + y_offset + n) : 0.0;",
                                "yr[n] = widen(y0, dtype, t * ldy + y_offset + n);"),
    "base_skipped_without_adapter": ("/* base product: y += W x */\n            for (int64_t n = 0; n < o; ++n) {",
                                     "/* base product: y += W x */\n            for (int64_t n = 0; n < o && ids[t] >= 0; ++n) {"),
}

PIN_TESTS = [
    lambda: [pins.test_loop_matches_grouped_matrix_products(n, d)
             for n in ("tiny_sgmv", "multirank_decode") for d in (False, True)],
    lambda: pins.test_single_adapter_equals_merged_weight("tiny_sgmv"),
    lambda: [pins.test_selection_matrices_closed_form("f32", *s) for s in [(8, 8, 8), (24, 8, 16)]],
    pins.test_rank_one_closed_form,
    lambda: pins.test_zero_B_or_zero_scale_leaves_y_unchanged("B"),
    pins.test_delta_linear_in_scale,
    pins.test_mixed_ranks_equal_per_adapter_runs,
    pins.test_output_slice_offset,
    pins.test_exhaustive_tiny_against_outer_products,
    lambda: [pins.test_segments_equal_stable_argsort(s) for s in (1, 2)],
    lambda: [pins.test_sigma_identity_is_the_plain_delta(k) for k in ("full", "diag")],
    pins.test_sigma_diagonal_of_powers_of_two_folds_into_B,
    lambda: [pins.test_sigma_equals_merged_three_factor_weight(k) for k in ("full", "diag")],
    pins.test_sigma_shrink_is_sigma_times_shrink,
    pins.test_merged_single_slot_unit_weight_is_the_plain_delta,
    pins.test_merged_equals_merged_weight_closed_form,
    pins.test_merged_slot_order_and_duplicate_slots,
    lambda: [pins.test_sigma_loop_matches_grouped_products(k, d) for k in ("full", "diag") for d in (False, True)],
    lambda: [pins.test_merged_loop_matches_grouped_products(d) for d in (False, True)],
    pins.test_base_with_zero_weight_is_the_delta,
    pins.test_base_single_adapter_equals_merged_weight,
    pins.test_base_rows_without_adapter_and_accumulate_flag,
    lambda: [pins.test_base_selection_matrix_closed_form(h, o) for h, o in ((24, 16), (16, 40))],
    pins.test_base_linear_in_weight_and_matches_grouped_products,
]


@pytest.mark.parametrize("mut", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(mut, tmp_path):
    old, new = MUTATIONS[mut]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor not unique: %s" % mut
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = str(tmp_path / ("libmut_%s.so" % mut))
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-std=c99", "-o", so, str(path)])
    saved = oracle._load()
    oracle._lib = oracle.bind(so)
    failures = 0
    try:
        for pin in PIN_TESTS:
            try:
                pin()
            except (AssertionError, oracle.OracleError, ValueError):
                failures += 1
    finally:
        oracle._lib = saved
    assert failures > 0, "no pin caught the planted mistake %s" % mut
