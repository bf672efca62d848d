"""The pins catch plausible mistakes in the oracle.

Each case copies the oracle's C source, plants one mistake (wrong head map,
wrong block index, transposed cache index, dropped scale, wrong merge sign,
...), builds the copy on the CPU and checks that at least one pin of
test_oracle_pins fails against it. The real oracle is untouched.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins
import test_oracle_prefill as prefill_pins
import test_oracle_qkv as qkv_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")

MUTATIONS = {
    "head_map_modulo": ("int g = h / G;                                  /* R1 */",
                        "int g = h % Hkv;"),
    "block_index_swapped": ("int32_t phys = bt_row[t / block_size];",
                            "int32_t phys = bt_row[t % block_size];"),
    "cache_index_transposed": ("int64_t idx = (slot * Hkv + g) * D + d;",
                               "int64_t idx = (slot * D + d) * Hkv + g;"),
    "scale_dropped": ("s[t - t0] = scale * dot;", "s[t - t0] = dot;"),
    "merge_sign": ("double w = lp[p] * exp(mp[p] - M);", "double w = lp[p] * exp(M - mp[p]);"),
    "merge_drops_l": ("double w = lp[p] * exp(mp[p] - M);", "double w = exp(mp[p] - M);"),
    "no_normalise": ("for (int d = 0; d < D; ++d) o[d] /= l;", ";"),
    "last_token_dropped": ("for (int t = t0; t < t1; ++t) {\n        double p = exp",
                           "for (int t = t0; t < t1 - (t1 > t0 + 1); ++t) {\n        double p = exp"),
    "fp8_scale_ignored": ("if (kv_fp8) return oracle_e4m3_to_f64(((const uint8_t*)cache)[idx]) * scale;",
                          "if (kv_fp8) return oracle_e4m3_to_f64(((const uint8_t*)cache)[idx]);"),
    "e4m3_bias_off_by_one": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    "e4m3_ties_away": ("double r = rint(a / quantum) * quantum;",
                       "double r = floor(a / quantum + 0.5) * quantum;"),
    "cache_write_row": ("int64_t blk = s / block_size, row = s % block_size;",
                        "int64_t blk = s / block_size, row = (s + 1) % block_size;"),
    # fused residual add + RMSNorm + QKV projection
    "f16_ties_away": ("double r = quantum * rint(a / quantum);",
                      "double r = quantum * floor(a / quantum + 0.5);"),
    "f16_overflow_early": ("if (a >= 65520.0) return sign | 0x7C00;",
                           "if (a > 65504.0) return sign | 0x7C00;"),
    "residual_unrounded": ("y[k] = oracle_f16_to_f64(s16);", "y[k] = sum;"),
    "rms_mean_off_by_one": ("double inv_rms = 1.0 / sqrt(sumsq / H + eps);",
                            "double inv_rms = 1.0 / sqrt(sumsq / (H + 1) + eps);"),
    "rms_eps_dropped": ("double inv_rms = 1.0 / sqrt(sumsq / H + eps);",
                        "double inv_rms = 1.0 / sqrt(sumsq / H);"),
    "gamma_dropped": ("y[k] = y[k] * inv_rms * oracle_f16_to_f64(gamma[k]);", "y[k] = y[k] * inv_rms;"),
    "weight_transposed": ("acc += oracle_f16_to_f64(wr[k]) * y[k];",
                          "acc += oracle_f16_to_f64(w[(int64_t)k * N + n]) * y[k];"),
    "bias_dropped": ("if (bias) acc += oracle_f16_to_f64(bias[n]);", ";"),
    # paged prefill
    "prefill_causal_off_by_one": ("0, pos + 1)) {", "0, pos + (pos == 0))) {"),
    "prefill_position_from_start": ("int pos = L - n + i;", "int pos = i;"),
    "prefill_rows_reversed": ("const int i = (int)(row - query_start[b]);",
                              "const int i = (int)(query_start[b + 1] - 1 - row);"),
}

PIN_TESTS = [
    lambda: pins.test_e4m3_decode_all_codes_matches_torch(),
    lambda: pins.test_e4m3_round_matches_bruteforce_and_torch(),
    lambda: pins.test_e4m3_round_saturation_and_ties(),
    lambda: pins.test_cache_write_touches_only_target_slots("f16"),
    lambda: pins.test_cache_write_touches_only_target_slots("fp8"),
    lambda: pins.test_decode_matches_dense_bruteforce(12, 2, 0),
    lambda: pins.test_fp8_decode_matches_dense_on_dequantised_values(),
    lambda: pins.test_worked_example_closed_form(),
    lambda: pins.test_split_merge_equals_single_pass(8),
    lambda: pins.test_head_map_contiguous_groups(),
    lambda: qkv_pins.test_f16_rounding_ties_and_limits(),
    lambda: qkv_pins.test_residual_add_rounds_once_to_nearest_even(),
    lambda: qkv_pins.test_worked_example_by_hand(),
    lambda: qkv_pins.test_constant_row_and_eps(),
    lambda: qkv_pins.test_unit_rows_select_the_normalised_stream(),
    lambda: qkv_pins.test_qkv_split_follows_the_row_order(),
    lambda: prefill_pins.test_one_query_per_sequence_is_decode(),
    lambda: prefill_pins.test_matches_dense_causal_bruteforce([3, 1, 7, 40, 2]),
    lambda: prefill_pins.test_later_positions_do_not_reach_earlier_queries(),
]


def _build_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique/found"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(old, new))
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                    "-o", str(lib), str(path), "-lm"], check=True)
    return str(lib)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    lib_path = _build_mutant(tmp_path, name, *MUTATIONS[name])
    saved_lib, saved_build = oracle._lib, oracle.build
    try:
        oracle._lib = None
        oracle.build = lambda force=False: lib_path
        oracle._load()
        caught = 0
        for pin in PIN_TESTS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught += 1
        assert caught > 0, f"no pin caught mutation {name}"
    finally:
        oracle._lib, oracle.build = saved_lib, saved_build


def test_unmutated_copy_passes_every_pin(tmp_path):
    lib_path = _build_mutant(tmp_path, "identity", "/* R1 */", "/* R1 */")
    saved_lib, saved_build = oracle._lib, oracle.build
    try:
        oracle._lib = None
        oracle.build = lambda force=False: lib_path
        oracle._load()
        for pin in PIN_TESTS:
            pin()
    finally:
        oracle._lib, oracle.build = saved_lib, saved_build
