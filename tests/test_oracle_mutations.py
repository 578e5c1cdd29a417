"""Plant plausible mistakes in copies of the oracle and check the pins catch them.

Each mutant is a textual edit of ``oracle/oracle.c`` compiled into a
temporary library; the pin tests are then run against it and at least one
must fail.  The real oracle is untouched.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_fp8_pins as fp8pins
from tests import test_oracle_pins as pins

SRC = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()

MUTANTS = {
    "gqa_group_modulo": ("int g = h / r;", "int g = h % p->n_kv_head;"),
    "scale_dropped": ("double s = p->scale * dot;", "double s = dot;"),
    "causal_excludes_diagonal": ("int P = ctx + a;                                   /* absolute position */",
                                 "int P = ctx + a - (a > 0);"),
    "chunk_top_left_aligned": ("int P = ctx + a;", "int P = a;"),
    "softmax_sign_flipped": ("w[j] = exp(w[j] - m);", "w[j] = exp(m - w[j]);"),
    "k_and_v_swapped": ("const uint16_t *krow = kv_row(p, i, j, g, 0);",
                        "const uint16_t *krow = kv_row(p, i, j, g, 1);"),
    "wrong_kv_head_row": ("return base + (row * G + (size_t)g) * d;", "return base + (row * G) * d;"),
    "prefix_boundary_off_by_one": ("if (j >= ctx) {", "if (j > ctx) {"),
    "cache_slot_wrong": ("size_t slot = (size_t)(j % p->block_size);",
                         "size_t slot = (size_t)((j + 1) % p->block_size);"),
    "v_written_over_k": ("uint16_t *vd = kv_cache + (((size_t)page * 2 + 1)",
                         "uint16_t *vd = kv_cache + (((size_t)page * 2 + 0)"),
    "no_normalisation": ("for (int j = j0; j <= P; ++j) w[j] /= l;", "for (int j = j0; j <= P; ++j) w[j] /= 1.0;"),
    "value_column_fixed": ("out[x] += w[j] * bf16_bits_to_double(vrow[x]);",
                           "out[x] += w[j] * bf16_bits_to_double(vrow[0]);"),
    "window_excludes_self": ("j0 = P - p->window + 1;", "j0 = P - p->window + 2;"),
    "window_one_key_too_wide": ("j0 = P - p->window + 1;", "j0 = P - p->window;"),
    "window_ignored": ("if (p->window > 0 && P - p->window + 1 > 0)", "if (0)"),
    "window_from_chunk_row": ("if (p->window > 0 && P - p->window + 1 > 0) j0 = P - p->window + 1;",
                              "if (p->window > 0 && a - p->window + 1 > 0) j0 = a - p->window + 1;"),
    "e4m3_bias_off": ("return (uint8_t)(sign | (uint8_t)((E + 7) << 3) | (uint8_t)m);",
                      "return (uint8_t)(sign | (uint8_t)((E + 6) << 3) | (uint8_t)m);"),
    "e4m3_ties_away": ("double m = nearbyint((2.0 * f - 1.0) * 8.0);", "double m = round((2.0 * f - 1.0) * 8.0);"),
    "e4m3_no_saturation": ("if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
                           "if (a >= 1e30) return (uint8_t)(sign | 0x7E);"),
    "fp8_scale_multiplied": ("out[x] = oracle_e4m3_encode(v / scale);", "out[x] = oracle_e4m3_encode(v * scale);"),
    "fp8_v_scale_on_keys": ("kq[x] = oracle_e4m3_decode(kc[x]) * (double)k_scale[g];",
                            "kq[x] = oracle_e4m3_decode(kc[x]) * (double)v_scale[g];"),
    "chunk_fp8_top_left_aligned": ("int P = ctx + (t - c0); /* absolute position of the row */",
                                   "int P = (t - c0); /* absolute position of the row */"),
    "chunk_fp8_prefix_boundary_off_by_one": ("                if (j < ctx) {\n                    int lp = j / block_size;",
                                             "                if (j <= ctx) {\n                    int lp = j / block_size;"),
    "chunk_fp8_values_from_key_codes": ("vc = vc8 + ((size_t)(c0 + j - ctx) * G + (size_t)g) * d;",
                                        "vc = kc8 + ((size_t)(c0 + j - ctx) * G + (size_t)g) * d;"),
    "chunk_fp8_keys_quantized_with_v_scale": ("d, k_scale[g], kc8 + ((size_t)t * G + g) * d);",
                                              "d, v_scale[g], kc8 + ((size_t)t * G + g) * d);"),
}

# pins run against each mutant (the cheap ones; the byte-count pin is run separately)
PIN_CALLS = [
    lambda: pins.test_softmax_rows_sum_to_one([5, 70, 1], 6, 3, 32),
    lambda: pins.test_softmax_weights_chunked_sum_to_one(),
    lambda: pins.test_first_row_outputs_v0_exactly(),
    lambda: pins.test_identical_keys_give_prefix_mean(),
    lambda: pins.test_gqa_equals_mha_with_repeated_kv(8, 2),
    lambda: pins.test_brute_force_tiny([3, 7, 1], 2, 1, 3),
    lambda: pins.test_matches_torch_sdpa_fp64([300, 129, 2], 8, 2, 32),
    lambda: pins.test_chunk_matches_torch_sdpa_with_explicit_mask(),
    lambda: pins.test_chunked_equals_unchunked(100, 16),
    lambda: pins.test_block_table_invariance_and_gather(),
    lambda: pins.test_chunk_prefix_read_through_table(),
    lambda: pins.test_window_one_outputs_own_value_exactly(),
    lambda: pins.test_window_matches_torch_sdpa_band_mask([300, 129, 2], 64),
    lambda: pins.test_window_chunk_matches_torch_sdpa_band_mask(),
    lambda: fp8pins.test_code_table_values(),
    lambda: fp8pins.test_every_finite_code_round_trips(),
    lambda: fp8pins.test_midpoints_round_to_the_even_code(),
    lambda: fp8pins.test_saturation(),
    lambda: fp8pins.test_kv_write_fp8_bytes_and_untouched_slots(),
    lambda: fp8pins.test_decode_fp8_empty_context_returns_dequantized_value(),
    lambda: fp8pins.test_decode_fp8_close_to_bf16_attention(),
    lambda: fp8pins.test_decode_fp8_equals_bf16_definition_when_values_are_exact(),
    lambda: fp8pins.test_chunked_fp8_one_row_chunks_equal_decode(),
    lambda: fp8pins.test_chunked_fp8_exact_values_equal_bf16_definition(),
    lambda: fp8pins.test_chunked_fp8_split_invariance(),
]


def _all_pins_pass() -> bool:
    for call in PIN_CALLS:
        try:
            call()
        except (AssertionError, RuntimeError):
            return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) >= 1, f"mutation anchor for {name} not found"
    src = tmp_path / "oracle_mutant.c"
    src.write_text(SRC.replace(old, new, 1))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(src), "-o", str(lib), "-lm"])
    handle = oracle._swap_library(str(lib))
    try:
        assert not _all_pins_pass(), f"mutant {name} passed every pin"
    finally:
        oracle._restore_library(handle)


def test_unmutated_copy_passes(tmp_path):
    src = tmp_path / "oracle_copy.c"
    src.write_text(SRC)
    lib = tmp_path / "liboracle_copy.so"
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(src), "-o", str(lib), "-lm"])
    handle = oracle._swap_library(str(lib))
    try:
        assert _all_pins_pass()
    finally:
        oracle._restore_library(handle)
