"""Mutation tests: the oracle pins must catch plausible slips in the oracle.

Each mutant is a copy of ``oracle/bq_oracle.c`` with one small change of the
kind the pins are meant to catch (a swapped nibble, a wrong tie rule, a wrong
index, a dropped term, an off-by-one tail...).  It is compiled on the CPU into
a temporary library, swapped in for the real oracle, and at least one pin must
then fail.  Nothing here touches a GPU.
"""
import os
import shutil

import pytest

import oracle
from oracle import build as obuild

import test_oracle_pins as pins

SRC = open(obuild.SRC).read()

# (name, original text, replacement, pins expected to notice it)
MUTANTS = [
    ("swap_nibbles",
     "out[i >> 1] |= (uint8_t)(idx << 4);   /* element 2i: high nibble */",
     "out[i >> 1] |= (uint8_t)idx;   /* element 2i: high nibble */"),
    ("ties_go_high", "if (d < best) {", "if (d <= best) {"),
    ("tail_off_by_one",
     "int64_t hi = lo + blocksize < n ? lo + blocksize : n;",
     "int64_t hi = lo + blocksize < n ? lo + blocksize : n - 1;"),
    ("absmax_reversed", "absmax[b] = A;", "absmax[nb - 1 - b] = A;"),
    ("absmax_no_abs", "A = fmaxf(A, fabsf(load_elem(x, dtype, i)));",
     "A = fmaxf(A, load_elem(x, dtype, i));"),
    ("division_transposed", "0.0f : v / A;", "0.0f : A / v;"),
    ("distance_no_abs", "float d = fabsf(xn - code[j]);", "float d = xn - code[j];"),
    ("dequant_nibbles_swapped", "idx = (i & 1) ? (q[i >> 1] & 15) : (q[i >> 1] >> 4);",
     "idx = (i & 1) ? (q[i >> 1] >> 4) : (q[i >> 1] & 15);"),
    ("dequant_absmax_index", "code[idx] * absmax[i / blocksize];",
     "code[idx] * absmax[(i + 1) / blocksize];"),
    ("q8_unsigned", "int qv = (int)(int8_t)blk[2 + j];", "int qv = (int)blk[2 + j];"),
    ("q4_nibbles_swapped", "int lo = blk[2 + j] & 15;", "int lo = blk[2 + j] >> 4;"),
    ("q4_no_offset", "d * (float)(lo - 8)", "d * (float)(lo)"),
    ("q4_1_min_dropped", "d * (float)lo + m);", "d * (float)lo);"),
    ("q5_qh_bit_order", "(((qh >> e) & 1u) << 4)", "(((qh >> (31 - e)) & 1u) << 4)"),
    ("q5_0_offset", "(float)(q5_value(blk + 6, qh, e) - 16)", "(float)(q5_value(blk + 6, qh, e) - 15)"),
    ("q5_1_qh_offset", "uint32_t qh = u32_at(blk + 4);", "uint32_t qh = u32_at(blk + 2);"),
    ("q4k_scale_min_nibbles", "*scale = (sc[i + 4] & 15) | ((sc[i - 4] >> 6) << 4);",
     "*scale = (sc[i + 4] >> 4) | ((sc[i - 4] >> 6) << 4);"),
    ("q4k_top_bits_source", "*mn = (sc[i + 4] >> 4) | ((sc[i] >> 6) << 4);",
     "*mn = (sc[i + 4] >> 4) | ((sc[i - 4] >> 6) << 4);"),
    ("q4k_nibble_halves", "int q = h ? (qs[32 * g + l] >> 4) : (qs[32 * g + l] & 15);",
     "int q = h ? (qs[32 * g + l] & 15) : (qs[32 * g + l] >> 4);"),
    ("q6k_offset", "int q = (lo4 | (hi2 << 4)) - 32;", "int q = (lo4 | (hi2 << 4)) - 31;"),
    ("q6k_scale_index", "sc[8 * n + l / 16 + 2 * c]", "sc[8 * n + l / 16 + c]"),
    ("q6k_qh_shift", "int hi2 = (qh[32 * n + l] >> (2 * c)) & 3;", "int hi2 = (qh[32 * n + l] >> c) & 3;"),
    ("q2k_scale_min_swapped",
     "float a = d * (float)(scales[j] & 15), b = dmin * (float)(scales[j] >> 4);",
     "float a = d * (float)(scales[j] >> 4), b = dmin * (float)(scales[j] & 15);"),
    ("q2k_shift", "int q = (qs[32 * n + 16 * h + l] >> (2 * c)) & 3;",
     "int q = (qs[32 * n + 16 * h + l] >> c) & 3;"),
    ("q3k_hmask_polarity", "int q = low - (hb ? 0 : 4);", "int q = low - (hb ? 4 : 0);"),
    ("q3k_top_bits", "int hi = (sc[8 + (i & 3)] >> (2 * (i >> 2))) & 3;",
     "int hi = (sc[8 + (i >> 2)] >> (2 * (i & 3))) & 3;"),
    ("q3k_no_offset", "return (lo | (hi << 4)) - 32;", "return (lo | (hi << 4));"),
    ("q5k_qh_bit", "int q = nib | (((qh[l] >> (2 * g + h)) & 1) << 4);",
     "int q = nib | (((qh[l] >> (g + h)) & 1) << 4);"),
    ("q8_enc_divisor", "float d = amax / 127.0f;", "float d = amax / 128.0f;"),
    ("q8_enc_round_half_even", "float r = roundf(load_elem(x, dtype, 32 * k + j) * id);",
     "float r = rintf(load_elem(x, dtype, 32 * k + j) * id);"),
    ("q4_enc_last_tie_wins", "if (fabsf(v) > amax) {", "if (fabsf(v) >= amax) {"),
    ("q4_enc_abs_max", "float d = m / -8.0f;", "float d = amax / -8.0f;"),
    ("q4_enc_no_half", "* id + 8.5f);", "* id + 8.0f);"),
    ("q4_enc_nibble_order", "blk[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4));",
     "blk[2 + j] = (uint8_t)((q[j] << 4) | q[j + 16]);"),
    ("f16_bias", "ldexpf((float)(m + 1024), e - 25)", "ldexpf((float)(m + 1024), e - 24)"),
    ("bf16_ties_away", "if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))",
     "if (lower >= 0x8000u)"),
    ("f16_ties_away", "if (rem > 0x1000u || (rem == 0x1000u && (h & 1u)))",
     "if (rem >= 0x1000u)"),
]


def _all_pins():
    """The pin checks, as zero-argument callables."""
    checks = [
        pins.test_f16_widen_matches_numpy_all_patterns,
        pins.test_bf16_widen_matches_torch_all_patterns,
        pins.test_f32_to_f16_matches_numpy_rne,
        pins.test_f32_to_bf16_matches_torch_rne,
        pins.test_gguf_hand_worked_blocks,
        pins.test_gguf_matches_gguf_package,
        pins.test_gguf_encode_hand_worked_blocks,
        pins.test_gguf_encode_matches_gguf_package,
        pins.test_nearest_code_ties_go_low,
        pins.test_quantize_hand_worked_packing,
        lambda: pins.test_nearest_code_brute_force("nf4"),
        lambda: pins.test_nearest_code_brute_force("fp4"),
        lambda: pins.test_quantize_absmax_and_codes_reference("bf16", 64),
        lambda: pins.test_quantize_absmax_and_codes_reference("f32", 32),
        lambda: pins.test_round_trip_every_entry("nf4"),
        lambda: pins.test_all_zero_block("fp4", 7),
        lambda: pins.test_dequantize_is_one_product_then_narrow("f32"),
        lambda: pins.test_dequantize_is_one_product_then_narrow("bf16"),
    ]
    return checks


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(name, old, new, tmp_path):
    assert SRC.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "bq_oracle.c"
    src.write_text(SRC.replace(old, new))
    shutil.copy(obuild.HDR, tmp_path / "bq_oracle.h")
    so = obuild.compile_oracle(str(src), str(tmp_path / "libmutant.so"))
    mutant = oracle.load_library(so)
    saved = oracle._lib
    oracle.lib()                      # make sure the real one is loaded to restore
    saved = oracle._lib
    oracle._lib = mutant
    caught = []
    try:
        for check in _all_pins():
            try:
                check()
            except (AssertionError, ValueError, IndexError):
                caught.append(getattr(check, "__name__", "lambda"))
    finally:
        oracle._lib = saved
    assert caught, f"no pin noticed mutant {name}"


def test_mutation_sites_exist_once():
    for name, old, _ in MUTANTS:
        assert SRC.count(old) == 1, name
    assert os.path.exists(obuild.SRC)
