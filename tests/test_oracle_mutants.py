"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of oracle/kvs_oracle.c (on the CPU,
never in the product), builds it, points the oracle binding at it, and runs
the pin tests: at least one of them must fail.  The real oracle passes them.
"""
import ctypes
import os
import shutil
import subprocess

import pytest

import oracle
import test_oracle_attention as TA
import test_oracle_fp16 as TF
import test_oracle_pages as TP
import test_oracle_q5_0 as T5
import test_oracle_q_min as TM
import test_oracle_k_f16 as TK16
import test_oracle_v_f16 as TV16
import test_oracle_quant as TQ

SRC = os.path.join(os.path.dirname(oracle.__file__), "kvs_oracle.c")
HDR = os.path.join(os.path.dirname(oracle.__file__), "kvs_oracle.h")

MUTANTS = {
    "q8 ties to even": ("q = (int)roundf(x[i] / d);", "q = (int)rintf(x[i] / d);"),
    "q8 scale /128": ("float d = amax / 127.0f;", "float d = amax / 128.0f;"),
    "q4 last index wins": ("if (a > amax) { /* strict", "if (a >= amax) { /* strict"),
    "q4 offset 8.0": ("(int)(x[i] / d + 8.5f)", "(int)(x[i] / d + 8.0f)"),
    "q4 nibble order": ("out[2 + j] = (uint8_t)(q[j] | (q[j + 16] << 4))",
                        "out[2 + j] = (uint8_t)((q[j] << 4) | q[j + 16])"),
    "q4_1 nibble order": ("out[4 + j] = (uint8_t)(q[j] | (q[j + 16] << 4))",
                          "out[4 + j] = (uint8_t)((q[j] << 4) | q[j + 16])"),
    "q4 dequant offset": ("(int)(blk[2 + j] & 0x0f) - 8)", "(int)(blk[2 + j] & 0x0f) - 7)"),
    "scale 1/d": ("double scale = 1.0 / sqrt((double)dim);", "double scale = 1.0 / (double)dim;"),
    "causal off by one": ("int n_keys = pos0 + j + 1;", "int n_keys = pos0 + j;"),
    "gqa interleaved": ("int g = h / group;", "int g = h % n_kv;"),
    "lse base 2": ("lse[(size_t)j * n_qh + h] = m + log(sum);", "lse[(size_t)j * n_qh + h] = m + log2(sum);"),
    "fp16 ties down": ("if (rem > 0x1000u || (rem == 0x1000u && (hm & 1u))) {", "if (rem > 0x1000u) {"),
    "q5 last index wins": ("if (a > amax) { /* the first index", "if (a >= amax) { /* the first index"),
    "q5 offset 16.0": ("(int)(x[i] / d + 16.5f)", "(int)(x[i] / d + 16.0f)"),
    "q5 scale /-15": ("float d = m / -16.0f;", "float d = m / -15.0f;"),
    "q5 no clamp": ("q[i] = t < 31 ? t : 31;", "q[i] = t;"),
    "q5 high bits reversed": ("high |= (uint32_t)(q[i] >> 4) << i;", "high |= (uint32_t)(q[i] >> 4) << (31 - i);"),
    "q5 dequant offset": ("out[j] = d * (double)(lo - 16);", "out[j] = d * (double)(lo - 15);"),
    "v type dispatch": ("else if (v_type == 6) oracle_dequant_q5_0(blk, out);",
                        "else if (v_type == 6) oracle_dequant_q4_0(blk, out);"),
    "q1 no rounding offset": ("int t = (int)((x[i] - lo) / d + 0.5f);", "int t = (int)((x[i] - lo) / d);"),
    "q1 stores the max": ("*mh = oracle_float_to_half(lo);", "*mh = oracle_float_to_half(hi);"),
    "q1 one step too many": ("float d = (hi - lo) / (float)levels;", "float d = (hi - lo) / (float)(levels + 1);"),
    "q4_1 dequant drops m": ("out[j] = d * (double)(blk[4 + j] & 0x0f) + m;", "out[j] = d * (double)(blk[4 + j] & 0x0f);"),
    "q5_1 fifth bit shifted": ("int a = (int)(blk[8 + j] & 0x0f) | (int)(((top >> j) & 1u) << 4);",
                               "int a = (int)(blk[8 + j] & 0x0f) | (int)(((top >> (j + 1)) & 1u) << 4);"),
    "f16 V byte order": ("out[2 * i] = (uint8_t)(x_h[i] & 0xff);", "out[2 * i] = (uint8_t)(x_h[i] >> 8);"),
    "q8 reciprocal": ("if (d != 0.0f) q = (int)roundf(x[i] / d);",
                      "if (d != 0.0f) q = (int)roundf(x[i] * (1.0f / d));"),
    "q8 fp16 divisor": ("if (d != 0.0f) q = (int)roundf(x[i] / d);",
                        "if (d != 0.0f) q = (int)roundf(x[i] / oracle_half_to_float(dh));"),
    "q4 reciprocal": ("int t = (int)(x[i] / d + 8.5f);", "int t = (int)(x[i] * (1.0f / d) + 8.5f);"),
    "q4 fp16 divisor": ("int t = (int)(x[i] / d + 8.5f);",
                        "int t = (int)(x[i] / oracle_half_to_float(dh) + 8.5f);"),
    "q5 reciprocal": ("int t = (int)(x[i] / d + 16.5f);", "int t = (int)(x[i] * (1.0f / d) + 16.5f);"),
    "q5 fp16 divisor": ("int t = (int)(x[i] / d + 16.5f);",
                        "int t = (int)(x[i] / oracle_half_to_float(dh) + 16.5f);"),
    "q1 reciprocal": ("int t = (int)((x[i] - lo) / d + 0.5f);", "int t = (int)((x[i] - lo) * (1.0f / d) + 0.5f);"),
    "q1 fp16 divisor": ("int t = (int)((x[i] - lo) / d + 0.5f);",
                        "int t = (int)((x[i] - lo) / oracle_half_to_float(*dh) + 0.5f);"),
    "f16 K read as Q8_0": ("if (k_type == 8) oracle_dequant_q8_0(kblk, kd);\n                    else f16_dequant(kblk, kd);",
                           "oracle_dequant_q8_0(kblk, kd);"),
    "f16 K stored as Q8_0": ("else f16_block(kx, k_blocks + ((size_t)r * nb + b) * kbb);",
                             "else oracle_q8_0_block(kx, k_blocks + ((size_t)r * nb + b) * kbb);"),
    "resident window": ("if (page >= P - n_resident) {", "if (page > P - n_resident) {"),
    "auto floor": ("long floor_pages = (2048 + page_tokens - 1) / page_tokens;",
                   "long floor_pages = (4096 + page_tokens - 1) / page_tokens;"),
}


def pins():
    return [
        TQ.test_q8_0_hand_worked, TQ.test_q4_0_hand_worked, TQ.test_zero_block,
        lambda: TQ.test_constant_block(1.0), lambda: TQ.test_single_nonzero(7, -2.5),
        TQ.test_q4_0_error_bound_and_range,
        TA.test_two_key_closed_form_pins_scale, TA.test_gqa_grouping_is_contiguous,
        TA.test_zero_query_is_uniform_mean_with_causal_lengths, TA.test_against_scipy_softmax_random,
        TA.test_single_key_returns_its_value,
        TP.test_auto_resident_matches_printed_numbers, TP.test_auto_resident_floor_and_ceiling,
        lambda: TP.test_page_location_invariants(1025, 4),
        TF.test_float_to_half_random,
        T5.test_q5_0_hand_worked, T5.test_q5_0_dequant_of_hand_block, T5.test_q5_0_error_bound_and_range,
        T5.test_q5_0_zero_query_is_uniform_mean, T5.test_q5_0_against_scipy_softmax_random,
        lambda: TM.test_hand_worked("q4_1"), lambda: TM.test_hand_worked("q5_1"),
        lambda: TM.test_error_bound_and_range("q4_1"), lambda: TM.test_error_bound_and_range("q5_1"),
        lambda: TM.test_against_scipy_softmax_random("q5_1"),
        TV16.test_v_blocks_are_the_input_bits, TV16.test_against_scipy_over_exact_values,
        TK16.test_k_blocks_are_the_input_bits, TK16.test_f16_f16_against_scipy_over_exact_values,
    ]


def run_pins():
    failures = 0
    for pin in pins():
        try:
            pin()
        except AssertionError:
            failures += 1
    return failures


def test_real_oracle_passes_its_pins():
    assert run_pins() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not found: {old}"
    d = tmp_path / "m"
    d.mkdir()
    shutil.copy(HDR, d / "kvs_oracle.h")
    (d / "kvs_oracle.c").write_text(src.replace(old, new))
    so = str(d / "libmutant.so")
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
                    "-o", so, str(d / "kvs_oracle.c"), "-lm"], check=True)
    real = oracle.lib()
    try:
        oracle._lib = oracle.bind(ctypes.CDLL(so))
        caught = run_pins()
    finally:
        oracle._lib = real
    assert caught >= 1, f"no pin caught the mutant '{name}'"
