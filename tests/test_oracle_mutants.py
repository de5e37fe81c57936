"""Planted mistakes: copies of the oracle with one plausible error each must fail a pin.

The mistakes are planted in temporary copies of oracle/q4_oracle.c on the CPU; the
committed oracle is never modified. This shows that the pins would catch a wrong
sign, a dropped term, a swapped index, a changed rounding or a wrong nibble order.
"""
import os
import subprocess

import pytest

import oracle
import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "q4_oracle.c")

MUTANTS = {
    "scale_sign": ("m / -8.0f", "m / 8.0f"),
    "round_to_floor": ("scaled + 8.5f", "scaled + 8.0f"),
    "divide_not_reciprocal": ("volatile float scaled = w[j] * id;",
                              "volatile float scaled = (d != 0.0f) ? w[j] / d : 0.0f;"),
    "tie_last_index": ("if (a > amax) {", "if (a >= amax) {"),
    "nibble_order": ("(uint8_t)(q[j] | (q[j + ORACLE_QK / 2] << 4))",
                     "(uint8_t)((q[j] << 4) | q[j + ORACLE_QK / 2])"),
    "no_clamp": ("if (code > 15) code = 15;", ""),
    "dequant_offset": ("d * (float)(block_code(blk, j) - 8)", "d * (float)(block_code(blk, j) - 7)"),
    "gemv_offset": ("d * (double)(block_code(blk, j) - 8)", "d * (double)(block_code(blk, j) - 7)"),
    "gemv_dropped_term": ("for (int j = 0; j < ORACLE_QK; ++j) {\n                double w_hat",
                          "for (int j = 1; j < ORACLE_QK; ++j) {\n                double w_hat"),
    "gemv_x_reversed": ("(double)x[b * ORACLE_QK + j]", "(double)x[b * ORACLE_QK + (ORACLE_QK - 1 - j)]"),
    "gemv_abs_sum": ("sabs += fabs(term);", "sabs += term;"),
    "f16_ties_down": ("(rem == halfway && (kept & 1u))", "(rem == halfway && 0)"),
    "f16_bias": ("ldexp((double)(1024 + mant), ex - 25)", "ldexp((double)(1024 + mant), ex - 24)"),
    "high_nibble_weight": ("return j < 16 ? (byte & 0x0f) : (byte >> 4);",
                           "return j < 16 ? (byte >> 4) : (byte & 0x0f);"),
    "planes_swap": ("memcpy(qs + i * 16, blk + 2, 16);", "memcpy(qs + i * 16, blk + 1, 16);"),
    # batched form (the pin's matrices have n < k, so these reads stay inside X)
    "batched_token_zero": ("X + t * k, Y + t * n", "X, Y + t * n"),
    "batched_x_stride": ("X + t * k, Y + t * n", "X + t * n, Y + t * n"),
    "batched_abs_sum_row": ("abs_sum ? abs_sum + t * n : (double *)0", "abs_sum ? abs_sum : (double *)0"),
}


def _first_failure(lib):
    for check in pins.ALL_CHECKS:
        try:
            check(lib)
        except AssertionError as e:
            return f"{check.__name__}: {e}"
    try:
        pins.check_roundtrip(lib, 20000)
    except AssertionError as e:
        return f"check_roundtrip: {e}"
    return None


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src.replace(old, new))
    so = str(tmp_path / f"libmut_{name}.so")
    subprocess.check_call(["gcc", *oracle.CFLAGS, str(path), "-o", so, "-lm"])
    lib = oracle.load(so)
    failure = _first_failure(lib)
    assert failure is not None, f"planted mistake {name} passed every pin"
