"""Mistakes planted in copies of the oracle (on the CPU) must each fail some pin.

Each mutation rewrites one expression of ``oracle/lowbit_oracle.c`` into a plausible
error (a wrong bit position, sign, index, dropped term, transposed operand or lower
accumulation precision), compiles the copy into a temporary directory and runs the
pin battery against it. The real oracle is not modified.
"""
import ctypes
import os

import pytest

import oracle
from tests import _pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lowbit_oracle.c")

MUTATIONS = {
    "plain_lsb_first_positions": ("return (int)((i % 2) * 16 + (i / 2) * bits);", "return (int)(i * bits);"),
    "ternary_sign_flipped": ("return s * (double)((int)f - 1);", "return s * (double)(1 - (int)f);"),
    "binary_sign_flipped": ("if (bits == 1) return f ? s : -s;", "if (bits == 1) return f ? -s : s;"),
    "scale_index_transposed": ("double s = oracle_f16_to_f64(scales[(k / g) * N + n]);",
                               "double s = oracle_f16_to_f64(scales[n * (K / g) + k / g]);"),
    "zero_point_added": ("return ((double)f - z) * s;", "return ((double)f + z) * s;"),
    "zero_point_dropped": ("return ((double)f - z) * s;", "return ((double)f) * s;"),
    "first_term_dropped": ("for (int64_t k = 0; k < K; ++k) acc += xr[k] * wr[k];",
                           "for (int64_t k = 1; k < K; ++k) acc += xr[k] * wr[k];"),
    "float_accumulator": ("double acc = 0.0;\n            for (int64_t k = 0; k < K; ++k) acc += xr[k]",
                          "float acc = 0.0f;\n            for (int64_t k = 0; k < K; ++k) acc += xr[k]"),
    "weights_transposed": ("for (int64_t k = 0; k < K; ++k) acc += xr[k] * wr[k];",
                           "for (int64_t k = 0; k < K; ++k) acc += xr[k] * W[(k % N) * K + n % K];"),
    "group_of_next_column": ("double s = oracle_f16_to_f64(scales[(k / g) * N + n]);",
                             "double s = oracle_f16_to_f64(scales[((k + 1) % K / g) * N + n]);"),
    "fp16_exponent_bias": ("v = ldexp(1024.0 + (double)f, e - 25);", "v = ldexp(1024.0 + (double)f, e - 24);"),
    "bf16_shift": ("uint32_t b = (uint32_t)h << 16;", "uint32_t b = (uint32_t)h << 15;"),
    "word_row_stride": ("uint32_t word = packed[n * (K / cpw) + j];",
                        "uint32_t word = packed[n * (K / cpw) + j % 1];"),
    "block_pair_and_lane_swapped": ("return 4 * cpw * b + 8 * p + 2 * q + d;",
                                    "return 4 * cpw * b + 8 * q + 2 * p + d;"),
    "block_order_not_used": ("if (bits != 1 && j < wpr / 4 * 4) {", "if (bits != 1 && j < 0) {"),
    "unpack_lane_from_pair_index": ("*j = 4 * b + (r % 8) / 2;", "*j = 4 * b + (r / 8) % 4;"),
    "invalid_ternary_field_decodes_zero": ("if (f == 3) return NAN;", "if (f == 3) return 0.0;"),
    "invalid_ternary_field_not_checked": ("if (f == 3) return NAN;", "if (f == 4) return NAN;"),
    "ternary_field_map": ("if (c >= -1 && c <= 1) { *field = (uint32_t)(c + 1); return 0; }",
                          "if (c >= -1 && c <= 1) { *field = (uint32_t)(c + 1) ^ 2u; return 0; }"),
}


@pytest.fixture(scope="module")
def source():
    with open(SRC) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTATIONS[name]
    assert source.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = source.replace(old, new)
    src = tmp_path / "mutant.c"
    src.write_text(mutated)
    lib = oracle.compile_oracle(str(src), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(oracle.bind(ctypes.CDLL(lib)))
    caught = []
    for pin in _pins.ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError) as e:  # ValueError: mutant rejects a valid call
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutation {name}"
