"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that
the pins in ``test_oracle_pins.py`` catch every one of them.

Each mutant is the oracle's C source with one edit, compiled to a temporary
library and swapped in for the real one while the pins run.
"""
import ctypes
import subprocess
from pathlib import Path

import pytest

import oracle
import oracle.ref as ref
from oracle import build as obuild

import test_oracle_pins as pins

SRC = Path(obuild.SRC).read_text()

MUTANTS = {
    "msb_first_packing": ("wq[r * words_per_row + c / per_word] |= q << ((c % per_word) * bits);",
                          "wq[r * words_per_row + c / per_word] |= q << ((per_word - 1 - c % per_word) * bits);"),
    "divisor_2_pow_bits": ("float scale32 = (hi - lo) / qmax;",
                           "float scale32 = (hi - lo) / (qmax + 1.0f);"),
    "floor_not_round": ("float t = rintf((v - b) / s);", "float t = floorf((v - b) / s);"),
    "bias_is_max": ("float b = store_elem(biases, dtype, sb, lo);",
                    "float b = store_elem(biases, dtype, sb, hi);"),
    "sign_error": ("float t = rintf((v - b) / s);", "float t = rintf((b - v) / s);"),
    "dequant_drops_bias": ("float v = fmaf(s, q, b);", "float v = s * q;"),
    "dequant_wrong_group": ("const int64_t sb = r * groups_per_row + c / group_size;",
                            "const int64_t sb = r * groups_per_row + (c / group_size) % 1;"),
    "truncating_bf16": ("u += 0x7fffu + keep_lsb;", "u += 0u;"),
    "wrong_word_stride": ("uint32_t word = wq[r * words_per_row + c / per_word];",
                          "uint32_t word = wq[r + c / per_word];"),
}


def _pin_calls():
    """Every pin, with fixed parameters; each raises if its check fails."""
    import torch
    calls = [
        pins.test_from_dense_doctest_shapes,
        pins.test_quantized_dense_doctest_shape,
        pins.test_mlx_rs_quantized_matmul_bound,
        pins.test_mlx_rs_gather_qmm_cases,
        pins.test_hand_packed_int4,
        pins.test_hand_packed_int2,
        pins.test_hand_packed_int8,
        pins.test_one_hot_rows_pick_weight_columns,
    ]
    for bits in (2, 4, 8):
        calls.append(lambda bits=bits: pins.test_mlx_rs_quantize_dequantize_bound(bits))
        calls.append(lambda bits=bits: pins.test_code_is_nearest_grid_point(bits))
        calls.append(lambda bits=bits: pins.test_unpack_inverts_pack(bits))
        for tr in (True, False):
            calls.append(lambda bits=bits, tr=tr: pins.test_matmul_reduces_to_dense_on_grid(bits, tr))
        for dt in pins.DTYPES:
            calls.append(lambda bits=bits, dt=dt: pins.test_error_within_half_scale(dt, bits))
            calls.append(lambda bits=bits, dt=dt: pins.test_on_grid_round_trip_is_exact(dt, bits, 64))
    for dt in (torch.bfloat16, torch.float16):
        calls.append(lambda dt=dt: pins.test_dtype_rounding_matches_library(dt))
    return calls


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation site for {name} not found exactly once"
    src = tmp_path / "mutant.c"
    src.write_text(SRC.replace(old, new))
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", *obuild.CFLAGS, str(src), "-o", str(lib_path), "-lm"],
                   check=True, capture_output=True)
    saved = ref._lib
    try:
        ref._lib = None
        real_build = obuild.build
        obuild.build = lambda force=False: lib_path
        ref._load()
        caught = []
        for call in _pin_calls():
            try:
                call()
            except (AssertionError, ValueError, RuntimeError, IndexError):
                caught.append(call)
        assert caught, f"no pin caught mutant {name}"
    finally:
        obuild.build = real_build
        ref._lib = saved


def test_unmutated_oracle_passes_all_pin_calls():
    for call in _pin_calls():
        call()
