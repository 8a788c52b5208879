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

import test_oracle_mx_pins as mx_pins
import test_oracle_pins as pins

SRC = Path(obuild.SRC).read_text()

MUTANTS = {
    "msb_first_packing": ("row[bit / 32] |= q << off;", "row[bit / 32] |= q << (32 - bits - off);"),
    "straddle_dropped": ("row[bit / 32 + 1] |= q >> (32 - off);", "(void)0;"),
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
    "wrong_word_stride": ("const uint32_t *row = wq + r * words_per_row;\n    uint32_t v",
                          "const uint32_t *row = wq + r;\n    uint32_t v"),
    # microscaled modes
    "mx_emax_e2m1": ("const int emax = bits == 8 ? 8 : 2;", "const int emax = bits == 8 ? 8 : 3;"),
    "e8m0_bias": ("scode = (uint32_t)(shared + 127);", "scode = (uint32_t)(shared + 126);"),
    "e2m1_tie_up": ("if (a <= 0.25f) c = 0;", "if (a < 0.25f) c = 0;"),
    "nvfp4_divisor": ("scode = e4m3_encode(amax / 6.0f);", "scode = e4m3_encode(amax / 4.0f);"),
    "e4m3_no_saturation": ("if (e > 8 || (e == 8 && mi == 7.0f)) return sign | 0x7Eu;",
                           "if (e > 8) return sign | 0x7Eu;"),
    "e4m3_subnormal_step": ("const float m = rintf(ldexpf(a, 9));", "const float m = rintf(ldexpf(a, 8));"),
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
    for bits in (2, 3, 4, 6, 8):
        calls.append(lambda bits=bits: pins.test_mlx_rs_quantize_dequantize_bound(bits))
        calls.append(lambda bits=bits: pins.test_code_is_nearest_grid_point(bits))
        calls.append(lambda bits=bits: pins.test_unpack_inverts_pack(bits))
        if bits in (3, 6):
            calls.append(lambda bits=bits: pins.test_hand_packed_straddling_codes(bits))
        for tr in (True, False):
            calls.append(lambda bits=bits, tr=tr: pins.test_matmul_reduces_to_dense_on_grid(bits, tr))
        for dt in pins.DTYPES:
            calls.append(lambda bits=bits, dt=dt: pins.test_error_within_half_scale(dt, bits))
            calls.append(lambda bits=bits, dt=dt: pins.test_on_grid_round_trip_is_exact(dt, bits, 64))
    for dt in (torch.bfloat16, torch.float16):
        calls.append(lambda dt=dt: pins.test_dtype_rounding_matches_library(dt))
    calls += [mx_pins.test_e2m1_value_table, mx_pins.test_e2m1_rounding_ties_to_even_and_saturates,
              mx_pins.test_e4m3_named_points_and_saturation, mx_pins.test_e4m3_rounding_matches_torch_float8,
              mx_pins.test_e4m3_value_table_matches_torch_float8, mx_pins.test_e8m0_scale_values]
    for i in range(len(mx_pins.GOLD["blocks"]["cases"])):
        calls.append(lambda i=i: mx_pins.test_worked_blocks(i))
    for mode in ("mxfp4", "mxfp8", "nvfp4"):
        calls.append(lambda mode=mode: mx_pins.test_on_grid_blocks_round_trip_exactly(mode))
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


# quantized_dense adds the layer bias in Python (oracle/ref.py): mutants of
# that step, swapped in for oracle.quantized_dense while the dense pins run.
def _dense_mutants():
    import torch
    mm = ref.quantized_matmul

    def drops_bias(x, wq, s, b, bias=0, transpose=True, gs=64, bits=4):
        return mm(x, wq, s, b, transpose, gs, bits)

    def bias_twice(x, wq, s, b, bias=0, transpose=True, gs=64, bits=4):
        y = mm(x, wq, s, b, transpose, gs, bits)
        bb = bias.double().reshape(-1) if isinstance(bias, torch.Tensor) else float(bias)
        return y + 2 * bb

    def bias_along_rows(x, wq, s, b, bias=0, transpose=True, gs=64, bits=4):
        y = mm(x, wq, s, b, transpose, gs, bits)
        if isinstance(bias, torch.Tensor):
            return y + bias.double().reshape(-1)[: y.shape[0]].reshape(-1, 1)
        return y + float(bias)

    def ignores_number(x, wq, s, b, bias=0, transpose=True, gs=64, bits=4):
        y = mm(x, wq, s, b, transpose, gs, bits)
        return y + bias.double().reshape(-1) if isinstance(bias, torch.Tensor) else y

    return {"drops_bias": drops_bias, "bias_twice": bias_twice,
            "bias_along_rows": bias_along_rows, "ignores_number": ignores_number}


def _dense_pin_calls():
    return [lambda: pins.test_dense_one_hot_rows_give_weight_column_plus_bias(True),
            lambda: pins.test_dense_one_hot_rows_give_weight_column_plus_bias(False),
            pins.test_dense_on_grid_reduces_to_library_product_plus_bias,
            pins.test_dense_number_bias_equals_constant_tensor]


@pytest.mark.parametrize("name", sorted(_dense_mutants()))
def test_dense_pins_catch_mutant(name, monkeypatch):
    monkeypatch.setattr(oracle, "quantized_dense", _dense_mutants()[name])
    caught = 0
    for call in _dense_pin_calls():
        try:
            call()
        except (AssertionError, ValueError, RuntimeError, IndexError):
            caught += 1
    assert caught, f"no pin caught dense mutant {name}"


def test_unmutated_dense_passes_its_pins():
    for call in _dense_pin_calls():
        call()
