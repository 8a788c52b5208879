"""Pins for the oracle's microscaled modes (mxfp4, mxfp8, nvfp4).

The pages name these modes and their (group_size, bits) and say that each
group has one u8 scale in E8M0 or E4M3 and no bias (Emily.QuantizedWeight,
sections Layout and Microscaled modes).  They do not give the rule, so these
pins check the oracle against the published format definitions: values
written by hand from them (tests/golden/mx_formats.json, each with its
citation) and torch's own float8_e4m3fn conversion as an independent
implementation of E4M3 rounding.
"""
import json
from pathlib import Path

import pytest
import torch

import oracle
from quantized_matmul_03_b200 import workloads as wl

GOLD = json.loads((Path(__file__).parent / "golden" / "mx_formats.json").read_text())


def test_group_size_and_bits_are_fixed_per_mode():
    """Emily.QuantizedWeight, section Microscaled modes: mxfp4 32/4, mxfp8 32/8,
    nvfp4 16/4; a mismatch is an error."""
    assert {m: v[:2] for m, v in oracle.MX_MODES.items()} == {
        "mxfp4": (32, 4), "mxfp8": (32, 8), "nvfp4": (16, 4)}
    w = torch.zeros((2, 64))
    with pytest.raises(ValueError):
        oracle.quantize(w, 64, 4, "mxfp4")
    with pytest.raises(ValueError):
        oracle.quantize(w, 32, 4, "nvfp4")


def test_layout_shapes_and_no_bias():
    w = wl.normal((3, 5, 128), 1, 1.0, torch.bfloat16)
    for mode, (gs, bits, _) in oracle.MX_MODES.items():
        wq, s, b = oracle.quantize(w, gs, bits, mode)
        assert b is None
        assert wq.shape == (3, 5, 128 * bits // 32) and wq.dtype == torch.int32
        assert s.shape == (3, 5, 128 // gs) and s.dtype == torch.uint8


def _word_of_codes(codes, bits):
    """Hand packing, least-significant code first."""
    v = 0
    for i, c in enumerate(codes):
        v |= int(c) << (i * bits)
    return v - (1 << 32) if v >= 1 << 31 else v


def test_e2m1_value_table():
    """Every E2M1 code dequantized with scale byte 127 (X = 1)."""
    want = GOLD["e2m1_values"]["by_code"]
    words = [_word_of_codes(range(8), 4), _word_of_codes(range(8, 16), 4)] * 2
    wq = torch.tensor([words], dtype=torch.int32)             # one row of 32 codes
    s = torch.full((1, 1), 127, dtype=torch.uint8)
    d = oracle.dequantize(wq, s, None, 32, 4, "mxfp4", torch.float32)[0]
    for c in range(16):
        assert d[c].item() == want[c] and d[16 + c].item() == want[c]
        if c == 8:
            assert torch.signbit(d[c])


def test_e2m1_rounding_ties_to_even_and_saturates():
    cases = GOLD["e2m1_rounding"]["cases"]
    vals = torch.tensor([c[0] for c in cases], dtype=torch.float32)
    got = oracle.encode_elements(vals, "mxfp4").tolist()
    assert got == [c[1] for c in cases]


def test_e4m3_named_points_and_saturation():
    for key in ("e4m3_points", "e4m3_saturation"):
        cases = GOLD[key]["cases"]
        vals = torch.tensor([c[0] for c in cases], dtype=torch.float32)
        assert oracle.encode_elements(vals, "mxfp8").tolist() == [c[1] for c in cases]


def test_e4m3_rounding_matches_torch_float8():
    """Inside the range where torch's cast does not overflow (|v| <= 464:
    above it, nearest-even rounding reaches 480, which torch turns into NaN
    and the saturating conversion into 448) the oracle's E4M3 codes are
    torch.float8_e4m3fn's, including exact ties and subnormals."""
    g = torch.Generator().manual_seed(5)
    v = torch.cat([
        torch.randn(20000, generator=g) * torch.pow(2.0, torch.randint(-12, 9, (20000,), generator=g)),
        torch.tensor([464.0, 2.0 ** -10, 3 * 2.0 ** -10, 0.0029296875, 17.0, 18.0, 19.0, -0.0]),
    ])
    v = v[v.abs() <= 464]
    want = v.to(torch.float8_e4m3fn).view(torch.uint8)
    assert torch.equal(oracle.encode_elements(v, "mxfp8"), want)


def test_e4m3_value_table_matches_torch_float8():
    """mxfp8 dequantize with X = 1 gives every finite E4M3 value as torch reads it."""
    codes = [c for c in range(256) if c not in (0x7F, 0xFF)]
    codes = codes + [0] * (256 - len(codes))                 # 256 codes = 8 groups of 32
    words = [_word_of_codes(codes[4 * i:4 * i + 4], 8) for i in range(64)]
    wq = torch.tensor([words], dtype=torch.int32)
    s = torch.full((1, 8), 127, dtype=torch.uint8)
    d = oracle.dequantize(wq, s, None, 32, 8, "mxfp8", torch.float32)[0]
    want = torch.tensor(codes, dtype=torch.uint8).view(torch.float8_e4m3fn).float()
    assert torch.equal(d, want)


def test_e8m0_scale_values():
    """The dequantized value of code 2 (E2M1 1.0) is the scale's value."""
    for byte, val in GOLD["e8m0"]["cases"]:
        wq = torch.tensor([[_word_of_codes([2] * 8, 4)] * 4], dtype=torch.int32)
        s = torch.full((1, 1), byte, dtype=torch.uint8)
        d = oracle.dequantize(wq, s, None, 32, 4, "mxfp4", torch.float32)
        assert d[0, 0].item() == val


@pytest.mark.parametrize("case", range(len(GOLD["blocks"]["cases"])))
def test_worked_blocks(case):
    c = GOLD["blocks"]["cases"][case]
    gs, bits, _ = oracle.MX_MODES[c["mode"]]
    w = torch.zeros((1, gs))
    w[0, :4] = torch.tensor(c["values_head"])
    wq, s, _ = oracle.quantize(w, gs, bits, c["mode"])
    assert s.reshape(-1).tolist() == [c["scale"]]
    codes = oracle.unpack_codes(wq, bits)[0, :4].tolist()
    assert codes == c["codes_head"]


@pytest.mark.parametrize("mode", ["mxfp4", "mxfp8", "nvfp4"])
def test_on_grid_blocks_round_trip_exactly(mode):
    """Blocks built as scale x element values (each block holding the
    element format's largest value, so the scale rule recovers the scale)
    dequantize back to themselves."""
    gs, bits, _ = oracle.MX_MODES[mode]
    g = torch.Generator().manual_seed(9)
    rows, groups = 6, 4
    if bits == 4:
        elems = torch.tensor(GOLD["e2m1_values"]["by_code"])
        top = 6.0
    else:
        elems = torch.arange(256, dtype=torch.uint8)
        elems = elems[(elems & 0x7F) != 0x7F].view(torch.float8_e4m3fn).float()
        top = 448.0
    pick = elems[torch.randint(0, elems.numel(), (rows, groups, gs), generator=g)]
    pick[:, :, 0] = top
    if mode == "nvfp4":
        scale = torch.pow(2.0, torch.randint(-6, 3, (rows, groups, 1), generator=g).float())
    else:
        scale = torch.pow(2.0, torch.randint(-20, 20, (rows, groups, 1), generator=g).float())
    w = (pick * scale).reshape(rows, groups * gs)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    d = oracle.dequantize(wq, s, None, gs, bits, mode, torch.float32)
    assert torch.equal(d, w)


@pytest.mark.parametrize("mode", ["mxfp4", "mxfp8", "nvfp4"])
def test_error_within_half_step_unless_saturated(mode):
    """Each element is within half an element step (times the scale) of its
    value, except where the scale rule saturates it to the largest element."""
    gs, bits, _ = oracle.MX_MODES[mode]
    w = wl.normal((32, 256), 3, 1.0, torch.float32)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    d = oracle.dequantize(wq, s, None, gs, bits, mode, torch.float32)
    if mode == "nvfp4":
        x = s.view(torch.float8_e4m3fn).float()
    else:
        x = torch.pow(2.0, s.float() - 127)
    x = x.repeat_interleave(gs, dim=1)
    top = 6.0 if bits == 4 else 448.0
    unsat = (w.abs() / x) <= top
    # largest element step: 2 (E2M1 between 4 and 6), 32 (E4M3 between 256 and 448)
    step = torch.where(w.abs() / x >= (4.0 if bits == 4 else 256.0),
                       torch.tensor(2.0 if bits == 4 else 32.0), torch.tensor(1.0 if bits == 4 else 16.0))
    assert ((d - w).abs() <= step / 2 * x + 1e-30)[unsat].all()
    assert (d[~unsat].abs() == top * x[~unsat]).all()


def test_matmul_uses_the_microscaled_weight():
    """quantized_matmul in a microscaled mode is the float64 product with the
    dequantized weight (a library matmul)."""
    w = wl.normal((40, 128), 4, 0.05, torch.bfloat16)
    x = wl.normal((3, 128), 5, 1.0, torch.bfloat16)
    for mode, (gs, bits, _) in oracle.MX_MODES.items():
        wq, s, _ = oracle.quantize(w, gs, bits, mode)
        deq = oracle.dequantize(wq, s, None, gs, bits, mode, torch.float32).double()
        y = oracle.quantized_matmul(x, wq, s, None, True, gs, bits, mode)
        assert torch.allclose(y, x.double() @ deq.T, rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# qqmm (mlx-rs ops/quantization.rs): both operands quantized, nvfp4 / mxfp8.
# --------------------------------------------------------------------------

def _on_grid_rows(rows, cols, mode, seed):
    """Rows whose every group is scale x element values with the group's
    largest element at the format's top, so quantizing them is exact."""
    gs, bits, _ = oracle.MX_MODES[mode]
    g = torch.Generator().manual_seed(seed)
    if bits == 4:
        elems = torch.tensor(GOLD["e2m1_values"]["by_code"])
        top = 6.0
    else:
        elems = torch.arange(256, dtype=torch.uint8)
        elems = elems[(elems & 0x7F) != 0x7F].view(torch.float8_e4m3fn).float()
        top = 448.0
    pick = elems[torch.randint(0, elems.numel(), (rows, cols // gs, gs), generator=g)]
    pick[:, :, 0] = top
    lo, hi = (-6, 3) if mode == "nvfp4" else (-12, 4)
    scale = torch.pow(2.0, torch.randint(lo, hi, (rows, cols // gs, 1), generator=g).float())
    return (pick * scale).reshape(rows, cols)


@pytest.mark.parametrize("mode", ["nvfp4", "mxfp8"])
def test_qqmm_on_grid_is_the_exact_product(mode):
    """Operands already on their grids quantize exactly, so qqmm is the plain
    float64 product of the inputs (a library matmul)."""
    x = _on_grid_rows(5, 128, mode, 11)
    w = _on_grid_rows(24, 128, mode, 12)
    gs, bits, _ = oracle.MX_MODES[mode]
    y = oracle.qqmm(x, w, None, gs, bits, mode)
    assert torch.equal(y, x.double() @ w.double().T)


@pytest.mark.parametrize("mode", ["nvfp4", "mxfp8"])
def test_qqmm_dense_weight_equals_prequantized(mode):
    gs, bits, _ = oracle.MX_MODES[mode]
    x = wl.normal((3, 256), 13, 1.0, torch.bfloat16)
    w = wl.normal((40, 256), 14, 0.1, torch.bfloat16)
    wq, ws, _ = oracle.quantize(w, gs, bits, mode)
    assert torch.equal(oracle.qqmm(x, w, None, gs, bits, mode), oracle.qqmm(x, wq, ws, gs, bits, mode))


def test_qqmm_quantizes_the_activations():
    """Off-grid activations are rounded: the result differs from the product
    with x kept exact, by no more than the activations' quantization error."""
    gs, bits, _ = oracle.MX_MODES["mxfp8"]
    x = wl.normal((4, 256), 15, 1.0, torch.float32)
    w = _on_grid_rows(16, 256, "mxfp8", 16)
    y = oracle.qqmm(x, w, None, gs, bits, "mxfp8")
    exact = x.double() @ w.double().T
    xq, xs, _ = oracle.quantize(x, gs, bits, "mxfp8")
    xd = oracle.dequantize(xq, xs, None, gs, bits, "mxfp8", torch.float32).double()
    assert not torch.equal(y, exact)
    assert torch.allclose(y, xd @ w.double().T, rtol=1e-12, atol=1e-12)
    bound = (xd - x.double()).abs() @ w.double().abs().T
    assert ((y - exact).abs() <= bound + 1e-9).all()
