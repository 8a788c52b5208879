"""Pins for the CPU oracle: checks against what the cited documents and the mathematics
fix, never against the oracle's own formulas retyped.

Each test names the documented passage (or the mathematical fact) it rests on and the
plausible oracle mistake it would catch.
"""
import json
import math
from pathlib import Path

import pytest
import torch

import oracle
from quantized_matmul_03_b200 import workloads as wl

GOLDEN = json.loads((Path(__file__).parent / "golden" / "page_examples.json").read_text())
DTYPES = [torch.float32, torch.bfloat16, torch.float16]
QMAX = {2: 3, 3: 7, 4: 15, 6: 63, 8: 255}
ALL_BITS = [2, 3, 4, 6, 8]   # Emily.QuantizedWeight, from_dense: :bits one of [2, 3, 4, 6, 8]


def u32(t: torch.Tensor):
    """int32-stored packed words as Python unsigned ints."""
    return [int(v) & 0xFFFFFFFF for v in t.reshape(-1).tolist()]


# --------------------------------------------------------------------------
# Shapes printed in the documents (doctests) -- catch a wrong packing ratio, a
# wrong group axis, a transposed product.
# --------------------------------------------------------------------------

def test_from_dense_doctest_shapes():
    g = GOLDEN["from_dense_doctest"]
    w = wl.iota(g["w_shape"], torch.float32)
    wq, s, b = oracle.quantize(w, g["group_size"], g["bits"])
    assert list(wq.shape) == g["expect"]["value_shape"]
    assert list(s.shape) == [4, 64 // g["group_size"]] and s.dtype == w.dtype
    assert b.shape == s.shape and b.dtype == w.dtype


def test_to_dense_doctest_shape():
    g = GOLDEN["to_dense_doctest"]
    w = wl.iota(g["w_shape"], torch.float32)
    d = g["defaults"]
    dense = oracle.dequantize(*oracle.quantize(w, d["group_size"], d["bits"]),
                              d["group_size"], d["bits"])
    assert list(dense.shape) == g["expect"]["dense_shape"]


def test_quantized_dense_doctest_shape():
    g = GOLDEN["quantized_dense_doctest"]
    d = g["defaults"]
    w = wl.iota(g["w_shape"], torch.float32)
    x = wl.iota(g["x_shape"], torch.float32)
    wq, s, b = oracle.quantize(w, d["group_size"], d["bits"])
    y = oracle.quantized_matmul(x, wq, s, b, d["transpose"], d["group_size"], d["bits"])
    assert list(y.shape) == g["expect"]["y_shape"]
    # The doctest calls quantized_dense with its default bias (0): the same product.
    yd = oracle.quantized_dense(x, wq, s, b, 0, d["transpose"], d["group_size"], d["bits"])
    assert list(yd.shape) == g["expect"]["y_shape"] and torch.equal(yd, y)


@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_packed_axis_shrinks_by_32_over_bits(bits, gs):
    w = wl.normal((3, 5, 256), 7, 1.0, torch.float32)
    wq, s, b = oracle.quantize(w, gs, bits)
    assert tuple(wq.shape) == (3, 5, 256 * bits // 32)
    assert tuple(s.shape) == (3, 5, 256 // gs)


# --------------------------------------------------------------------------
# mlx-rs unit tests restated (bounds printed on the page).
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", ALL_BITS)
def test_mlx_rs_quantize_dequantize_bound(bits):
    g = GOLDEN["mlx_rs_test_quantize_dequantize"]
    x = torch.arange(0, 512, dtype=torch.float32).expand(g["rows"], 512).contiguous()
    wq, s, b = oracle.quantize(x, g["group_size"], bits)
    assert list(wq.shape) == [128, 512 * bits // 32]   # = 512 / (32 / bits) for 2, 4, 8
    assert list(s.shape) == g["expect"]["scales_shape"]
    assert list(b.shape) == g["expect"]["biases_shape"]
    x_hat = oracle.dequantize(wq, s, b, g["group_size"], bits)
    assert (x - x_hat).abs().max().item() <= 127.0 / (1 << bits)


def test_mlx_rs_quantized_matmul_bound():
    g = GOLDEN["mlx_rs_test_quantized_matmul"]
    m, n, k = g["m"], g["n"], g["k"]
    scale = 1.0 / math.sqrt(k)
    x = wl.normal((m, k), 0) .float() * scale
    w = wl.normal((k, n), 1).float() * scale
    wq, s, b = oracle.quantize(w, g["group_size"], g["bits"])
    w_hat = oracle.dequantize(wq, s, b, g["group_size"], g["bits"])
    y_q = oracle.quantized_matmul(x, wq, s, b, False, g["group_size"], g["bits"])
    y_hat = x @ w_hat                       # fp32 dense product, as on the page
    assert y_q.shape == y_hat.shape
    assert (y_q - y_hat.double()).abs().max().item() < g["bound_max_abs_diff"]


def test_mlx_rs_gather_qmm_cases():
    g = GOLDEN["mlx_rs_test_gather_qmm"]
    m, n, k, e = g["m"], g["n"], g["k"], g["experts"]
    w = wl.normal((e, n, k), 11, 1.0, torch.float32)
    wq, s, b = oracle.quantize(w, g["group_size"], g["bits"])
    w_hat = oracle.dequantize(wq, s, b, g["group_size"], g["bits"]).transpose(-1, -2)
    for i, case in enumerate(g["cases"]):
        x = wl.normal((case["x_batch"], m, k), 12 + i, 1.0, torch.float32)
        lhs = torch.tensor(case["lhs_indices"], dtype=torch.int32)
        rhs = torch.tensor(case["rhs_indices"], dtype=torch.int32)
        # gather_mm written independently: index both operands, batched matmul.
        c1 = x[lhs.long()] @ w_hat[rhs.long()]
        c2 = oracle.gather_qmm(x, wq, s, b, lhs, rhs, True, g["group_size"], g["bits"])
        assert c2.shape == c1.shape
        assert torch.allclose(c1.double(), c2, rtol=g["rtol"], atol=g["atol"])


# --------------------------------------------------------------------------
# Hand-packed words: catch MSB-first packing, a wrong shift, a wrong word index.
# The weights are chosen so that min=0 and max=2^bits-1, hence scale=1, bias=0
# and the codes equal the values.
# --------------------------------------------------------------------------

def test_hand_packed_int4():
    row = [1, 2, 3, 4, 5, 6, 7, 8, 0, 15, 9, 10, 11, 12, 13, 14] + [0] * 48
    w = torch.tensor([row], dtype=torch.float32)
    wq, s, b = oracle.quantize(w, 64, 4)
    assert s.item() == 1.0 and b.item() == 0.0
    assert u32(wq) == [0x87654321, 0xEDCBA9F0, 0, 0, 0, 0, 0, 0]


def _stream_words(codes, bits):
    """Pack codes into uint32 words the long way: one Python integer holding
    the whole row's bit stream (code j at bit j*bits), cut into 32-bit words
    least significant first."""
    v = 0
    for j, c in enumerate(codes):
        v |= int(c) << (j * bits)
    n = len(codes) * bits // 32
    return [(v >> (32 * i)) & 0xFFFFFFFF for i in range(n)]


@pytest.mark.parametrize("bits", [3, 6])
def test_hand_packed_straddling_codes(bits):
    """3- and 6-bit codes (from_dense allows them) sit back to back in the
    row's bit stream, so some straddle two words: 3-bit code 10 occupies bits
    30..32, 6-bit code 5 bits 30..35."""
    qmax = QMAX[bits]
    codes = [(7 * j + 3) % (qmax + 1) for j in range(64)]
    codes[0], codes[1] = 0, qmax          # the group's min and max are on the grid
    codes[32], codes[33] = 0, qmax
    w = torch.tensor([codes], dtype=torch.float32)   # scale 1, bias 0 per group
    wq, s, b = oracle.quantize(w, 32, bits)
    assert torch.equal(s, torch.ones((1, 2))) and torch.equal(b, torch.zeros((1, 2)))
    assert u32(wq) == _stream_words(codes, bits)
    assert oracle.unpack_codes(wq, bits).reshape(-1).tolist() == codes


def test_hand_packed_int2():
    row = [1, 2, 3, 0, 3, 3, 0, 1, 2, 2, 2, 2, 0, 0, 0, 0] + [0] * 16
    w = torch.tensor([row], dtype=torch.float32)
    wq, s, b = oracle.quantize(w, 32, 2)
    assert s.item() == 1.0 and b.item() == 0.0
    assert u32(wq) == [0x00AA4F39, 0]


def test_hand_packed_int8():
    row = [0x11, 0x22, 0x33, 0x44, 255, 0, 7, 128] + [0] * 24
    w = torch.tensor([row], dtype=torch.float32)
    wq, s, b = oracle.quantize(w, 32, 8)
    assert s.item() == 1.0 and b.item() == 0.0
    assert u32(wq) == [0x44332211, 0x800700FF] + [0] * 6


@pytest.mark.parametrize("bits", ALL_BITS)
def test_unpack_inverts_pack(bits):
    w = wl.normal((4, 128), 5, 1.0, torch.float32)
    wq, s, b = oracle.quantize(w, 32, bits)
    q = oracle.unpack_codes(wq, bits)
    # Re-pack each row as one bit stream (Python integers) and compare the words.
    want = []
    for r in range(4):
        want += _stream_words(q[r].tolist(), bits)
    assert u32(wq) == want


# --------------------------------------------------------------------------
# Exact round trip of weights already on the grid: catch a wrong scale divisor
# (2^bits instead of 2^bits-1), bias = max or mean, floor instead of round.
# --------------------------------------------------------------------------

def _on_grid(rows, cols, gs, bits, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    qmax = QMAX[bits]
    G = cols // gs
    e = torch.randint(-8, 1, (rows, G), generator=g).double()
    s = torch.pow(2.0, e)
    # bias = j * s with |j + q| <= 255 so every value is exact even in bf16
    j = torch.randint(-qmax, 1, (rows, G), generator=g).double()
    b = j * s
    q = torch.randint(0, qmax + 1, (rows, G, gs), generator=g)
    q[:, :, 0] = 0
    q[:, :, 1] = qmax
    perm = torch.argsort(torch.rand((rows, G, gs), generator=g), dim=-1)
    q = torch.gather(q, -1, perm)
    w = (b[..., None] + s[..., None] * q.double()).reshape(rows, cols)
    wt = w.to(dtype)
    assert torch.equal(wt.double(), w), "grid values must be exact in the dtype"
    return wt, q.reshape(rows, cols), s, b


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_on_grid_round_trip_is_exact(dtype, bits, gs):
    w, q, s, b = _on_grid(6, 256, gs, bits, dtype, seed=bits * 1000 + gs)
    wq, so, bo = oracle.quantize(w, gs, bits)
    assert torch.equal(so.double(), s)
    assert torch.equal(bo.double(), b)
    assert torch.equal(oracle.unpack_codes(wq, bits).long(), q.long())
    assert torch.equal(oracle.dequantize(wq, so, bo, gs, bits), w)


# --------------------------------------------------------------------------
# Brute force on tiny inputs: the code must be the nearest grid point (checked
# in float64 against every candidate code).  Catches floor/ceil, an off-by-one
# clamp, a sign error in (w - b).
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", ALL_BITS)
def test_code_is_nearest_grid_point(bits):
    w = wl.normal((16, 64), 21 + bits, 3.0, torch.float32)
    wq, s, b = oracle.quantize(w, 32, bits)
    q = oracle.unpack_codes(wq, bits).double()
    cand = torch.arange(QMAX[bits] + 1, dtype=torch.float64)
    sr = s.double().repeat_interleave(32, dim=1)
    br = b.double().repeat_interleave(32, dim=1)
    grid = br[..., None] + sr[..., None] * cand              # [16, 64, 2^bits]
    best = (w.double()[..., None] - grid).abs().min(-1).values
    mine = (w.double() - (br + sr * q)).abs()
    assert torch.all(mine <= best + 1e-6 * sr)


# --------------------------------------------------------------------------
# Error invariant |w - deq(quant(w))| <= s/2 (+ rounding slack), and the
# degenerate constant group.
# --------------------------------------------------------------------------

def _ulp(t: torch.Tensor) -> torch.Tensor:
    """Spacing of the dtype's grid at |t|, as float64."""
    f = torch.finfo(t.dtype)
    a = t.double().abs()
    e = torch.floor(torch.log2(torch.clamp(a, min=f.tiny)))
    return torch.pow(2.0, e) * f.eps


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("bits", ALL_BITS)
def test_error_within_half_scale(dtype, bits):
    w = wl.with_outliers((32, 512), 31 + bits, 0.02, 0.01, 20.0, dtype)
    for gs in (32, 64, 128):
        wq, s, b = oracle.quantize(w, gs, bits)
        deq = oracle.dequantize(wq, s, b, gs, bits)
        sr = s.repeat_interleave(gs, dim=1)
        br = b.repeat_interleave(gs, dim=1)
        err = (w.double() - deq.double()).abs()
        slack = (0.5 * sr.double() * (1 + 2.0 ** -10)
                 + 0.5 * _ulp(br) + QMAX[bits] * 0.5 * _ulp(sr) + 0.5 * _ulp(deq))
        assert torch.all(err <= slack)


@pytest.mark.parametrize("dtype", DTYPES)
def test_constant_group_is_exact(dtype):
    w = torch.full((2, 64), -0.375, dtype=dtype)
    w[1] = 5.0
    wq, s, b = oracle.quantize(w, 32, 4)
    assert torch.all(s == 0) and torch.all(oracle.unpack_codes(wq, 4) == 0)
    assert torch.equal(oracle.dequantize(wq, s, b, 32, 4), w)


# --------------------------------------------------------------------------
# The oracle's dtype rounding against torch's (a library routine): catches a
# truncating conversion or a wrong tie rule in the stored scales and biases.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
def test_dtype_rounding_matches_library(dtype):
    v = wl.normal((4096,), 41, 10.0, torch.float32)
    # exact ties: values halfway between two neighbours of the target grid
    a = torch.tensor([1.0, 3.0, -7.0, 0.15625, 1000.0], dtype=torch.float32).to(dtype)
    half = (_ulp(a) / 2).float()
    ties = torch.cat([a.float() + half, a.float() - half])
    v = torch.cat([v, ties])
    assert torch.equal(oracle.round_to_dtype(v, dtype), v.to(dtype))


# --------------------------------------------------------------------------
# The product reduces to a library float64 matmul when the weight is on the
# grid (dequantize is then exact): catches a transposed operand, groups on the
# wrong axis for transpose=False, a dropped bias term.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", ALL_BITS)
@pytest.mark.parametrize("transpose", [True, False])
def test_matmul_reduces_to_dense_on_grid(bits, transpose):
    w, _, _, _ = _on_grid(48, 128, 32, bits, torch.float32, seed=77 + bits)
    # transpose=True stores W as [out=48, in=128]; False stores [in=48, out=128].
    wq, s, b = oracle.quantize(w, 32, bits)
    k = 128 if transpose else 48
    x = wl.normal((5, k), 78, 1.0, torch.float32)
    y = oracle.quantized_matmul(x, wq, s, b, transpose, 32, bits)
    dense = w.double().T if transpose else w.double()
    assert torch.allclose(y, torch.matmul(x.double(), dense), rtol=1e-12, atol=1e-12)


def test_one_hot_rows_pick_weight_columns():
    w = wl.normal((16, 64), 81, 1.0, torch.float32)        # [out, in]
    wq, s, b = oracle.quantize(w, 64, 4)
    deq = oracle.dequantize(wq, s, b, 64, 4)
    x = torch.zeros((3, 64))
    x[0, 0] = 1.0
    x[1, 63] = 1.0
    x[2, 17] = 2.0
    y = oracle.quantized_matmul(x, wq, s, b, True, 64, 4)
    assert torch.equal(y[0], deq[:, 0].double())
    assert torch.equal(y[1], deq[:, 63].double())
    assert torch.equal(y[2], 2.0 * deq[:, 17].double())


def test_gather_defaults_broadcast():
    """lhs None: x[b] (or x[0] when x has one batch entry); rhs None: expert b."""
    w = wl.normal((2, 8, 64), 90, 1.0, torch.float32)
    wq, s, b = oracle.quantize(w, 64, 4)
    deq = oracle.dequantize(wq, s, b, 64, 4).double()
    x1 = wl.normal((1, 3, 64), 91, 1.0, torch.float32)
    y = oracle.gather_qmm(x1, wq, s, b, None, torch.tensor([1, 0, 1]), True, 64, 4)
    for i, e in enumerate([1, 0, 1]):
        assert torch.allclose(y[i], x1[0].double() @ deq[e].T, rtol=0, atol=1e-12)
    x2 = wl.normal((2, 3, 64), 92, 1.0, torch.float32)
    y = oracle.gather_qmm(x2, wq, s, b, None, None, True, 64, 4)
    for i in range(2):
        assert torch.allclose(y[i], x2[i].double() @ deq[i].T, rtol=0, atol=1e-12)


# --------------------------------------------------------------------------
# quantized_dense (Emily.Quantization.Layers): x @ W (+ bias), the bias a tensor
# over the output features or a number.  Catches a dropped bias, a bias
# broadcast along the rows instead of the features, a bias scaled or added
# twice, the number form ignored.
# --------------------------------------------------------------------------

@pytest.mark.parametrize("transpose", [True, False])
def test_dense_one_hot_rows_give_weight_column_plus_bias(transpose):
    # transpose=True: W stored [out=16, in=64]; False: W stored [in=64, out=32]
    # (quantized along out, one group of 32).
    if transpose:
        w = wl.normal((16, 64), 93, 1.0, torch.float32)
        wq, s, b = oracle.quantize(w, 64, 4)
        col = lambda j: oracle.dequantize(wq, s, b, 64, 4)[:, j]
    else:
        w = wl.normal((64, 32), 93, 1.0, torch.float32)       # out = 32, one group of 32
        wq, s, b = oracle.quantize(w, 32, 4)
        col = lambda j: oracle.dequantize(wq, s, b, 32, 4)[j, :]
    n = 16 if transpose else 32
    gs = 64 if transpose else 32
    bias = torch.arange(n, dtype=torch.float32) * 0.25 - 1.0
    x = torch.zeros((3, 64))
    x[0, 0] = 1.0
    x[1, 63] = 1.0
    x[2, 17] = -2.0
    y = oracle.quantized_dense(x, wq, s, b, bias, transpose, gs, 4)
    assert y.shape == (3, n)
    assert torch.equal(y[0], col(0).double() + bias.double())
    assert torch.equal(y[1], col(63).double() + bias.double())
    assert torch.equal(y[2], -2.0 * col(17).double() + bias.double())


def test_dense_on_grid_reduces_to_library_product_plus_bias():
    w, _, _, _ = _on_grid(48, 128, 32, 4, torch.float32, seed=95)   # [out=48, in=128]
    wq, s, b = oracle.quantize(w, 32, 4)
    x = wl.normal((5, 128), 96, 1.0, torch.float32)
    bias = wl.normal((48,), 97, 1.0, torch.float32)
    y = oracle.quantized_dense(x, wq, s, b, bias, True, 32, 4)
    ref = torch.nn.functional.linear(x.double(), w.double(), bias.double())
    assert torch.allclose(y, ref, rtol=1e-12, atol=1e-12)


def test_dense_number_bias_equals_constant_tensor():
    w = wl.normal((24, 64), 98, 1.0, torch.float32)
    wq, s, b = oracle.quantize(w, 64, 4)
    x = wl.normal((4, 64), 99, 1.0, torch.float32)
    y_num = oracle.quantized_dense(x, wq, s, b, 0.75, True, 64, 4)
    y_vec = oracle.quantized_dense(x, wq, s, b, torch.full((24,), 0.75), True, 64, 4)
    y0 = oracle.quantized_dense(x, wq, s, b, 0, True, 64, 4)
    assert torch.equal(y_num, y_vec)
    assert torch.allclose(y_num - y0, torch.full((4, 24), 0.75, dtype=torch.float64),
                          rtol=0, atol=1e-12)
