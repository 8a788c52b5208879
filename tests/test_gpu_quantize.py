"""GPU parity: quantize and dequantize are bit-exact against the oracle."""
import pytest
import torch

import oracle
from parity import words
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu

DTYPES = [torch.float32, torch.bfloat16, torch.float16]


def check_quantize(w_cpu, gs, bits):
    wq, s, b = qb.qmm_quantize(w_cpu.cuda(), gs, bits)
    torch.cuda.synchronize()
    rq, rs, rb = oracle.quantize(w_cpu, gs, bits)
    assert torch.equal(words(wq), words(rq))
    assert torch.equal(s.cpu(), rs)
    assert torch.equal(b.cpu(), rb)
    d = qb.qmm_dequantize(wq, s, b, gs, bits)
    torch.cuda.synchronize()
    assert torch.equal(d.cpu(), oracle.dequantize(rq, rs, rb, gs, bits))


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
def test_quantize_dequantize_bit_exact(dtype, bits, gs):
    # 37 rows x 640 cols: several thread blocks and a ragged last block.
    w = wl.with_outliers((37, 640), seed=100 + bits + gs, dtype=dtype)
    check_quantize(w, gs, bits)


@pytest.mark.parametrize("bits", [2, 4, 8])
def test_quantize_rank3_and_minimal_row(bits):
    check_quantize(wl.normal((3, 5, 128), 7, 1.0, torch.bfloat16), 64, bits)
    check_quantize(wl.normal((1, 32), 8, 1.0, torch.float32), 32, bits)


def test_quantize_degenerate_and_iota():
    w = torch.zeros((4, 128), dtype=torch.bfloat16)
    w[1] = 3.5
    w[2, 5] = -1.0
    check_quantize(w, 64, 4)
    check_quantize(wl.iota((4, 64)), 64, 4)
    check_quantize(wl.iota((4, 128)), 64, 4)


def test_quantize_empty_rows():
    w = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    wq, s, b = qb.qmm_quantize(w, 64, 4)
    assert wq.shape == (0, 16) and s.shape == (0, 2)


@pytest.mark.slow
def test_quantize_full_decode_weight():
    """The 14336 x 4096 bf16 weight of the decode/prefill workloads, int4 and int8."""
    w = wl.normal((14336, 4096), 1, 0.02, torch.bfloat16)
    for bits in (4, 8):
        check_quantize(w, 64, bits)


def test_invalid_args_raise():
    w = torch.zeros((4, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantize(w, 64, 4)
    assert e.value.status == 1
    with pytest.raises(qb.QmmError) as e:      # nvfp4 fixes group_size 16
        qb.qmm_quantize(w, 32, 4, mode="nvfp4")
    assert e.value.status == 1
    with pytest.raises(qb.QmmError) as e:      # bits 5 is no format
        qb.qmm_quantize(w, 32, 5)
    assert e.value.status == 1


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("bits", [2, 4, 8])
def test_quantize_codes_on_and_next_to_ties(dtype, bits):
    """Elements whose quotient (v - b) / s lies exactly on a half integer or a
    few units in the last place from one: the code must be the rounded IEEE
    quotient's, ties to even, in every group."""
    qmax = (1 << bits) - 1
    g = torch.Generator().manual_seed(bits)
    rows = []
    for r in range(64):
        lo = float(torch.randn(1, generator=g)) * 10 ** (r % 7 - 3)
        step = float(torch.rand(1, generator=g) + 0.05) * 10 ** (r % 5 - 2)
        if r % 4 == 0:          # power-of-two step: s and b exact, so exact ties
            step = 2.0 ** (r % 9 - 4)
            lo = -float(r) * step
        row = torch.empty(128, dtype=torch.float64)
        row[0], row[1] = lo, lo + qmax * step
        k = torch.randint(0, qmax, (126,), generator=g).double()
        nudge = torch.tensor([0.0, 1e-7, -1e-7, 1e-6, -1e-6, 1e-4, -1e-4, 2e-3, -2e-3] * 14)
        row[2:] = lo + (k + 0.5 + nudge) * step
        rows.append(row)
    w = torch.stack(rows).to(dtype)
    check_quantize(w, 64, bits)
    check_quantize(w, 32, bits)
