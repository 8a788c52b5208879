"""GPU parity of the decode tensor-core kernel (1..16 activation rows, W
stored [N, K], 2- and 4-bit codes) against the oracle's dequantize-then-float64
product, on the forced path and through the automatic choice."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_path():
    yield
    qb.qmm_set_path("auto")


def run(x, w, gs, bits, path="decode_tc"):
    wq, s, b = oracle.quantize(w, gs, bits)
    ref = oracle.quantized_matmul(x, wq, s, b, True, gs, bits)
    qb.qmm_set_path(path)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, gs, bits)
    qb.qmm_device_status()
    assert y.shape == ref.shape and y.dtype == s.dtype
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[s.dtype], f"rel err {err}"


@pytest.mark.parametrize("m", list(range(1, 17)))
@pytest.mark.parametrize("bits", [2, 4])
def test_every_row_count(m, bits):
    """Each activation-row count (the kernel is built for 1, 2, 4, 8 or 16
    rows; counts in between leave rows of the operand unused)."""
    w = wl.with_outliers((1000, 1024), seed=60 + bits, dtype=torch.bfloat16)
    x = wl.normal((m, 1024), 61 + m, 1.0, torch.bfloat16)
    run(x, w, 64, bits)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("n,k", [(1, 1024), (7, 512), (200, 4096), (4099, 1024), (20000, 512)])
@pytest.mark.parametrize("m", [1, 3, 16])
def test_shapes(dtype, bits, gs, n, k, m):
    """Ragged N (one row; fewer rows than CTAs; more rows than 124 per SM, so
    several waves), K from one activation stage to eight, every group size."""
    if (k // gs) % 8:
        pytest.skip("needs groups per row a multiple of 8")
    w = wl.with_outliers((n, k), seed=n + k + bits + gs, dtype=dtype)
    x = wl.normal((m, k), k + m + 3, 1.0, dtype)
    run(x, w, gs, bits)


def test_one_launch_per_call():
    """The kernel serves every M in 1..16 with one launch."""
    w = wl.normal((512, 1024), 70, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    qb.qmm_set_path("decode_tc")
    for m in (1, 5, 16):
        x = wl.normal((m, 1024), 71, 1.0, torch.bfloat16).cuda()
        n0 = qb.qmm_launch_count()
        qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4)
        assert qb.qmm_launch_count() - n0 == 1


def test_refuses_what_it_cannot_run():
    w = wl.normal((64, 1024), 72, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 8))  # 8-bit codes
    x = wl.normal((2, 1024), 73, 1.0, torch.bfloat16).cuda()
    qb.qmm_set_path("decode_tc")
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 8)
    assert e.value.status == 2


def test_repeated_calls_agree_bit_for_bit():
    """Consecutive calls overlap (programmatic dependent launch) and must not
    disturb each other's results."""
    w = wl.with_outliers((14336, 4096), seed=74, dtype=torch.bfloat16).cuda()
    x = wl.normal((4, 4096), 75, 1.0, torch.bfloat16).cuda()
    wq, s, b = qb.qmm_quantize(w, 64, 4)
    qb.qmm_set_path("decode_tc")
    y0 = qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4).clone()
    ys = [qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4) for _ in range(8)]
    torch.cuda.synchronize()
    for y in ys:
        assert torch.equal(y, y0)
