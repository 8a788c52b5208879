"""GPU parity of the microscaled modes (mxfp4, mxfp8, nvfp4): quantize and
dequantize bit for bit against the oracle, the products within the stated
tolerance, through the C ABI."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MODES = ["mxfp4", "mxfp8", "nvfp4"]


def gb(mode):
    return oracle.MX_MODES[mode][:2]


def special_weight(rows, cols, seed, dtype):
    """N(0, 0.02^2) rows plus groups that hit the edge cases: all zeros, exact
    element-format ties, negative zeros and values that round to zero,
    saturation, a huge and a tiny group."""
    w = wl.with_outliers((rows, cols), seed, 0.02, 0.01, 20.0, torch.float32)
    w[0, :32] = 0.0
    w[1, :32] = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4)
    w[2, :32] = torch.tensor([-0.0, -1e-6, 1e-6, -3.0] * 8)
    w[3, :32] = torch.linspace(-7.9, 7.9, 32)
    big = 6e4 if dtype == torch.float16 else 1e30
    w[4, :32] = torch.linspace(-big, big, 32)
    w[5, :32] = torch.linspace(-1e-4, 1e-4, 32) if dtype == torch.float16 else torch.linspace(-1e-30, 1e-30, 32)
    return w.to(dtype)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("rows,cols", [(7, 64), (130, 512), (1000, 1024)])
def test_quantize_dequantize_bit_exact(dtype, mode, rows, cols):
    gs, bits = gb(mode)
    w = special_weight(rows, cols, rows + cols + bits, dtype)
    rq, rs, rb = oracle.quantize(w, gs, bits, mode)
    assert rb is None
    wq, s, b = qb.qmm_quantize(w.cuda(), gs, bits, mode)
    torch.cuda.synchronize()
    assert b is None
    assert torch.equal(s.cpu(), rs), "scale bytes differ"
    assert torch.equal(wq.cpu(), rq), "packed codes differ"
    for odt in (torch.float32, torch.bfloat16, torch.float16):
        d = qb.qmm_dequantize(wq, s, None, gs, bits, mode, dtype=odt)
        ref = oracle.dequantize(rq, rs, None, gs, bits, mode, odt)
        torch.cuda.synchronize()
        assert torch.equal(d.cpu().view(torch.int16 if odt != torch.float32 else torch.int32),
                           ref.view(torch.int16 if odt != torch.float32 else torch.int32))


@pytest.mark.parametrize("mode", MODES)
def test_full_size_weight_bit_exact(mode):
    gs, bits = gb(mode)
    w = wl.normal((14336, 4096), 1, 0.02, torch.bfloat16)
    rq, rs, _ = oracle.quantize(w, gs, bits, mode)
    wq, s, _ = qb.qmm_quantize(w.cuda(), gs, bits, mode)
    torch.cuda.synchronize()
    assert torch.equal(s.cpu(), rs) and torch.equal(wq.cpu(), rq)


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("m", [1, 3, 17])
def test_quantized_matmul(dtype, mode, transpose, m):
    gs, bits = gb(mode)
    n, k = (300, 512) if transpose else (512, 256)      # W stored [n, k] / [k, n]
    rows, cols = (n, k) if transpose else (k, n)
    w = wl.with_outliers((rows, cols), seed=m + bits + gs, std=0.5, dtype=dtype)
    x = wl.normal((m, k), m + 7, 1.0, dtype)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    ref = oracle.quantized_matmul(x, wq, s, None, transpose, gs, bits, mode)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), None, transpose, gs, bits, mode)
    qb.qmm_device_status()
    assert y.dtype == dtype and y.shape == ref.shape
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[dtype], f"rel err {err}"


@pytest.mark.parametrize("mode", MODES)
def test_quantized_dense_with_bias(mode):
    gs, bits = gb(mode)
    w = wl.normal((256, 512), 3, 0.5, torch.bfloat16)
    x = wl.normal((4, 512), 4, 1.0, torch.bfloat16)
    bias = wl.normal((256,), 5, 1.0, torch.bfloat16)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    ref = oracle.quantized_matmul(x, wq, s, None, True, gs, bits, mode) + bias.double()
    y = qb.qmm_quantized_dense(x.cuda(), wq.cuda(), s.cuda(), None, bias.cuda(), True, gs, bits, mode)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


def test_mode_arguments_are_checked():
    w = wl.normal((8, 64), 6, 1.0, torch.bfloat16).cuda()
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantize(w, 64, 4, "mxfp4")               # mxfp4 needs group 32
    assert e.value.status == 1
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantize(w, 32, 8, "nvfp4")               # nvfp4 needs 16 / 4
    assert e.value.status == 1
    wq, s, _ = qb.qmm_quantize(w, 32, 4, "mxfp4")
    x = wl.normal((2, 64), 7, 1.0, torch.bfloat16).cuda()
    with pytest.raises(qb.QmmError) as e:                 # microscaled weights have no biases
        qb.qmm_quantized_matmul(x, wq, s, s.clone(), True, 32, 4, "mxfp4")
    assert e.value.status == 1
    # gather_qmm takes affine weights (its callers pass mode "affine")
    rhs = torch.zeros(2, dtype=torch.int32, device="cuda")
    y = torch.empty((2, 1, 8), dtype=torch.bfloat16, device="cuda")
    st = qb.lib().qmm_gather_qmm(x.data_ptr(), 2, 1, 64, wq.data_ptr(), s.data_ptr(), None, 1, 1, 8,
                                 None, rhs.data_ptr(), 2, 1, 32, 4, b"mxfp4", 0, y.data_ptr(), None, 0,
                                 None)
    assert st == 2


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", ["nvfp4", "mxfp8"])
@pytest.mark.parametrize("m", [1, 5, 64])
def test_qqmm(dtype, mode, m):
    """mlx-rs qqmm: activations quantized on the fly, the weight given packed
    (and once dense), against the oracle's float64 product of the two
    dequantized operands."""
    gs, bits = gb(mode)
    n, k = 200, 512
    w = wl.with_outliers((n, k), seed=m + bits, std=0.5, dtype=dtype)
    x = wl.normal((m, k), m + 11, 1.0, dtype)
    wq, ws, _ = oracle.quantize(w, gs, bits, mode)
    ref = oracle.qqmm(x, wq, ws, gs, bits, mode)
    y = qb.qmm_qqmm(x.cuda(), wq.cuda(), ws.cuda(), mode=mode)
    qb.qmm_device_status()
    assert y.dtype == dtype and y.shape == ref.shape
    assert row_rel_err(y, ref) <= REL_TOL[dtype]
    y2 = qb.qmm_qqmm(x.cuda(), w.cuda(), None, mode=mode)      # dense weight, quantized first
    qb.qmm_device_status()
    assert torch.equal(y, y2)


def test_qqmm_arguments_are_checked():
    x = wl.normal((2, 64), 8, 1.0, torch.bfloat16).cuda()
    w = wl.normal((16, 64), 9, 1.0, torch.bfloat16).cuda()
    wq, ws, _ = qb.qmm_quantize(w, 32, 4, "mxfp4")
    y = torch.empty((2, 16), dtype=torch.bfloat16, device="cuda")
    L = qb.lib()
    args = (x.data_ptr(), 2, 64, 1, wq.data_ptr(), ws.data_ptr(), 16)
    assert L.qmm_qqmm(*args, 32, 4, b"mxfp4", y.data_ptr(), None, 0, None) == 2   # mode not served
    wq8, ws8, _ = qb.qmm_quantize(w, 32, 8, "mxfp8")
    args = (x.data_ptr(), 2, 64, 1, wq8.data_ptr(), ws8.data_ptr(), 16)
    assert L.qmm_qqmm(*args, 32, 8, b"mxfp8", y.data_ptr(), None, 0, None) == 6   # no workspace


@pytest.fixture
def _auto_path():
    yield
    qb.qmm_set_path("auto")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("m,n,k", [(5, 200, 512), (64, 300, 1024), (300, 128, 512), (17, 1000, 2048)])
@pytest.mark.parametrize("path", ["gemm", "gemv"])
def test_products_on_each_path(dtype, mode, m, n, k, path, _auto_path):
    """Microscaled weights on the tensor-core GEMM (each 64-element k-block
    dequantized exactly into tensor memory from E2M1/E4M3 codes and the
    group scale bytes) and on the SIMT kernels."""
    gs, bits = gb(mode)
    w = wl.with_outliers((n, k), seed=m + n + bits, std=0.5, dtype=dtype)
    x = wl.normal((m, k), m + k, 1.0, dtype)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    ref = oracle.quantized_matmul(x, wq, s, None, True, gs, bits, mode)
    qb.qmm_set_path(path)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), None, True, gs, bits, mode)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[dtype]


@pytest.mark.slow
@pytest.mark.parametrize("mode", MODES)
def test_prefill_full_size_sampled(mode):
    """x [2048, 4096] against W [14336, 4096] in a microscaled mode, checked on
    sampled rows spread over the activation tiles."""
    gs, bits = gb(mode)
    c = wl.prefill_case(4)
    wq, s, _ = oracle.quantize(c.w, gs, bits, mode)
    y = qb.qmm_quantized_matmul(c.x.cuda(), wq.cuda(), s.cuda(), None, True, gs, bits, mode)
    torch.cuda.synchronize()
    rows = torch.cat([torch.arange(0, 2048, 256) + o for o in (0, 1, 100, 255)])
    ref = oracle.quantized_matmul(c.x[rows], wq, s, None, True, gs, bits, mode)
    assert row_rel_err(y.cpu()[rows], ref) <= REL_TOL[torch.bfloat16]
