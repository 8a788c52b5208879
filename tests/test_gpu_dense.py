"""GPU parity of quantized_dense (x @ W + bias, the bias added in each kernel's
epilogue) against the oracle's float64 quantized_dense, on every kernel path."""
import ctypes

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


def run(x, w, gs, bits, transpose, bias, path="auto"):
    wq, s, b = oracle.quantize(w, gs, bits)
    ref = oracle.quantized_dense(x, wq, s, b, bias, transpose, gs, bits)
    qb.qmm_set_path(path)
    bias_dev = bias.cuda() if isinstance(bias, torch.Tensor) else bias
    y = qb.qmm_quantized_dense(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), bias_dev, transpose, gs, bits)
    qb.qmm_device_status()
    assert y.shape == ref.shape and y.dtype == s.dtype
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[s.dtype], f"rel err {err}"


def vec(n, dtype, seed=5):
    return wl.normal((n,), seed, 0.5, dtype)


# (name, dtype, bits, gs, transpose, m, n, k, path)
CASES = [
    ("decode_tc_m1", torch.bfloat16, 4, 64, True, 1, 1000, 1024, "decode_tc"),
    ("decode_tc_m5", torch.bfloat16, 2, 64, True, 5, 300, 512, "decode_tc"),
    ("decode_tc_m16_f16", torch.float16, 4, 32, True, 16, 777, 1024, "decode_tc"),
    ("stream_decode_int8", torch.bfloat16, 8, 64, True, 3, 1000, 1024, "auto"),
    ("simt_t_f32", torch.float32, 4, 64, True, 7, 200, 512, "gemv"),
    ("simt_n_f32", torch.float32, 4, 32, False, 3, 512, 256, "gemv"),
    ("simt_t_bf16", torch.bfloat16, 8, 128, True, 2, 130, 512, "gemv"),
    ("gemm_nk", torch.bfloat16, 4, 64, True, 100, 300, 512, "gemm"),
    ("gemm_nk_wide", torch.float16, 8, 64, True, 300, 256, 256, "gemm"),
    ("gemm_nk_stream_k", torch.bfloat16, 8, 64, True, 16, 1024, 2048, "gemm"),
    ("gemm_kn", torch.bfloat16, 4, 64, False, 40, 384, 512, "gemm"),
    ("gemm_kn_m1", torch.bfloat16, 4, 64, False, 1, 1024, 4096, "auto"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("form", ["vector", "number", "zero"])
def test_dense_bias_on_every_path(case, form):
    _, dtype, bits, gs, transpose, m, n, k, path = case
    w = wl.with_outliers((n, k) if transpose else (k, n), seed=m + n + k + bits, dtype=dtype)
    x = wl.normal((m, k), k + m + 9, 1.0, dtype)
    bias = {"vector": vec(n, dtype), "number": -0.375, "zero": 0}[form]
    run(x, w, gs, bits, transpose, bias, path)


def test_zero_bias_equals_quantized_matmul_bit_for_bit():
    w = wl.with_outliers((1000, 1024), seed=11, dtype=torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    for m in (1, 4, 16, 64):
        x = wl.normal((m, 1024), 12 + m, 1.0, torch.bfloat16).cuda()
        y0 = qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4)
        y1 = qb.qmm_quantized_dense(x, wq, s, b, 0, True, 64, 4)
        torch.cuda.synchronize()
        assert torch.equal(y0, y1)


def test_vector_and_number_together_through_the_c_abi():
    """The C entry takes both forms at once: bias[n] + bias_value."""
    n, k, m = 512, 1024, 4
    w = wl.with_outliers((n, k), seed=13, dtype=torch.bfloat16)
    x = wl.normal((m, k), 14, 1.0, torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 4)
    bias = vec(n, torch.bfloat16, 15)
    ref = oracle.quantized_dense(x, wq, s, b, bias, True, 64, 4) + 2.5
    xd, wqd, sd, bd, biasd = (t.cuda() for t in (x, wq, s, b, bias))
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    L = qb.lib()
    st = L.qmm_quantized_dense(xd.data_ptr(), m, k, wqd.data_ptr(), sd.data_ptr(), bd.data_ptr(),
                               1, n, 1, 64, 4, b"affine", biasd.data_ptr(), ctypes.c_double(2.5),
                               y.data_ptr(), None, 0, torch.cuda.current_stream().cuda_stream)
    assert st == 0
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


def test_rejects_misaligned_bias_and_non_finite_number():
    n, k = 64, 512
    wq, s, b = (t.cuda() for t in oracle.quantize(wl.normal((n, k), 16, 0.02, torch.bfloat16), 64, 4))
    x = wl.normal((2, k), 17, 1.0, torch.bfloat16).cuda()
    y = torch.empty((2, n), dtype=torch.bfloat16, device="cuda")
    buf = torch.zeros(n + 1, dtype=torch.bfloat16, device="cuda")
    L = qb.lib()
    args = (x.data_ptr(), 2, k, wq.data_ptr(), s.data_ptr(), b.data_ptr(), 1, n, 1, 64, 4, b"affine")
    st = L.qmm_quantized_dense(*args, buf.data_ptr() + 1, ctypes.c_double(0.0), y.data_ptr(), None, 0,
                               None)
    assert st == 1
    st = L.qmm_quantized_dense(*args, None, ctypes.c_double(float("inf")), y.data_ptr(), None, 0, None)
    assert st == 1
