"""GPU parity for affine 3- and 6-bit codes (Emily.QuantizedWeight, from_dense:
:bits one of [2, 3, 4, 6, 8]): codes run back to back in each row's bit
stream, some straddling two words.  Quantize/dequantize bit for bit, products
(both layouts, gather) within the stated tolerance, against the oracle."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err, words
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _reset_path():
    yield
    qb.qmm_set_path("auto")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [3, 6])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("rows,cols", [(5, 128), (333, 1024)])
def test_quantize_dequantize_bit_exact(dtype, bits, gs, rows, cols):
    w = wl.with_outliers((rows, cols), seed=rows + bits + gs, dtype=dtype)
    w[0, :gs] = 0.25                                       # a constant group
    rq, rs, rb = oracle.quantize(w, gs, bits)
    wq, s, b = qb.qmm_quantize(w.cuda(), gs, bits)
    torch.cuda.synchronize()
    assert torch.equal(words(wq), words(rq))
    assert torch.equal(s.cpu(), rs) and torch.equal(b.cpu(), rb)
    d = qb.qmm_dequantize(wq, s, b, gs, bits)
    torch.cuda.synchronize()
    assert torch.equal(d.cpu(), oracle.dequantize(rq, rs, rb, gs, bits))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [3, 6])
@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("m", [1, 4, 17, 40])
def test_quantized_matmul(dtype, bits, transpose, m):
    n, k = (300, 512) if transpose else (512, 256)
    rows, cols = (n, k) if transpose else (k, n)
    w = wl.with_outliers((rows, cols), seed=m + bits, dtype=dtype)
    x = wl.normal((m, k), m + bits + 1, 1.0, dtype)
    wq, s, b = oracle.quantize(w, 64, bits)
    ref = oracle.quantized_matmul(x, wq, s, b, transpose, 64, bits)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), transpose, 64, bits)
    qb.qmm_device_status()
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[dtype], f"rel err {err}"


@pytest.mark.parametrize("bits", [3, 6])
def test_decode_full_size(bits):
    """x bf16 [1, 4096] against W [14336, 4096] (the decode workload's shape)."""
    c = wl.decode_case(1)
    wq, s, b = oracle.quantize(c.w, 64, bits)
    ref = oracle.quantized_matmul(c.x, wq, s, b, True, 64, bits)
    y = qb.qmm_quantized_matmul(c.x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, bits)
    torch.cuda.synchronize()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


@pytest.mark.parametrize("bits", [3, 6])
def test_gather_and_dense(bits):
    w = wl.with_outliers((4, 256, 512), seed=bits, dtype=torch.bfloat16)
    wq, s, b = oracle.quantize(w, 32, bits)
    x = wl.normal((24, 1, 512), bits + 2, 1.0, torch.bfloat16)
    rhs = wl.zipf_experts(24, 4, 1.2, bits + 3)
    ref = oracle.gather_qmm(x, wq, s, b, None, rhs, True, 32, bits)
    y = qb.qmm_gather_qmm(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), None, rhs.cuda(), True, 32, bits)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]
    bias = wl.normal((256,), bits + 4, 1.0, torch.bfloat16)
    ref = oracle.quantized_dense(x[:, 0], wq[1], s[1], b[1], bias, True, 32, bits)
    y = qb.qmm_quantized_dense(x[:, 0].contiguous().cuda(), wq[1].contiguous().cuda(),
                               s[1].contiguous().cuda(), b[1].contiguous().cuda(), bias.cuda(),
                               True, 32, bits)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [3, 6])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("m,n,k", [(5, 384, 512), (64, 1024, 1024), (300, 128, 512), (17, 1000, 2048)])
def test_tensor_core_products(dtype, bits, gs, transpose, m, n, k):
    """The tcgen05 GEMM with bit-stream codes: each 64-code k-block is BITS
    words of a row (3-bit: staged as 32 bytes from the 16-byte boundary at or
    below it), pairs of codes cut out with a funnel shift; both layouts."""
    if not transpose and n % 128:
        pytest.skip("[K, N] rows of whole 16-byte units need N % 128 == 0 for 3-bit codes")
    rows, cols = (n, k) if transpose else (k, n)
    w = wl.with_outliers((rows, cols), seed=m + n + bits + gs, dtype=dtype)
    x = wl.normal((m, k), m + k + bits, 1.0, dtype)
    wq, s, b = oracle.quantize(w, gs, bits)
    ref = oracle.quantized_matmul(x, wq, s, b, transpose, gs, bits)
    qb.qmm_set_path("gemm")
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), transpose, gs, bits)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[dtype]


def test_three_bit_rows_not_in_16_byte_units():
    """K = 576: a 3-bit row is 216 bytes, which a tensor map cannot stride, so
    the forced tensor-core path refuses and the automatic choice takes the
    SIMT kernel."""
    w = wl.normal((256, 576), 80, 0.02, torch.bfloat16)
    x = wl.normal((40, 576), 81, 1.0, torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 3)
    ref = oracle.quantized_matmul(x, wq, s, b, True, 64, 3)
    args = (x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, 3)
    qb.qmm_set_path("gemm")
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantized_matmul(*args)
    assert e.value.status == 2
    qb.qmm_set_path("auto")
    y = qb.qmm_quantized_matmul(*args)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


@pytest.mark.parametrize("bits", [3, 6])
def test_gather_on_tensor_cores(bits):
    """gather_qmm with 256 tokens over 4 experts (grouped tcgen05 kernel)."""
    w = wl.with_outliers((4, 512, 1024), seed=90 + bits, dtype=torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, bits)
    x = wl.normal((256, 1, 1024), 91 + bits, 1.0, torch.bfloat16)
    rhs = wl.zipf_experts(256, 4, 1.2, 92 + bits)
    ref = oracle.gather_qmm(x, wq, s, b, None, rhs, True, 64, bits)
    y = qb.qmm_gather_qmm(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), None, rhs.cuda(), True, 64, bits)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


@pytest.mark.slow
@pytest.mark.parametrize("bits", [3, 6])
def test_prefill_full_size_sampled(bits):
    """x [2048, 4096] against W [14336, 4096] with 3-/6-bit codes, sampled rows
    spread over the activation tiles."""
    c = wl.prefill_case(4)
    wq, s, b = oracle.quantize(c.w, 64, bits)
    y = qb.qmm_quantized_matmul(c.x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, bits)
    torch.cuda.synchronize()
    rows = torch.cat([torch.arange(0, 2048, 256) + o for o in (0, 1, 100, 255)])
    ref = oracle.quantized_matmul(c.x[rows], wq, s, b, True, 64, bits)
    assert row_rel_err(y.cpu()[rows], ref) <= REL_TOL[torch.bfloat16]
