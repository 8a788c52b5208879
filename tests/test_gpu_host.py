"""GPU tests of qmm_quantized_matmul_host: x copied in from host memory, the
product, y copied back, one C call per step (page-locked buffers by copy
kernels chained with the product, pageable ones by the copy engines)."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("m", [1, 4, 40])
def test_matches_the_device_call(pinned, m):
    w = wl.with_outliers((1000, 2048), seed=90 + m, dtype=torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    x = wl.normal((m, 2048), 91 + m, 1.0, torch.bfloat16)
    x_host = x.pin_memory() if pinned else x.clone()
    y_host = torch.empty((m, 1000), dtype=torch.bfloat16)
    if pinned:
        y_host = y_host.pin_memory()
    x_dev = torch.empty_like(x, device="cuda")
    y_dev = torch.empty((m, 1000), dtype=torch.bfloat16, device="cuda")
    qb.qmm_quantized_matmul_host(x_host, x_dev, wq, s, b, y_dev, y_host, True, 64, 4)
    torch.cuda.synchronize()
    qb.qmm_device_status()
    y_ref = qb.qmm_quantized_matmul(x.cuda(), wq, s, b, True, 64, 4)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_ref.cpu())
    ref = oracle.quantized_matmul(x, wq.cpu(), s.cpu(), b.cpu(), True, 64, 4)
    assert row_rel_err(y_host, ref) <= REL_TOL[torch.bfloat16]


def test_back_to_back_steps_keep_their_own_inputs():
    """Six calls without synchronization, three inputs in turn, one device x/y
    pair, six host outputs: each step's copy in waits for the previous product
    to have read x_dev, and its copy out reads its own product's y_dev."""
    w = wl.with_outliers((14336, 4096), seed=92, dtype=torch.bfloat16)
    wq, s, b = qb.qmm_quantize(w.cuda(), 64, 4)
    xs = [wl.normal((1, 4096), 93 + i, 1.0, torch.bfloat16).pin_memory() for i in range(3)]
    ys = [torch.empty((1, 14336), dtype=torch.bfloat16).pin_memory() for _ in range(6)]
    x_dev = torch.empty((1, 4096), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((1, 14336), dtype=torch.bfloat16, device="cuda")
    torch.cuda.synchronize()
    for i in range(6):
        qb.qmm_quantized_matmul_host(xs[i % 3], x_dev, wq, s, b, y_dev, ys[i], True, 64, 4)
    torch.cuda.synchronize()
    qb.qmm_device_status()
    for i in range(6):
        ref = qb.qmm_quantized_matmul(xs[i % 3].cuda(), wq, s, b, True, 64, 4)
        torch.cuda.synchronize()
        assert torch.equal(ys[i], ref.cpu()), f"step {i}"


def test_f32_and_odd_sizes():
    """f32 (SIMT kernels) and an output whose byte count is not a multiple of
    16 (the copy kernel falls back to byte copies)."""
    w = wl.normal((37, 128), 94, 0.1, torch.float32)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    x = wl.normal((3, 128), 95, 1.0, torch.float32)
    x_host, y_host = x.pin_memory(), torch.empty((3, 37), dtype=torch.float32).pin_memory()
    x_dev, y_dev = torch.empty_like(x, device="cuda"), torch.empty((3, 37), device="cuda")
    qb.qmm_quantized_matmul_host(x_host, x_dev, wq, s, b, y_dev, y_host, True, 64, 4)
    torch.cuda.synchronize()
    ref = oracle.quantized_matmul(x, wq.cpu(), s.cpu(), b.cpu(), True, 64, 4)
    assert row_rel_err(y_host, ref) <= REL_TOL[torch.float32]


@pytest.mark.parametrize("m,launches", [(1, 2), (4, 2), (40, 3)])
def test_prepared_mapped_call(m, launches):
    """Page-locked buffers: the prepared call looks their mappings up once and
    goes through qmm_quantized_matmul_mapped.  With 1..4 rows the decode
    kernel writes y_host itself (copy in + product: two launches); with 40
    rows the GEMM result is copied out by a kernel (three launches).  y_dev
    holds the result too."""
    w = wl.with_outliers((2000, 4096), seed=96 + m, dtype=torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    x = wl.normal((m, 4096), 97 + m, 1.0, torch.bfloat16)
    x_host, y_host = x.pin_memory(), torch.zeros((m, 2000), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x, device="cuda")
    y_dev = torch.zeros((m, 2000), dtype=torch.bfloat16, device="cuda")
    call = qb.HostMatmul(x_host, x_dev, wq, s, b, y_dev, y_host, True, 64, 4)
    assert call._fn is qb.lib().qmm_quantized_matmul_mapped
    n0 = qb.qmm_launch_count()
    call()
    torch.cuda.synchronize()
    qb.qmm_device_status()
    assert qb.qmm_launch_count() - n0 == launches
    y_ref = qb.qmm_quantized_matmul(x.cuda(), wq, s, b, True, 64, 4)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_ref.cpu()) and torch.equal(y_dev, y_ref)


def test_prepared_calls_back_to_back():
    """Three prepared calls (three weights, shared x_dev / y_dev, own host
    outputs) enqueued twice over without synchronization."""
    ws = [wl.with_outliers((3000, 2048), seed=98 + i, dtype=torch.bfloat16) for i in range(3)]
    packs = [tuple(t.cuda() for t in oracle.quantize(w, 64, 4)) for w in ws]
    xs = [wl.normal((1, 2048), 99 + i, 1.0, torch.bfloat16).pin_memory() for i in range(3)]
    ys = [torch.empty((1, 3000), dtype=torch.bfloat16).pin_memory() for _ in range(6)]
    x_dev = torch.empty((1, 2048), dtype=torch.bfloat16, device="cuda")
    y_dev = torch.empty((1, 3000), dtype=torch.bfloat16, device="cuda")
    calls = [qb.HostMatmul(xs[i % 3], x_dev, *packs[i % 3], y_dev, ys[i], True, 64, 4)
             for i in range(6)]
    torch.cuda.synchronize()
    for c in calls:
        c()
    torch.cuda.synchronize()
    qb.qmm_device_status()
    for i in range(6):
        ref = qb.qmm_quantized_matmul(xs[i % 3].cuda(), *packs[i % 3], True, 64, 4)
        torch.cuda.synchronize()
        assert torch.equal(ys[i], ref.cpu()), f"step {i}"
