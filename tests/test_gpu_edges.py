"""GPU parity on inputs that the kernels treat specially: activations of mixed
magnitude (the decode kernel's block fixed point), a weight written by
qmm_quantize just before a decode call on the same stream (the decode kernel's
early start), and the bits/group/layout sweep at its own 4096 x 4096 size."""
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


def mixed_activations(m, k, dtype, seed):
    """N(0,1) rows whose 8-element slices (16 bytes) mix magnitudes: 1e3 beside
    1e-3, exact zeros and subnormals in every slice, plus (f16) values near the
    top of the range, and one row of very large (bf16) or very small values."""
    x = wl.normal((m, k), seed, 1.0, torch.float32)
    sl = x.view(m, k // 8, 8)
    sl[:, :, 0] = 1e3
    sl[:, :, 1] = 1e-3
    sl[:, :, 2] = 0.0
    sub = 1e-39 if dtype == torch.bfloat16 else 3e-6     # below the normal range
    sl[:, :, 3] = sub
    sl[:, ::2, 4] = -sub
    if dtype == torch.float16:
        sl[0, :2, 5] = 60000.0                            # near the top, 65504
    if m > 1:   # bf16: values up to 1e36; f16: a row at +-2000 (the output stays finite)
        x[1] = x[1] * 1e33 if dtype == torch.bfloat16 else x[1].clamp(-1, 1) * 2000.0
    if m > 2:
        x[2] = x[2] * 1e-30 if dtype == torch.bfloat16 else x[2] * 1e-3
    return x.to(dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("m", [1, 2, 3, 4])
def test_decode_mixed_magnitude_activations(dtype, bits, m):
    n, k, gs = 640, 4096, 64
    # (f16: no outliers, so that 60000 * w stays inside the f16 range)
    w = (wl.with_outliers((n, k), seed=40 + bits, dtype=dtype) if dtype == torch.bfloat16
         else wl.normal((n, k), 40 + bits, 0.02, dtype))
    x = mixed_activations(m, k, dtype, seed=41 + m)
    assert torch.isfinite(x.float()).all()
    wq, s, b = oracle.quantize(w, gs, bits)
    ref = oracle.quantized_matmul(x, wq, s, b, True, gs, bits)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, gs, bits)
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[dtype], f"rel err {err}"


@pytest.mark.parametrize("reuse", [False, True])
def test_quantize_then_decode_same_stream_no_sync(reuse):
    """qmm_quantize writes a weight and a one-row decode call reads it right
    after, on the same stream with no synchronisation; several rounds, into
    fresh buffers or into the very buffers the previous call read."""
    n, k, gs, bits = 14336, 4096, 64, 4
    dev = torch.device("cuda")
    x = wl.normal((1, k), 51, 1.0, torch.bfloat16)
    ws = [wl.normal((n, k), 52 + i, 0.02, torch.bfloat16) for i in range(3)]
    wd = [w.to(dev) for w in ws]
    xd = x.to(dev)
    bufs = None
    ys = []
    torch.cuda.synchronize()
    for w in wd:
        if reuse and bufs is not None:
            packed = qb.qmm_quantize(w, gs, bits, out=bufs)
        else:
            packed = qb.qmm_quantize(w, gs, bits)
        bufs = packed
        ys.append(qb.qmm_quantized_matmul(xd, *packed, True, gs, bits).clone())
    torch.cuda.synchronize()
    qb.qmm_device_status()
    for w, y in zip(ws, ys):
        wq, s, b = oracle.quantize(w, gs, bits)
        ref = oracle.quantized_matmul(x, wq, s, b, True, gs, bits)
        err = row_rel_err(y, ref)
        assert err <= REL_TOL[torch.bfloat16], f"rel err {err}"


@pytest.fixture(scope="module")
def sweep_weight():
    return wl.sweep_weight()


@pytest.mark.slow
@pytest.mark.parametrize("bits,gs", [(2, 32), (4, 64), (8, 128), (4, 32), (2, 128), (8, 64)])
@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("m", [1, 16, 256])
def test_sweep_full_size(sweep_weight, bits, gs, transpose, m):
    """The sweep workload at its own size: W bf16 [4096, 4096] ~ N(0, 0.02^2)
    with 1 % outliers x20, x [m, 4096]; for m = 256 the comparison uses 48
    sampled rows spread over the activation tiles."""
    wq, s, b = oracle.quantize(sweep_weight, gs, bits)
    x = wl.sweep_x(m)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), transpose, gs, bits)
    torch.cuda.synchronize()
    rows = torch.arange(m) if m <= 16 else torch.cat(
        [torch.arange(0, 256, 64) + o for o in (0, 1, 15, 16, 31, 33, 47, 48, 62, 63, 17, 40)])
    ref = oracle.quantized_matmul(x[rows], wq, s, b, transpose, gs, bits)
    err = row_rel_err(y.cpu()[rows], ref)
    assert err <= REL_TOL[torch.bfloat16], f"rel err {err}"
