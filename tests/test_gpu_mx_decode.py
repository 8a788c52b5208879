"""GPU parity of the streaming decode kernel on microscaled E2M1 weights
(mxfp4: E8M0 scale per 32 codes; nvfp4: E4M3 scale per 16 codes), 1..4
activation rows, W stored [N, K], against the oracle's dequantize-then-float64
product; and bit-for-bit repetition of the decode kernel's results."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu

FP4 = ["mxfp4", "nvfp4"]


def gb(mode):
    return oracle.MX_MODES[mode][:2]


def run(x, w, mode):
    gs, bits = gb(mode)
    wq, s, _ = oracle.quantize(w, gs, bits, mode)
    ref = oracle.quantized_matmul(x, wq, s, None, True, gs, bits, mode)
    n0 = qb.qmm_launch_count()
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), None, True, gs, bits, mode)
    qb.qmm_device_status()
    if x.shape[1] <= 12288:
        # one launch for up to 4 rows (two 16-byte slices per lane, past 12288
        # codes, fit the registers for one row at a time)
        assert qb.qmm_launch_count() - n0 == 1
    assert y.shape == ref.shape and y.dtype == x.dtype
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[x.dtype], f"rel err {err}"
    return y


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", FP4)
@pytest.mark.parametrize("n,k", [(1, 512), (7, 1024), (333, 4096), (4099, 512), (300, 16384)])
@pytest.mark.parametrize("m", [1, 2, 3, 4])
def test_shapes(dtype, mode, n, k, m):
    """Ragged N (one row; fewer rows than CTAs; several stages per CTA), K
    from one scale row of 16 bytes to two 16-byte slices per lane."""
    w = wl.with_outliers((n, k), seed=n + k + m, std=0.5, dtype=dtype)
    x = wl.normal((m, k), k + m, 1.0, dtype)
    run(x, w, mode)


@pytest.mark.parametrize("mode", FP4)
def test_edge_groups(mode):
    """Groups of zeros, exact element-format ties, negative zeros, codes at
    the format's largest magnitude, huge and tiny scales, beside ordinary
    rows."""
    k = 1024
    w = wl.with_outliers((64, k), 100, 0.02, 0.01, 20.0, torch.float32)
    w[0, :32] = 0.0
    w[1, :32] = torch.tensor([6.0, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0] * 4)
    w[2, :32] = torch.tensor([-0.0, -1e-6, 1e-6, -3.0] * 8)
    w[3, :32] = torch.linspace(-7.9, 7.9, 32)
    w[4, :32] = torch.linspace(-1e30, 1e30, 32)
    w[5, :32] = torch.linspace(-1e-30, 1e-30, 32)
    w[6] = -6.0
    x = wl.normal((3, k), 101, 1.0, torch.bfloat16)
    run(x, w.to(torch.bfloat16), mode)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("mode", FP4)
def test_activation_magnitudes(dtype, mode):
    """Block fixed point per 32 activations: slices that mix 1e3 with 1e-3,
    all-zero slices, single nonzero elements, values near the top of the
    format's range."""
    k = 2048
    x = wl.normal((4, k), 102, 1.0, torch.float32)
    x[0, 0::2] *= 1e3
    x[0, 1::2] *= 1e-3
    x[1, :64] = 0.0
    x[1, 70] = 7.0
    x[2] = 0.0
    x[2, 3] = -1.0
    x[3, ::64] = 6.0e4 if dtype == torch.float16 else 1e30
    w = wl.normal((300, k), 103, 0.02 if dtype == torch.float16 else 0.5, torch.float32)
    run(x.to(dtype), w.to(dtype), mode)


@pytest.mark.parametrize("mode", FP4)
def test_decode_workload_full_size(mode):
    """x [M, 4096] against W [14336, 4096], M in 1 and 4."""
    for m in (1, 4):
        c = wl.decode_case(m)
        run(c.x, c.w, mode)


@pytest.mark.parametrize("mode", ["affine4", "affine2", "affine8", "mxfp4", "nvfp4"])
@pytest.mark.parametrize("m", [1, 4])
def test_repeated_calls_agree_bit_for_bit(mode, m):
    """Every row's partial sums are combined in a fixed order: a call repeats
    its result bit for bit, also when calls overlap (programmatic dependent
    launch) and K spreads a row over several warps."""
    k = 8192
    w = wl.with_outliers((4096, k), seed=104, dtype=torch.bfloat16).cuda()
    if mode.startswith("affine"):
        gs, bits, md = 64, int(mode[6:]), "affine"
    else:
        (gs, bits), md = gb(mode), mode
    wq, s, b = qb.qmm_quantize(w, gs, bits, md)
    xs = [wl.normal((m, k), 105 + i, 1.0, torch.bfloat16).cuda() for i in range(2)]
    y0 = [qb.qmm_quantized_matmul(x, wq, s, b, True, gs, bits, md).clone() for x in xs]
    torch.cuda.synchronize()
    ys = [qb.qmm_quantized_matmul(xs[i % 2], wq, s, b, True, gs, bits, md).clone() for i in range(8)]
    torch.cuda.synchronize()
    qb.qmm_device_status()
    for i, y in enumerate(ys):
        assert torch.equal(y, y0[i % 2]), f"call {i}"
