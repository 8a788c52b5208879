"""GPU parity of the decode tensor-core kernel (integer MMA; 1..16 activation
rows, W stored [N, K], 2- and 4-bit codes) against the oracle's
dequantize-then-float64 product, on the forced path."""
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
    return y, ref


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
    """Ragged N (one row; fewer rows than CTAs; more rows than 128 per SM, so
    several waves), K from one code stage to sixteen, every group size."""
    if (k // gs) % 8:
        pytest.skip("needs groups per row a multiple of 8")
    w = wl.with_outliers((n, k), seed=n + k + bits + gs, dtype=dtype)
    x = wl.normal((m, k), k + m + 3, 1.0, dtype)
    run(x, w, gs, bits)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("gs", [32, 128])
def test_activation_magnitudes(dtype, gs):
    """Block fixed point per (row, group): groups that mix 1e3 with 1e-3,
    all-zero groups, single nonzero elements, and (f16) values near 65504 and
    subnormal; the error stays within 2^-14 of each group's largest |x|."""
    k = 1024
    x = wl.normal((6, k), 62, 1.0, torch.float32)
    x[0, 0::2] *= 1e3
    x[0, 1::2] *= 1e-3
    x[1, :gs] = 0.0
    x[1, gs + 5] = 7.0
    x[2] = 0.0
    x[2, 3] = -1.0
    if dtype == torch.float16:
        x[3, ::64] = 6.0e4           # (sparse, so that the products stay finite in f16)
    else:
        x[3, ::3] = 1e30
        x[4] = 1e-30 * torch.sign(x[4])
    w = wl.with_outliers((300, k), seed=63, dtype=dtype)
    run(x.to(dtype), w, gs, 4)
    if dtype == torch.float16:
        # subnormal activations, against a weight large enough that the outputs
        # are normal f16 values (subnormal outputs would be rounded to a
        # quantum of several percent of themselves)
        xs = (3e-7 * torch.sign(wl.normal((2, k), 64, 1.0, torch.float32))).to(dtype)
        run(xs, wl.normal((300, k), 65, 20.0, dtype), gs, 4)


def test_two_launches_per_call():
    """A prep kernel (activations to block fixed point) and the product, for
    every M in 1..16."""
    w = wl.normal((512, 1024), 70, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    qb.qmm_set_path("decode_tc")
    for m in (1, 5, 16):
        x = wl.normal((m, 1024), 71, 1.0, torch.bfloat16).cuda()
        n0 = qb.qmm_launch_count()
        qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4)
        assert qb.qmm_launch_count() - n0 == 2


def test_refuses_what_it_cannot_run():
    w = wl.normal((64, 1024), 72, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 8))  # 8-bit codes
    x = wl.normal((2, 1024), 73, 1.0, torch.bfloat16).cuda()
    qb.qmm_set_path("decode_tc")
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 8)
    assert e.value.status == 2


def test_needs_its_workspace():
    """Without a workspace, or with one too small, the forced path returns
    QMM_ERR_WORKSPACE and launches nothing."""
    w = wl.normal((256, 1024), 74, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    x = wl.normal((4, 1024), 75, 1.0, torch.bfloat16).cuda()
    y = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    qb.qmm_set_path("decode_tc")
    need = qb.qmm_quantized_matmul_workspace_size(4, 1024, 256, True, 4)
    assert need >= 4096 + 32 * 1024
    L = qb.lib()
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    n0 = qb.qmm_launch_count()
    for ws, nbytes in ((None, 0), (small.data_ptr(), small.numel())):
        st = L.qmm_quantized_matmul_ws(x.data_ptr(), 4, 1024, wq.data_ptr(), s.data_ptr(), b.data_ptr(),
                                       1, 256, 1, 64, 4, b"affine", y.data_ptr(), ws, nbytes, None)
        assert st == 6
    assert qb.qmm_launch_count() == n0


def test_workspace_flag_bytes_stay_zero():
    """The prepared activations go past the workspace's first 4096 bytes, which
    every call leaves zero (the stream-K flags of the GEMM share them)."""
    w = wl.normal((512, 2048), 76, 0.02, torch.bfloat16)
    wq, s, b = (t.cuda() for t in oracle.quantize(w, 64, 4))
    x = wl.normal((16, 2048), 77, 1.0, torch.bfloat16).cuda()
    qb.qmm_set_path("decode_tc")
    need = qb.qmm_quantized_matmul_workspace_size(16, 2048, 512, True, 4)
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:4096].count_nonzero()) == 0
    assert int(ws[4096:].count_nonzero()) > 0
    # a stream-K GEMM call on the same workspace still runs correctly
    qb.qmm_set_path("gemm")
    ref = oracle.quantized_matmul(x.cpu(), *(t.cpu() for t in (wq, s, b)), True, 64, 4)
    y = qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4, workspace=ws)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


def test_decode_workload_full_size():
    """x [M, 4096] against W [14336, 4096], int4 group 64, M in 1, 4, 16."""
    for m in (1, 4, 16):
        c = wl.decode_case(m)
        run(c.x, c.w, 64, 4)


def test_repeated_calls_agree_bit_for_bit():
    """Consecutive calls overlap (programmatic dependent launch: the next
    call's prep kernel waits for the previous product before it rewrites the
    workspace) and must not disturb each other's results."""
    w = wl.with_outliers((14336, 4096), seed=74, dtype=torch.bfloat16).cuda()
    wq, s, b = qb.qmm_quantize(w, 64, 4)
    qb.qmm_set_path("decode_tc")
    xs = [wl.normal((4, 4096), 75 + i, 1.0, torch.bfloat16).cuda() for i in range(3)]
    y0 = [qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4).clone() for x in xs]
    torch.cuda.synchronize()
    ys = [qb.qmm_quantized_matmul(xs[i % 3], wq, s, b, True, 64, 4).clone() for i in range(9)]
    torch.cuda.synchronize()
    for i, y in enumerate(ys):
        assert torch.equal(y, y0[i % 3])


@pytest.mark.parametrize("m", [3, 4, 8])
def test_automatic_path_takes_it_for_two_bit_rows(m):
    """Under the automatic path, 2-bit codes with 3..8 activation rows and a
    workspace run on this kernel (two launches), within the tolerance."""
    w = wl.with_outliers((4096, 4096), seed=80 + m, dtype=torch.bfloat16)
    x = wl.normal((m, 4096), 81 + m, 1.0, torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 2)
    ref = oracle.quantized_matmul(x, wq, s, b, True, 64, 2)
    args = (x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, 2)
    qb.qmm_set_path("auto")
    n0 = qb.qmm_launch_count()
    y = qb.qmm_quantized_matmul(*args)
    qb.qmm_device_status()
    assert qb.qmm_launch_count() - n0 == 2
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]
