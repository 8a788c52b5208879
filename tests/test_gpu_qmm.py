"""GPU parity: quantized_matmul against the oracle's dequantize-then-float64
product, on every kernel path that can run the case."""
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


def run_case(x, w, gs, bits, transpose, path="auto"):
    """Quantize w with the oracle (so both sides share packed inputs), run the
    GPU product on `path` and compare with the oracle's product."""
    wq, s, b = oracle.quantize(w, gs, bits)
    ref = oracle.quantized_matmul(x, wq, s, b, transpose, gs, bits)
    qb.qmm_set_path(path)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), transpose, gs, bits)
    torch.cuda.synchronize()
    assert y.shape == ref.shape and y.dtype == s.dtype
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[s.dtype], f"rel err {err}"
    return err


def test_tiny_f32_case():
    c = wl.tiny_case()
    run_case(c.x, c.w, c.group_size, c.bits, c.transpose, "gemv")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("bits", [2, 4, 8])
@pytest.mark.parametrize("gs", [32, 64, 128])
@pytest.mark.parametrize("transpose", [True, False])
@pytest.mark.parametrize("m", [1, 3, 16])
def test_gemv_small(dtype, bits, gs, transpose, m):
    # W stored [rows, cols]; groups along cols.  Ragged rows (not a multiple of
    # any tile) and a K that spans several chunks.
    rows, cols = (200, 1024) if transpose else (384, 640)
    w = wl.with_outliers((rows, cols), seed=bits * 7 + gs, dtype=dtype)
    k = cols if transpose else rows
    x = wl.normal((m, k), seed=m + 5, dtype=dtype)
    run_case(x, w, gs, bits, transpose, "gemv")


@pytest.mark.parametrize("transpose", [True, False])
def test_gemv_m_larger_than_tile(transpose):
    w = wl.normal((96, 256), 3, 0.02, torch.bfloat16)
    x = wl.normal((37, 256 if transpose else 96), 4, 1.0, torch.bfloat16)
    run_case(x, w, 64, 4, transpose, "gemv")


def test_mlx_rs_quantized_matmul_restated():
    """mlx-rs unit test test_quantized_matmul: m=32, n=k=128, gs 64, 4 bits,
    x and w ~ N(0,1)/sqrt(k), w stored [k, n], transpose=False; |y - x@w_hat| < 1e-3."""
    m, n, k = 32, 128, 128
    x = wl.normal((m, k), 0).float() / k ** 0.5
    w = wl.normal((k, n), 1).float() / k ** 0.5
    wq, s, b = oracle.quantize(w, 64, 4)
    w_hat = oracle.dequantize(wq, s, b, 64, 4)
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), False, 64, 4)
    torch.cuda.synchronize()
    assert (y.cpu() - x @ w_hat).abs().max().item() < 1e-3


def test_empty_problems_are_noops():
    wq, s, b = oracle.quantize(wl.normal((64, 128), 1, 1.0, torch.bfloat16), 64, 4)
    x = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    y = qb.qmm_quantized_matmul(x, wq.cuda(), s.cuda(), b.cuda(), True, 64, 4)
    assert y.shape == (0, 64)


@pytest.mark.slow
@pytest.mark.parametrize("m", [1, 4, 8, 16])
def test_decode_full_size(m):
    """x bf16 [m, 4096] against W [14336, 4096] int4 gs64 (the decode workload)."""
    c = wl.decode_case(m)
    run_case(c.x, c.w, c.group_size, c.bits, c.transpose)


@pytest.mark.parametrize("dtype,bits,gs", [
    (torch.bfloat16, 4, 32), (torch.bfloat16, 4, 64), (torch.bfloat16, 4, 128),
    (torch.bfloat16, 2, 64), (torch.bfloat16, 2, 128),
    (torch.bfloat16, 8, 32), (torch.bfloat16, 8, 128),
    (torch.float16, 4, 64), (torch.float16, 8, 32), (torch.float16, 8, 128), (torch.float16, 2, 64),
])
@pytest.mark.parametrize("n,k", [(1, 4096), (301, 4096), (77, 14336), (1000, 1024),
                                 (4099, 1024), (150, 2048)])
@pytest.mark.parametrize("m", [1, 2, 3, 4])
def test_gemv_few_rows(dtype, bits, gs, n, k, m):
    """1..4 activation rows (the decode-shaped streaming kernel where it
    applies, the general kernel elsewhere): ragged N, K from one slice per
    lane to teams of seven warps."""
    if k % gs:
        pytest.skip("K must be a multiple of the group size")
    w = wl.with_outliers((n, k), seed=n + k + bits, dtype=dtype)
    x = wl.normal((m, k), seed=k + m, dtype=dtype)
    run_case(x, w, gs, bits, True)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (4, 128), (8, 64), (8, 32), (2, 128), (2, 64)])
@pytest.mark.parametrize("m,n,k", [(1, 128, 64), (16, 200, 1024), (17, 256, 128),
                                   (100, 1000, 512), (300, 384, 256)])
def test_gemm_tensor_core(dtype, bits, gs, m, n, k):
    """The tcgen05 path: ragged activation rows (every tile width from 16 to
    256), ragged weight rows, several k-blocks."""
    if k % gs:
        pytest.skip("K must be a multiple of the group size")
    w = wl.with_outliers((n, k), seed=m + n + bits, dtype=dtype)
    x = wl.normal((m, k), seed=k + m, dtype=dtype)
    run_case(x, w, gs, bits, True, "gemm")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,gs", [(4, 64), (4, 32), (4, 128), (8, 64), (8, 32), (2, 128), (2, 64)])
@pytest.mark.parametrize("m,k,n", [(1, 64, 128), (16, 1024, 640), (17, 128, 384),
                                   (100, 512, 1152), (300, 256, 256)])
def test_gemm_tensor_core_kn_layout(dtype, bits, gs, m, k, n):
    """The tcgen05 path with the weight stored [K, N] (transpose = false),
    groups along N: MN-major dequantized tiles, ragged feature tiles."""
    if n % gs:
        pytest.skip("N must be a multiple of the group size")
    w = wl.with_outliers((k, n), seed=m + n + bits, dtype=dtype)
    x = wl.normal((m, k), seed=k + m + 1, dtype=dtype)
    run_case(x, w, gs, bits, False, "gemm")


def test_gemm_kn_ragged_features():
    # 160 features: the second 128-feature tile is 32 wide (TMA zero fill).
    w = wl.with_outliers((128, 160), seed=3, dtype=torch.bfloat16)
    x = wl.normal((40, 128), seed=4, dtype=torch.bfloat16)
    run_case(x, w, 32, 4, False, "gemm")


def test_gemm_path_refuses_unsupported():
    w = wl.normal((64, 96), 1, 1.0, torch.bfloat16)
    wq, s, b = oracle.quantize(w, 32, 4)
    x = wl.normal((8, 96), 2, 1.0, torch.bfloat16).cuda()
    qb.qmm_set_path("gemm")
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_quantized_matmul(x, wq.cuda(), s.cuda(), b.cuda(), True, 32, 4)
    assert e.value.status == 2


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 8])
def test_prefill_full_size_sampled(bits):
    """x [2048, 4096] against W [14336, 4096] (the prefill workload), checked
    on 96 sampled activation rows spread over every 256-row tile."""
    c = wl.prefill_case(bits)
    wq, s, b = oracle.quantize(c.w, c.group_size, c.bits)
    y = qb.qmm_quantized_matmul(c.x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, c.group_size,
                                c.bits)
    torch.cuda.synchronize()
    rows = torch.cat([torch.arange(0, 2048, 256) + o for o in (0, 1, 37, 100, 128, 200, 254, 255,
                                                                 17, 64, 190, 222)])
    ref = oracle.quantized_matmul(c.x[rows], wq, s, b, True, c.group_size, c.bits)
    err = row_rel_err(y.cpu()[rows], ref)
    assert err <= REL_TOL[torch.bfloat16], f"rel err {err}"


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m,k,n", [(16, 4096, 1024), (40, 2048, 640), (64, 1536, 384), (9, 4096, 128)])
def test_gemm_stream_k(bits, m, k, n):
    """Fewer 128-row tiles than SMs with narrow activation tiles: the k-blocks
    of each tile are split over several CTAs (up to eight parts per tile for
    16 x 4096 x 1024) and the parts combined by the tile's owner."""
    w = wl.with_outliers((n, k), seed=n + k + bits, dtype=torch.bfloat16)
    x = wl.normal((m, k), seed=m + k, dtype=torch.bfloat16)
    run_case(x, w, 64, bits, True, "gemm")


def test_gemm_stream_k_deterministic():
    """The owner adds the parts in a fixed order, so repeated calls agree bit
    for bit."""
    w = wl.with_outliers((1024, 4096), seed=5, dtype=torch.bfloat16).cuda()
    x = wl.normal((16, 4096), seed=6, dtype=torch.bfloat16).cuda()
    wq, s, b = qb.qmm_quantize(w, 64, 4)
    qb.qmm_set_path("gemm")
    y0 = qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4)
    for _ in range(5):
        y1 = qb.qmm_quantized_matmul(x, wq, s, b, True, 64, 4)
        assert torch.equal(y0, y1)


def test_gemm_stream_k_workspace_options():
    """Without a workspace (or with one too small) the call keeps whole tiles;
    both agree with the oracle, and a used workspace is left zeroed."""
    w = wl.with_outliers((1024, 4096), seed=7, dtype=torch.bfloat16)
    x = wl.normal((16, 4096), seed=8, dtype=torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 4)
    ref = oracle.quantized_matmul(x, wq, s, b, True, 64, 4)
    qb.qmm_set_path("gemm")  # (the automatic path sends 16 rows of 4-bit codes to the decode kernel)
    need = qb.qmm_quantized_matmul_workspace_size(16, 4096, 1024, True, 4, torch.bfloat16)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    small = torch.zeros(need // 2, dtype=torch.uint8, device="cuda")
    args = (x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, 4)
    for workspace in (None, small, ws):
        y = qb.qmm_quantized_matmul(*args, workspace=workspace)
        torch.cuda.synchronize()
        assert row_rel_err(y, ref) <= REL_TOL[s.dtype]
    assert int(ws[:4096].count_nonzero()) == 0  # the flags are cleared again


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("m,k,n", [(1, 4096, 1024), (16, 2048, 640), (40, 1024, 384)])
def test_gemm_stream_k_kn_layout(bits, m, k, n):
    """Stream-K with the weight stored [K, N] (groups along N): several parts
    per tile (eight for 4096 x 1024) combined by the owner."""
    w = wl.with_outliers((k, n), seed=n + k + bits + 1, dtype=torch.bfloat16)
    x = wl.normal((m, k), seed=m + k + 2, dtype=torch.bfloat16)
    run_case(x, w, 64, bits, False, "gemm")
