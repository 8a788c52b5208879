"""GPU parity: gather_qmm against the oracle's per-entry dequantize-then-float64
products, on the tensor-core grouped path and on the SIMT batched path."""
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


def experts(n_exp, rows, cols, seed, dtype, gs, bits):
    """Stacked experts [n_exp, rows, cols] quantized by the oracle."""
    w = wl.with_outliers((n_exp, rows, cols), seed, 0.02, 0.01, 20.0, dtype)
    return oracle.quantize(w, gs, bits)


def run_gather(x, packed, lhs, rhs, gs, bits, transpose=True, path="auto", sorted_indices=False):
    wq, s, b = packed
    ref = oracle.gather_qmm(x, wq, s, b, lhs, rhs, transpose, gs, bits)
    qb.qmm_set_path(path)
    cu = (lambda t: None if t is None else t.cuda())
    y = qb.qmm_gather_qmm(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), cu(lhs), cu(rhs), transpose,
                          gs, bits, sorted_indices=sorted_indices)
    qb.qmm_device_status()
    assert y.shape == ref.shape and y.dtype == s.dtype
    err = row_rel_err(y, ref)
    assert err <= REL_TOL[s.dtype], f"rel err {err}"
    return y, ref


def test_mlx_rs_gather_qmm_cases():
    """mlx-rs unit test test_gather_qmm: m=32, n=k=64, 3 experts, gs 64, 4 bits,
    f32; lhs [0] broadcast against rhs [2, 1] with x_batch 1, then lhs [0, 2]
    with x_batch 5; within rtol = atol = 1e-4 of gather_mm on the dequantized
    weight."""
    m, n, k = 32, 64, 64
    packed = oracle.quantize(wl.normal((3, n, k), 11, 1.0, torch.float32), 64, 4)
    for x_batch, lhs, rhs in ((1, [0], [2, 1]), (5, [0, 2], [2, 1])):
        x = wl.normal((x_batch, m, k), 12 + x_batch, 1.0, torch.float32)
        y, ref = run_gather(x, packed, torch.tensor(lhs, dtype=torch.int32),
                            torch.tensor(rhs, dtype=torch.int32), 64, 4)
        assert torch.allclose(y.cpu().double(), ref, rtol=1e-4, atol=1e-4)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("bits,gs", [(4, 64), (2, 32), (8, 128), (4, 128)])
def test_grouped_unsorted_zipf(dtype, bits, gs):
    # Ragged N (not a multiple of the 128-row tile) so a tile of one expert
    # reads rows of the next; several k-blocks.
    n_exp, n, k, batch = 8, 200, 512, 96
    packed = experts(n_exp, n, k, 21 + bits, dtype, gs, bits)
    x = wl.normal((batch, 1, k), 22, 1.0, dtype)
    rhs = wl.zipf_experts(batch, n_exp, 1.2, 23)
    run_gather(x, packed, None, rhs, gs, bits, path="gemm")


def test_grouped_sorted_rows_read_x_directly():
    n_exp, n, k, batch = 4, 256, 256, 50
    packed = experts(n_exp, n, k, 31, torch.bfloat16, 64, 4)
    x = wl.normal((batch, 1, k), 32, 1.0, torch.bfloat16)
    rhs = torch.sort(wl.zipf_experts(batch, n_exp, 1.2, 33)).values
    run_gather(x, packed, None, rhs, 64, 4, path="gemm", sorted_indices=True)
    # A wrong hint must not change the result.
    rhs_unsorted = wl.zipf_experts(batch, n_exp, 1.2, 34)
    run_gather(x, packed, None, rhs_unsorted, 64, 4, path="gemm", sorted_indices=True)


def test_grouped_lhs_indices_and_rows_per_entry():
    n_exp, n, k = 5, 384, 256
    packed = experts(n_exp, n, k, 41, torch.bfloat16, 64, 4)
    x = wl.normal((7, 3, k), 42, 1.0, torch.bfloat16)  # M = 3 rows per entry
    g = torch.Generator().manual_seed(43)
    lhs = torch.randint(0, 7, (40,), generator=g, dtype=torch.int32)
    rhs = torch.randint(0, n_exp, (40,), generator=g, dtype=torch.int32)
    run_gather(x, packed, lhs, rhs, 64, 4, path="gemm")


def test_grouped_broadcast_forms():
    n_exp, n, k = 3, 128, 128
    packed = experts(n_exp, n, k, 51, torch.bfloat16, 64, 4)
    # x_batch 1 shared by every entry, rhs picks the experts.
    x1 = wl.normal((1, 2, k), 52, 1.0, torch.bfloat16)
    run_gather(x1, packed, None, torch.tensor([2, 0, 1, 1], dtype=torch.int32), 64, 4, path="gemm")
    # No indices at all: entry b uses x[b] and expert b.
    x3 = wl.normal((3, 5, k), 53, 1.0, torch.bfloat16)
    run_gather(x3, packed, None, None, 64, 4, path="gemm")


def test_grouped_expert_larger_than_one_chunk():
    # 600 rows, most on expert 0: its rows span several 256-row chunks.
    n_exp, n, k, batch = 2, 256, 256, 600
    packed = experts(n_exp, n, k, 61, torch.bfloat16, 64, 4)
    x = wl.normal((batch, 1, k), 62, 1.0, torch.bfloat16)
    rhs = (torch.rand(batch, generator=torch.Generator().manual_seed(63)) < 0.15).to(torch.int32)
    run_gather(x, packed, None, rhs, 64, 4, path="gemm")


@pytest.mark.parametrize("batch", [1, 2, 63, 64, 65, 129, 257])
def test_grouped_tile_widths(batch):
    # Row totals on both sides of the 64 / 128 / 256-row tile widths.
    n_exp, n, k = 3, 128, 192
    packed = experts(n_exp, n, k, 71, torch.bfloat16, 64, 4)
    x = wl.normal((batch, 1, k), 72 + batch, 1.0, torch.bfloat16)
    rhs = torch.randint(0, n_exp, (batch,), generator=torch.Generator().manual_seed(73 + batch),
                        dtype=torch.int32)
    run_gather(x, packed, None, rhs, 64, 4, path="gemm")


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("transpose", [True, False])
def test_simt_batched_path(dtype, transpose):
    n_exp, rows, cols = 4, 192, 256  # stored [rows, cols] per expert
    packed = experts(n_exp, rows, cols, 81, dtype, 64, 4)
    k = cols if transpose else rows
    x = wl.normal((6, 2, k), 82, 1.0, dtype)
    g = torch.Generator().manual_seed(83)
    lhs = torch.randint(0, 6, (9,), generator=g, dtype=torch.int32)
    rhs = torch.randint(0, n_exp, (9,), generator=g, dtype=torch.int32)
    run_gather(x, packed, lhs, rhs, 64, 4, transpose, path="gemv")


@pytest.mark.parametrize("path", ["gemm", "gemv"])
def test_out_of_range_indices_zero_rows_and_report(path):
    n_exp, n, k = 3, 128, 128
    wq, s, b = experts(n_exp, n, k, 91, torch.bfloat16, 64, 4)
    x = wl.normal((4, 1, k), 92, 1.0, torch.bfloat16)
    rhs = torch.tensor([0, 3, 2, -1, 1, 2], dtype=torch.int32)  # 3 and -1 out of range
    lhs = torch.tensor([0, 1, 4, 2, 3, 3], dtype=torch.int32)   # 4 out of range
    qb.qmm_set_path(path)
    qb.qmm_device_status()  # clear anything earlier
    y = qb.qmm_gather_qmm(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), lhs.cuda(), rhs.cuda(), True,
                          64, 4)
    with pytest.raises(qb.QmmError, match="QMM_ERR_INDEX"):
        qb.qmm_device_status()
    y = y.cpu()
    bad = [1, 2, 3]
    assert torch.all(y[bad] == 0)
    good = [0, 4, 5]
    ref = oracle.gather_qmm(x, wq, s, b, lhs[good], rhs[good], True, 64, 4)
    assert row_rel_err(y[good], ref) <= REL_TOL[torch.bfloat16]


def test_empty_batch_is_noop():
    wq, s, b = experts(2, 128, 128, 95, torch.bfloat16, 64, 4)
    x = wl.normal((1, 1, 128), 96, 1.0, torch.bfloat16).cuda()
    y = qb.qmm_gather_qmm(x, wq.cuda(), s.cuda(), b.cuda(), None,
                          torch.empty(0, dtype=torch.int32, device="cuda"), True, 64, 4)
    assert y.shape == (0, 1, 128)


def test_workspace_too_small_is_rejected():
    wq, s, b = experts(2, 128, 128, 97, torch.bfloat16, 64, 4)
    x = wl.normal((8, 1, 128), 98, 1.0, torch.bfloat16).cuda()
    rhs = torch.zeros(8, dtype=torch.int32, device="cuda")
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(qb.QmmError, match="QMM_ERR_WORKSPACE"):
        qb.qmm_gather_qmm(x, wq.cuda(), s.cuda(), b.cuda(), None, rhs, True, 64, 4, workspace=ws)


@pytest.mark.slow
def test_moe_full_size_sampled():
    """8 experts W [8, 14336, 4096] int4 gs 64, x [512, 1, 4096], rhs Zipf(1.2):
    checked on 64 sampled entries over three 256-feature output slices."""
    c = wl.moe_case()
    wq, s, b = oracle.quantize(c.w, c.group_size, c.bits)
    del c.w
    y = qb.qmm_gather_qmm(c.x.cuda(), wq.cuda(), s.cuda(), b.cuda(), None, c.rhs_indices.cuda(),
                          True, c.group_size, c.bits)
    qb.qmm_device_status()
    y = y.cpu()
    ent = torch.randperm(512, generator=torch.Generator().manual_seed(5))[:64]
    for lo in (0, 7040, 14336 - 256):
        sl = slice(lo, lo + 256)
        ref = oracle.gather_qmm(c.x[ent], wq[:, sl], s[:, sl], b[:, sl], None,
                                c.rhs_indices[ent], True, c.group_size, c.bits)
        err = row_rel_err(y[ent][:, :, sl], ref)
        assert err <= REL_TOL[torch.bfloat16], f"rel err {err} at features {lo}.."
