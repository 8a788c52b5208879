"""The failure path of the bounded waits, made to run out on purpose in the
allowed form: a flag that nothing sets, a short wait limit, and an error status
that the host reads, after which the context stays usable.

The stream-K split of the tensor-core product leaves tile parts in the
caller's workspace and raises a ready flag per part; the tile's owner waits
(bounded) for those flags.  With QMM_FAULT_STREAMK_NO_PUBLISH the parts are
written but their flags never raised, so every owner's wait runs out.
"""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _restore():
    yield
    qb.qmm_inject_fault("none")
    qb.qmm_set_wait_limit_ns(0)
    qb.qmm_set_path("auto")


def test_streamk_owner_wait_runs_out_then_recovers():
    m, k, n = 16, 4096, 1024          # 8 tiles, each split over 8 CTAs
    w = wl.with_outliers((n, k), seed=31, dtype=torch.bfloat16)
    x = wl.normal((m, k), seed=32, dtype=torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 4)
    ref = oracle.quantized_matmul(x, wq, s, b, True, 64, 4)
    args = (x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, 4)
    qb.qmm_set_path("gemm")
    need = qb.qmm_quantized_matmul_workspace_size(m, k, n, True, 4, torch.bfloat16)
    assert need > 0
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    qb.qmm_device_status()            # start from a clear error word

    qb.qmm_set_wait_limit_ns(100_000)  # 0.1 ms
    qb.qmm_inject_fault("streamk_no_publish")
    qb.qmm_quantized_matmul(*args, workspace=ws)
    with pytest.raises(qb.QmmError) as e:
        qb.qmm_device_status()        # synchronises, reads and clears the word
    assert e.value.status == 4        # QMM_ERR_TIMEOUT
    qb.qmm_device_status()            # the word was cleared

    # Recovery: no injection, default limit, the workspace zeroed again as the
    # header asks after a timeout.  The next call is correct and leaves its
    # flags cleared.
    qb.qmm_inject_fault("none")
    qb.qmm_set_wait_limit_ns(0)
    ws.zero_()
    y = qb.qmm_quantized_matmul(*args, workspace=ws)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]
    assert int(ws[:4096].count_nonzero()) == 0


def test_short_wait_limit_alone_changes_nothing():
    """A short limit with nothing injected: owners find their flags raised,
    the waits that complete in time complete, and results are right."""
    m, k, n = 16, 2048, 640
    w = wl.with_outliers((n, k), seed=33, dtype=torch.bfloat16)
    x = wl.normal((m, k), seed=34, dtype=torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 4)
    ref = oracle.quantized_matmul(x, wq, s, b, True, 64, 4)
    qb.qmm_set_path("gemm")
    qb.qmm_device_status()
    qb.qmm_set_wait_limit_ns(50_000_000)  # 50 ms: far above any wait here
    y = qb.qmm_quantized_matmul(x.cuda(), wq.cuda(), s.cuda(), b.cuda(), True, 64, 4)
    qb.qmm_device_status()
    assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]
