"""The allocation-free gather entry point (qmm_gather_qmm_static), through the
C ABI, against the workspace entry point on the same inputs.  Collected last
so that it also runs after every other GPU test in the session."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(n_exp=8, n=384, k=512, batch=200, seed=7):
    w = wl.normal((n_exp, n, k), seed, 0.02, torch.bfloat16)
    wq, s, b = oracle.quantize(w, 64, 4)
    x = wl.normal((batch, 1, k), seed + 1, 1.0, torch.bfloat16)
    rhs = wl.zipf_experts(batch, n_exp, 1.2, seed + 2)
    return x.cuda(), wq.cuda(), s.cuda(), b.cuda(), rhs.cuda()


def test_static_scratch_matches_workspace_entry_twice():
    x, wq, s, b, rhs = _inputs()
    ref = qb.qmm_gather_qmm(x, wq, s, b, None, rhs, True, 64, 4)
    for _ in range(2):  # two calls in a row reuse the one scratch
        y = qb.qmm_gather_qmm_static(x, wq, s, b, None, rhs, True, 64, 4)
        qb.qmm_device_status()
        assert row_rel_err(y, ref) <= REL_TOL[torch.bfloat16]


def test_static_scratch_rejects_calls_beyond_its_size():
    k, batch = 4096, 2048  # 2048 sorted rows x 4096 x 2 bytes > 8 MiB
    need = qb.qmm_gather_qmm_workspace_size(batch, 1, k, 2, torch.bfloat16)
    assert need > 8 << 20
    x = torch.zeros((batch, 1, k), dtype=torch.bfloat16, device="cuda")
    wq = torch.zeros((2, 128, k // 8), dtype=torch.int32, device="cuda")
    s = torch.zeros((2, 128, k // 64), dtype=torch.bfloat16, device="cuda")
    rhs = torch.zeros(batch, dtype=torch.int32, device="cuda")
    with pytest.raises(qb.QmmError, match="QMM_ERR_WORKSPACE"):
        qb.qmm_gather_qmm_static(x, wq, s, s.clone(), None, rhs, True, 64, 4)
