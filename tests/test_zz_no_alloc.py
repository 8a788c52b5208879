"""The allocation-free gather entry point (qmm_gather_qmm_static), through the
C ABI: against the oracle's per-entry products and against the workspace entry
point on the same inputs, two calls in a row (the calls share one built-in
scratch).  Collected last so that it also runs after every other GPU test in
the session."""
import pytest
import torch

import oracle
from parity import REL_TOL, row_rel_err
from quantized_matmul_03_b200 import binding as qb
from quantized_matmul_03_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _inputs(dtype=torch.bfloat16, n_exp=8, n=384, k=512, batch=200, seed=7, sort=False):
    w = wl.normal((n_exp, n, k), seed, 0.02, dtype)
    wq, s, b = oracle.quantize(w, 64, 4)
    x = wl.normal((batch, 1, k), seed + 1, 1.0, dtype)
    rhs = wl.zipf_experts(batch, n_exp, 1.2, seed + 2)
    if sort:
        rhs = rhs.sort().values.contiguous()
    return x, wq, s, b, rhs


@pytest.mark.parametrize("case", ["unsorted_bf16", "sorted_bf16", "f32", "kn_layout_bf16"])
def test_static_scratch_matches_oracle_and_workspace_entry_twice(case):
    """Unsorted Zipf indices (rows copied into sorted order in the scratch),
    already-sorted indices (the copy is skipped and x read in place), an f32
    call and a weight stored [K, N] (both on the SIMT path, which uses no
    scratch)."""
    dtype = torch.float32 if case == "f32" else torch.bfloat16
    transpose = case != "kn_layout_bf16"
    x, wq, s, b, rhs = _inputs(dtype=dtype, sort=case == "sorted_bf16")
    if not transpose:  # experts stored [K, N]: quantize along N
        w = wl.normal((8, 512, 384), 17, 0.02, dtype)
        wq, s, b = oracle.quantize(w, 64, 4)
    ref = oracle.gather_qmm(x, wq, s, b, None, rhs, transpose, 64, 4)
    cu = [t.cuda() for t in (x, wq, s, b, rhs)]
    y_ws = qb.qmm_gather_qmm(cu[0], cu[1], cu[2], cu[3], None, cu[4], transpose, 64, 4)
    for _ in range(2):  # two calls in a row reuse the one scratch
        y = qb.qmm_gather_qmm_static(cu[0], cu[1], cu[2], cu[3], None, cu[4], transpose, 64, 4)
        qb.qmm_device_status()
        assert row_rel_err(y, ref) <= REL_TOL[dtype]
        assert row_rel_err(y, y_ws) <= REL_TOL[dtype]


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
    # The same sizes on the SIMT path use no scratch and are accepted.
    qb.qmm_set_path("gemv")
    try:
        y = qb.qmm_gather_qmm_static(x, wq, s, s.clone(), None, rhs, True, 64, 4)
        qb.qmm_device_status()
        assert int(y.count_nonzero()) == 0
    finally:
        qb.qmm_set_path("auto")
