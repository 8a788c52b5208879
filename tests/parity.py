"""Shared parity helpers for the GPU tests (no method arithmetic here)."""
import torch

# Matmul tolerances against the oracle's dequantize-then-float64 product:
# max over rows of  max_j |y - r| / max_j |r|.
REL_TOL = {torch.bfloat16: 2e-2, torch.float16: 2e-2, torch.float32: 1e-5}


def row_rel_err(y: torch.Tensor, ref: torch.Tensor) -> float:
    """Max over output rows of (max abs error in the row) / (max |ref| in the row)."""
    y = y.detach().double().cpu().reshape(-1, y.shape[-1])
    r = ref.detach().double().cpu().reshape(-1, ref.shape[-1])
    if y.numel() == 0:
        return 0.0
    num = (y - r).abs().amax(dim=1)
    den = r.abs().amax(dim=1).clamp_min(1e-30)
    return float((num / den).max())


def words(t: torch.Tensor) -> torch.Tensor:
    """Packed words as int64 unsigned values (for exact comparison)."""
    return t.detach().cpu().to(torch.int64) & 0xFFFFFFFF
