"""Python side of the CPU oracle (TEST INFRASTRUCTURE ONLY).

Tensors are CPU ``torch`` tensors; packed words are stored as ``torch.int32``
holding the uint32 bit patterns.  Quantize and dequantize run in the C half
(``qmm_oracle.c``); the products are a float64 matmul (library primitive) on
the dequantized weight (dequantize first, then an ordinary dense product),
which is how the mlx-rs tests ``test_quantized_matmul`` and ``test_gather_qmm`` define
the expected result of ``quantized_matmul`` and ``gather_qmm``.
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import build as _build

DTYPE_TAG = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(str(_build.build()))
        i64, i32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.oracle_quantize.argtypes = [vp, i32, i64, i64, i32, i32, vp, vp, vp]
        lib.oracle_dequantize.argtypes = [vp, vp, vp, i32, i64, i64, i32, i32, vp, vp]
        lib.oracle_unpack_codes.argtypes = [vp, i64, i64, i32, vp]
        lib.oracle_round_to_dtype.argtypes = [vp, i32, i64, vp]
        for f in (lib.oracle_quantize, lib.oracle_dequantize, lib.oracle_unpack_codes,
                  lib.oracle_round_to_dtype):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _cpu(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu", "the oracle runs on CPU tensors only"
    return t.contiguous()


def quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4):
    """Group-wise affine quantization along the last axis of a rank>=2 tensor.

    EMLX.Quantization, section ``quantize`` (rank 2 or higher, last axis);
    mlx-rs ops/quantization.rs, ``quantize`` (returns ``(wq, scales, biases)``);
    Emily.QuantizedWeight, section Layout (shapes and dtypes).
    Returns ``wq`` (int32 holding uint32 words, last axis ``cols*bits/32``),
    ``scales`` and ``biases`` (dtype of ``w``, last axis ``cols/group_size``).
    """
    w = _cpu(w)
    if w.dim() < 2:
        raise ValueError("quantize needs a tensor of rank 2 or higher")
    if w.dtype not in DTYPE_TAG:
        raise ValueError(f"unsupported dtype {w.dtype}")
    cols = w.shape[-1]
    rows = w.numel() // cols if cols else 0
    lead = tuple(w.shape[:-1])
    if bits not in (2, 4, 8) or group_size not in (32, 64, 128) or cols % group_size:
        raise ValueError("bits must be 2/4/8, group_size 32/64/128 dividing the last axis")
    wq = torch.empty(lead + (cols * bits // 32,), dtype=torch.int32)
    scales = torch.empty(lead + (cols // group_size,), dtype=w.dtype)
    biases = torch.empty_like(scales)
    rc = _load().oracle_quantize(_ptr(w), DTYPE_TAG[w.dtype], rows, cols, group_size,
                                 bits, _ptr(wq), _ptr(scales), _ptr(biases))
    if rc:
        raise ValueError("oracle_quantize rejected its arguments")
    return wq, scales, biases


def _deq(wq, scales, biases, group_size, bits, want_f32: bool):
    wq, scales, biases = _cpu(wq), _cpu(scales), _cpu(biases)
    cols = wq.shape[-1] * 32 // bits
    rows = wq.numel() // wq.shape[-1] if wq.shape[-1] else 0
    lead = tuple(wq.shape[:-1])
    if scales.shape != lead + (cols // group_size,) or biases.shape != scales.shape:
        raise ValueError("scales/biases shape does not match the packed weight")
    if want_f32:
        out = torch.empty(lead + (cols,), dtype=torch.float32)
        args = (ctypes.c_void_p(0), _ptr(out))
    else:
        out = torch.empty(lead + (cols,), dtype=scales.dtype)
        args = (_ptr(out), ctypes.c_void_p(0))
    rc = _load().oracle_dequantize(_ptr(wq), _ptr(scales), _ptr(biases),
                                   DTYPE_TAG[scales.dtype], rows, cols, group_size,
                                   bits, *args)
    if rc:
        raise ValueError("oracle_dequantize rejected its arguments")
    return out


def dequantize(wq, scales, biases, group_size: int = 64, bits: int = 4):
    """``w = scale * q + bias`` per element, rounded to the scales dtype.

    mlx-rs ops/quantization.rs, ``dequantize``; EMLX.Quantization, section
    ``dequantize`` (same logical shape as the dense tensor); output dtype is the
    scales dtype (EMLX.Quantization, section ``quantized_matmul``).
    """
    return _deq(wq, scales, biases, group_size, bits, want_f32=False)


def dequantize_f32(wq, scales, biases, group_size: int = 64, bits: int = 4):
    """The fp32 value ``fmaf(scale, q, bias)`` before rounding to the dtype."""
    return _deq(wq, scales, biases, group_size, bits, want_f32=True)


def unpack_codes(wq: torch.Tensor, bits: int) -> torch.Tensor:
    """The integer codes ``q`` (uint8) of a packed weight."""
    wq = _cpu(wq)
    cols = wq.shape[-1] * 32 // bits
    rows = wq.numel() // wq.shape[-1] if wq.shape[-1] else 0
    q = torch.empty(tuple(wq.shape[:-1]) + (cols,), dtype=torch.uint8)
    if _load().oracle_unpack_codes(_ptr(wq), rows, cols, bits, _ptr(q)):
        raise ValueError("oracle_unpack_codes rejected its arguments")
    return q


def round_to_dtype(t: torch.Tensor, dtype) -> torch.Tensor:
    """fp32 values rounded to nearest-even in ``dtype`` by the oracle's own
    conversion (the one quantize uses to store scales and biases)."""
    t = _cpu(t.to(torch.float32))
    out = torch.empty(t.shape, dtype=dtype)
    if _load().oracle_round_to_dtype(_ptr(t), DTYPE_TAG[dtype], t.numel(), _ptr(out)):
        raise ValueError("unsupported dtype")
    return out


def quantized_matmul(x, wq, scales, biases, transpose: bool = True,
                     group_size: int = 64, bits: int = 4) -> torch.Tensor:
    """float64 ``x @ W.T`` (transpose=True, W stored [out, in]) or ``x @ W``
    (transpose=False, W stored [in, out]) with W the dequantized weight.

    mlx-rs ops/quantization.rs, ``quantized_matmul``; Emily.Quantization.Layers,
    ``quantized_dense`` (the two layouts).  The weight enters as the fp32 value
    ``fmaf(scale, q, bias)``; products and sums are float64.
    """
    w = dequantize_f32(wq, scales, biases, group_size, bits).double()
    w = w.transpose(-1, -2) if transpose else w
    return _cpu(x).double() @ w


def gather_qmm(x, wq, scales, biases, lhs_indices=None, rhs_indices=None,
               transpose: bool = True, group_size: int = 64, bits: int = 4):
    """Mixture-of-experts quantized matmul, one batch entry at a time.

    EMLX.Quantization, section ``gather_quantized_matmul``; mlx-rs
    ops/quantization.rs, ``gather_qmm``.  ``x`` is [x_batch, M, K]; the packed
    weight stacks experts on its leading axis, [E, N, K*bits/32] (transpose) or
    [E, K, N*bits/32].  Batch entry b multiplies x[lhs[b]] (x[b], or x[0] when
    x_batch == 1, if lhs is None) by expert rhs[b] (expert b, or 0 when E == 1,
    if rhs is None).  Returns float64 [batch, M, N].
    """
    x = _cpu(x)
    if x.dim() != 3 or wq.dim() != 3:
        raise ValueError("x must be [x_batch, M, K] and wq [E, rows, words]")
    x_batch, n_exp = x.shape[0], wq.shape[0]
    sizes = [t.numel() for t in (lhs_indices, rhs_indices) if t is not None]
    if lhs_indices is None:
        sizes.append(x_batch)
    if rhs_indices is None:
        sizes.append(n_exp)
    batch = max(sizes)
    if any(n not in (1, batch) for n in sizes):
        raise ValueError("batch sizes do not broadcast")
    out = None
    cache = {}
    for b in range(batch):
        if lhs_indices is not None:
            xi = int(lhs_indices.reshape(-1)[b % lhs_indices.numel()])
        else:
            xi = 0 if x_batch == 1 else b
        if rhs_indices is not None:
            ei = int(rhs_indices.reshape(-1)[b % rhs_indices.numel()])
        else:
            ei = 0 if n_exp == 1 else b
        if ei not in cache:
            w = dequantize_f32(wq[ei], scales[ei], biases[ei], group_size, bits).double()
            cache[ei] = w.transpose(0, 1) if transpose else w
        yb = x[xi].double() @ cache[ei]
        if out is None:
            out = torch.empty((batch,) + tuple(yb.shape), dtype=torch.float64)
        out[b] = yb
    return out
