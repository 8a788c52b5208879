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
        lib.oracle_quantize_mx.argtypes = [vp, i32, i64, i64, i32, vp, vp]
        lib.oracle_dequantize_mx.argtypes = [vp, vp, i32, i64, i64, i32, vp, vp]
        lib.oracle_encode_elements.argtypes = [i32, vp, i64, vp]
        for f in (lib.oracle_quantize, lib.oracle_dequantize, lib.oracle_unpack_codes,
                  lib.oracle_round_to_dtype, lib.oracle_quantize_mx, lib.oracle_dequantize_mx,
                  lib.oracle_encode_elements):
            f.restype = ctypes.c_int
        _lib = lib
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _cpu(t: torch.Tensor) -> torch.Tensor:
    assert t.device.type == "cpu", "the oracle runs on CPU tensors only"
    return t.contiguous()


# Microscaled modes (Emily.QuantizedWeight, section Microscaled modes): their
# fixed (group_size, bits), and the oracle's own tags for them.
MX_MODES = {"mxfp4": (32, 4, 1), "mxfp8": (32, 8, 2), "nvfp4": (16, 4, 3)}


def _mx_mode(mode, group_size, bits):
    if mode not in MX_MODES:
        raise ValueError(f"unknown mode {mode!r}")
    gs, b, tag = MX_MODES[mode]
    if group_size != gs or bits != b:
        raise ValueError(f"mode {mode} needs group_size={gs} and bits={b}")
    return tag


def quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4, mode: str = "affine"):
    """Group-wise quantization along the last axis of a rank>=2 tensor.

    ``mode`` "affine" (below), or a microscaled mode ("mxfp4", "mxfp8",
    "nvfp4"), which returns ``(wq, scales, None)`` with one scale byte per group
    (Emily.QuantizedWeight, section Microscaled modes; the rule is in
    ``qmm_oracle.c``).
    """
    if mode != "affine":
        return _quantize_mx(w, group_size, bits, mode)
    return _quantize_affine(w, group_size, bits)


def _quantize_mx(w, group_size, bits, mode):
    tag = _mx_mode(mode, group_size, bits)
    w = _cpu(w)
    if w.dim() < 2 or w.dtype not in DTYPE_TAG:
        raise ValueError("quantize needs a float tensor of rank 2 or higher")
    cols = w.shape[-1]
    if cols % group_size:
        raise ValueError("the last axis must be a multiple of the group size")
    rows = w.numel() // cols
    lead = tuple(w.shape[:-1])
    wq = torch.empty(lead + (cols * bits // 32,), dtype=torch.int32)
    scales = torch.empty(lead + (cols // group_size,), dtype=torch.uint8)
    if _load().oracle_quantize_mx(_ptr(w), DTYPE_TAG[w.dtype], rows, cols, tag, _ptr(wq),
                                  _ptr(scales)):
        raise ValueError("oracle_quantize_mx rejected its arguments")
    return wq, scales, None


def _deq_mx(wq, scales, group_size, bits, mode, dtype, want_f32):
    tag = _mx_mode(mode, group_size, bits)
    wq, scales = _cpu(wq), _cpu(scales)
    cols = wq.shape[-1] * 32 // bits
    rows = wq.numel() // wq.shape[-1]
    lead = tuple(wq.shape[:-1])
    if scales.dtype != torch.uint8 or scales.shape != lead + (cols // group_size,):
        raise ValueError("microscaled scales are uint8 [..., cols / group_size]")
    out = torch.empty(lead + (cols,), dtype=torch.float32 if want_f32 else dtype)
    args = (ctypes.c_void_p(0), _ptr(out)) if want_f32 else (_ptr(out), ctypes.c_void_p(0))
    if _load().oracle_dequantize_mx(_ptr(wq), _ptr(scales), DTYPE_TAG[dtype], rows, cols, tag,
                                    *args):
        raise ValueError("oracle_dequantize_mx rejected its arguments")
    return out


def encode_elements(values: torch.Tensor, mode: str) -> torch.Tensor:
    """Element codes (uint8) of fp32 values in a microscaled mode's element
    format: E2M1 for mxfp4/nvfp4, E4M3 for mxfp8 (nearest-even, saturating)."""
    gs, bits, tag = MX_MODES[mode]
    v = _cpu(values.to(torch.float32)).reshape(-1)
    out = torch.empty(v.numel(), dtype=torch.uint8)
    _load().oracle_encode_elements(tag, _ptr(v), v.numel(), _ptr(out))
    return out.reshape(values.shape)


def _quantize_affine(w: torch.Tensor, group_size: int = 64, bits: int = 4):
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
    if bits not in (2, 3, 4, 6, 8) or group_size not in (32, 64, 128) or cols % group_size:
        raise ValueError("bits must be 2/3/4/6/8, group_size 32/64/128 dividing the last axis")
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


def dequantize(wq, scales, biases, group_size: int = 64, bits: int = 4, mode: str = "affine",
               dtype=torch.bfloat16):
    """``w = scale * q + bias`` per element, rounded to the scales dtype.

    Microscaled modes: ``w = X * element`` (no bias), rounded to ``dtype``.

    mlx-rs ops/quantization.rs, ``dequantize``; EMLX.Quantization, section
    ``dequantize`` (same logical shape as the dense tensor); output dtype is the
    scales dtype (EMLX.Quantization, section ``quantized_matmul``).
    """
    if mode != "affine":
        return _deq_mx(wq, scales, group_size, bits, mode, dtype, want_f32=False)
    return _deq(wq, scales, biases, group_size, bits, want_f32=False)


def dequantize_f32(wq, scales, biases, group_size: int = 64, bits: int = 4, mode: str = "affine"):
    """The fp32 value ``fmaf(scale, q, bias)`` (microscaled: ``X * element``,
    exact) before rounding to the dtype."""
    if mode != "affine":
        return _deq_mx(wq, scales, group_size, bits, mode, torch.float32, want_f32=True)
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
                     group_size: int = 64, bits: int = 4, mode: str = "affine") -> torch.Tensor:
    """float64 ``x @ W.T`` (transpose=True, W stored [out, in]) or ``x @ W``
    (transpose=False, W stored [in, out]) with W the dequantized weight.

    mlx-rs ops/quantization.rs, ``quantized_matmul``; Emily.Quantization.Layers,
    ``quantized_dense`` (the two layouts).  The weight enters as the fp32 value
    ``fmaf(scale, q, bias)`` (microscaled modes: ``X * element``); products and
    sums are float64.
    """
    w = dequantize_f32(wq, scales, biases, group_size, bits, mode).double()
    w = w.transpose(-1, -2) if transpose else w
    return _cpu(x).double() @ w


def quantized_dense(x, wq, scales, biases, bias=0, transpose: bool = True,
                    group_size: int = 64, bits: int = 4) -> torch.Tensor:
    """float64 ``x @ W (+ bias)``: the dense layer on a quantized weight.

    Emily.Quantization.Layers, ``quantized_dense``: the layer computes the
    quantized product in the weight's layout and adds a bias that is either a
    tensor or a number (0 when absent).  Read here as: a tensor holds one value
    per output feature and is broadcast over the rows of ``x``; a number is
    added to every output.  The sum is taken in float64, before any rounding to
    the output dtype (the bias is part of the fused product, not a second
    rounded step).
    """
    y = quantized_matmul(x, wq, scales, biases, transpose, group_size, bits)
    if isinstance(bias, torch.Tensor):
        return y + _cpu(bias).double().reshape(-1)
    return y + float(bias)


def qqmm(x, w, w_scales=None, group_size: int = 16, bits: int = 4, mode: str = "nvfp4"):
    """float64 product with both operands quantized: ``Q(x) @ Q(W).T``.

    mlx-rs ops/quantization.rs, ``qqmm``: ``x`` is quantized on the fly and
    ``w`` is already quantized (``w`` packed, ``w_scales`` given) or is dense
    (``w_scales`` None: quantized here); modes "nvfp4" (16, 4) and "mxfp8"
    (32, 8).  Read as: W is stored [N, K] (the call has no transpose
    argument), x is quantized along its last axis by the same rule as a
    weight, no per-tensor global scales (the mlx-rs call passes empty ones),
    and the product of the dequantized operands is taken in float64.
    """
    if mode not in ("nvfp4", "mxfp8"):
        raise ValueError("qqmm supports modes nvfp4 and mxfp8")
    _mx_mode(mode, group_size, bits)
    x = _cpu(x)
    if w_scales is None:
        wq, ws, _ = quantize(w, group_size, bits, mode)
    else:
        wq, ws = w, w_scales
    xq, xs, _ = quantize(x, group_size, bits, mode)
    xd = dequantize_f32(xq, xs, None, group_size, bits, mode).double()
    wd = dequantize_f32(wq, ws, None, group_size, bits, mode).double()
    return xd @ wd.transpose(-1, -2)


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
