"""Thin ctypes binding over libqmm's C ABI (``include/qmm.h``).

Argument marshalling only: shapes and dtypes are read off torch tensors,
outputs are allocated with torch on the input's device, and every step of the
computation runs in libqmm's CUDA kernels on torch's current stream.  There is
no fallback: if ``libqmm.so`` is missing or the tensors are not on a CUDA
device, the call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path
from typing import Optional

import torch

LIB_PATH = Path(__file__).resolve().parent / "libqmm.so"

QMM_OK = 0
STATUS_NAMES = {0: "QMM_OK", 1: "QMM_ERR_INVALID_ARG", 2: "QMM_ERR_UNSUPPORTED",
                3: "QMM_ERR_CUDA", 4: "QMM_ERR_TIMEOUT", 5: "QMM_ERR_INDEX",
                6: "QMM_ERR_WORKSPACE"}
PATHS = {"auto": 0, "gemv": 1, "gemm": 2, "decode_tc": 3}
DTYPES = {torch.float32: 0, torch.bfloat16: 1, torch.float16: 2}

_lib = None


class QmmError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load libqmm.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with quantized_matmul_03_b200.build.build() "
                "(or __graft_entry__.build()); there is no CPU fallback")
        L = ctypes.CDLL(str(LIB_PATH))
        i64, i32, vp, sz = ctypes.c_int64, ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        cp = ctypes.c_char_p
        sig = {
            "qmm_quantize": [vp, i32, i64, i64, i32, i32, cp, vp, vp, vp, vp],
            "qmm_dequantize": [vp, vp, vp, i32, i64, i64, i32, i32, cp, vp, vp],
            "qmm_quantized_matmul": [vp, i64, i64, vp, vp, vp, i32, i64, i32, i32, i32, cp,
                                     vp, vp],
            "qmm_quantized_matmul_ws": [vp, i64, i64, vp, vp, vp, i32, i64, i32, i32, i32, cp,
                                        vp, vp, sz, vp],
            "qmm_quantized_matmul_host": [vp, vp, i64, i64, vp, vp, vp, i32, i64, i32, i32, i32,
                                          cp, vp, vp, vp, sz, vp],
            "qmm_quantized_matmul_mapped": [vp, vp, i64, i64, vp, vp, vp, i32, i64, i32, i32,
                                            i32, cp, vp, vp, vp, sz, vp],
            "qmm_quantized_dense": [vp, i64, i64, vp, vp, vp, i32, i64, i32, i32, i32, cp,
                                    vp, ctypes.c_double, vp, vp, sz, vp],
            "qmm_qqmm": [vp, i64, i64, i32, vp, vp, i64, i32, i32, cp, vp, vp, sz, vp],
            "qmm_gather_qmm": [vp, i64, i64, i64, vp, vp, vp, i32, i64, i64, vp, vp, i64, i32,
                               i32, i32, cp, i32, vp, vp, sz, vp],
            "qmm_gather_qmm_static": [vp, i64, i64, i64, vp, vp, vp, i32, i64, i64, vp, vp, i64,
                                      i32, i32, i32, cp, i32, vp, vp],
            "qmm_device_status": [vp, i32],
            "qmm_set_path": [i32],
            "qmm_set_wait_limit_ns": [ctypes.c_uint64],
            "qmm_inject_fault": [i32],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.qmm_qqmm_workspace_size.argtypes = [i64, i64, i32, i32, i32]
        L.qmm_qqmm_workspace_size.restype = sz
        L.qmm_gather_qmm_workspace_size.argtypes = [i64, i64, i64, i64, i32]
        L.qmm_gather_qmm_workspace_size.restype = sz
        L.qmm_quantized_matmul_workspace_size.argtypes = [i64, i64, i64, i32, i32, i32]
        L.qmm_quantized_matmul_workspace_size.restype = sz
        L.qmm_status_string.argtypes = [i32]
        L.qmm_status_string.restype = cp
        L.qmm_last_error.argtypes = []
        L.qmm_last_error.restype = cp
        L.qmm_launch_count.argtypes = []
        L.qmm_launch_count.restype = ctypes.c_uint64
        L.qmm_version.argtypes = []
        L.qmm_version.restype = i32
        L.qmm_mapped_pointer.argtypes = [vp]
        L.qmm_mapped_pointer.restype = vp
        _lib = L
    return _lib


def _check(status: int):
    if status != QMM_OK:
        raise QmmError(status, (lib().qmm_last_error() or b"").decode())


def _p(t: Optional[torch.Tensor]):
    # A plain int (or None for NULL): ctypes converts it for c_void_p arguments.
    return t.data_ptr() if t is not None else None


def _stream(device: torch.device):
    return torch.cuda.current_stream(device).cuda_stream


def _mode(mode: Optional[str]):
    return None if mode is None else mode.encode()


def _cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("libqmm takes contiguous CUDA tensors")


def _dtype(t: torch.Tensor) -> int:
    if t.dtype not in DTYPES:
        raise ValueError(f"unsupported dtype {t.dtype}")
    return DTYPES[t.dtype]


# The microscaled modes (Emily.QuantizedWeight, section Microscaled modes):
# fixed (group_size, bits), one scale byte per group, no biases.
MX_MODES = {"mxfp4": (32, 4), "mxfp8": (32, 8), "nvfp4": (16, 4)}


def qmm_quantize(w: torch.Tensor, group_size: int = 64, bits: int = 4, mode: str = "affine",
                 out=None):
    """Quantize ``w`` (rank >= 2) along its last axis -> (wq, scales, biases).

    ``wq`` is int32 holding the uint32 words; scales/biases take ``w``'s dtype
    ("affine"); in a microscaled mode scales are uint8 and biases is None.
    ``out``: optional ``(wq, scales, biases)`` tensors to write into.
    """
    _cuda(w)
    cols = w.shape[-1]
    rows = w.numel() // cols if cols else 0
    lead = tuple(w.shape[:-1])
    micro = mode in MX_MODES
    if out is not None:
        wq, scales, biases = out
        _cuda(wq, scales, biases)
    else:
        wq = torch.empty(lead + (cols * bits // 32,), dtype=torch.int32, device=w.device)
        scales = torch.empty(lead + (max(cols // group_size, 0),),
                             dtype=torch.uint8 if micro else w.dtype, device=w.device)
        biases = None if micro else torch.empty_like(scales)
    _check(lib().qmm_quantize(_p(w), _dtype(w), rows, cols, group_size, bits, _mode(mode),
                              _p(wq), _p(scales), _p(biases), _stream(w.device)))
    return wq, scales, biases


def qmm_dequantize(wq, scales, biases, group_size: int = 64, bits: int = 4,
                   mode: str = "affine", dtype=torch.bfloat16):
    """Dense weight ``scale * q + bias`` in the scales dtype; in a microscaled
    mode ``X * element`` in ``dtype``."""
    _cuda(wq, scales, biases)
    cols = wq.shape[-1] * 32 // bits
    rows = wq.numel() // wq.shape[-1] if wq.shape[-1] else 0
    odt = dtype if mode in MX_MODES else scales.dtype
    out = torch.empty(tuple(wq.shape[:-1]) + (cols,), dtype=odt, device=wq.device)
    _check(lib().qmm_dequantize(_p(wq), _p(scales), _p(biases), _dtype(out), rows, cols,
                                group_size, bits, _mode(mode), _p(out), _stream(wq.device)))
    return out


# Zeroed stream-K workspaces, one per (device, stream), owned by this module
# (torch memory) and reused across calls; the library leaves them zeroed.
_mm_ws = {}
# Workspace sizes by call shape (they depend on the forced path too, so
# qmm_set_path clears this).
_mm_ws_size = {}


def qmm_quantized_matmul_workspace_size(M: int, K: int, N: int, transpose: bool = True,
                                        bits: int = 4, dtype=torch.bfloat16) -> int:
    key = (M, K, N, bool(transpose), bits, dtype)
    n = _mm_ws_size.get(key)
    if n is None:
        n = int(lib().qmm_quantized_matmul_workspace_size(M, K, N, int(bool(transpose)), bits,
                                                           DTYPES[dtype]))
        _mm_ws_size[key] = n
    return n


def _matmul_workspace(device: torch.device, nbytes: int) -> torch.Tensor:
    key = (device.index, torch.cuda.current_stream(device).cuda_stream)
    ws = _mm_ws.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _mm_ws[key] = ws
    return ws


def qmm_quantized_matmul(x, wq, scales, biases, transpose: bool = True, group_size: int = 64,
                         bits: int = 4, mode: str = "affine", out: Optional[torch.Tensor] = None,
                         workspace="auto"):
    """``x @ W.T`` (transpose) or ``x @ W`` with W packed; x is [..., K].

    workspace: "auto" (a zeroed workspace kept per device and stream, when the
    call can use one), None (whole tiles only) or a zeroed uint8 CUDA tensor
    of at least qmm_quantized_matmul_workspace_size(...) bytes."""
    _cuda(x, wq, scales, biases, out)
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    if transpose:
        N = wq.shape[-2]
    else:
        N = wq.shape[-1] * 32 // bits
    # (affine: the output takes the scales dtype; microscaled: the activations')
    odt = x.dtype if mode in MX_MODES else scales.dtype
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=odt, device=x.device)
    ws = None
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a tensor")
        if odt in DTYPES and mode not in MX_MODES:
            need = qmm_quantized_matmul_workspace_size(M, K, N, transpose, bits, odt)
            if need > 0:
                ws = _matmul_workspace(x.device, need)
    elif workspace is not None:
        _cuda(workspace)
        ws = workspace
    _check(lib().qmm_quantized_matmul_ws(_p(x), M, K, _p(wq), _p(scales), _p(biases),
                                         _dtype(out), N, int(bool(transpose)), group_size, bits,
                                         _mode(mode), _p(out), _p(ws),
                                         ws.numel() * ws.element_size() if ws is not None else 0,
                                         _stream(x.device)))
    return out


class HostMatmul:
    """One prepared ``qmm_quantized_matmul_host`` call: x from host memory,
    the product, y back to host memory, enqueued on the current stream of
    x_dev's device by a single C call each time the object is called.

    x_host / y_host: CPU tensors (pin_memory() for asynchronous copies) of the
    shapes of x_dev / y_dev; x_dev / y_dev: CUDA tensors.  The pointers,
    sizes, workspace and stream are fixed when the object is made, so a call
    costs one foreign-function call; when both host tensors are page-locked,
    their device mappings are looked up here once and each call goes through
    qmm_quantized_matmul_mapped.  y_host holds the result once the stream has
    run it (torch.cuda.synchronize() or an event)."""

    def __init__(self, x_host, x_dev, wq, scales, biases, y_dev, y_host, transpose: bool = True,
                 group_size: int = 64, bits: int = 4, mode: str = "affine", workspace="auto"):
        _cuda(x_dev, wq, scales, biases, y_dev)
        for h, d in ((x_host, x_dev), (y_host, y_dev)):
            if h.is_cuda or not h.is_contiguous() or h.shape != d.shape or h.dtype != d.dtype:
                raise ValueError("host buffers must be contiguous CPU tensors shaped like the device ones")
        K = x_dev.shape[-1]
        M = x_dev.numel() // K if K else 0
        N = wq.shape[-2] if transpose else wq.shape[-1] * 32 // bits
        if y_dev.shape[-1] != N or y_dev.numel() != M * N:
            raise ValueError(f"y must hold {M} x {N} values")
        ws = None
        if isinstance(workspace, str):
            if workspace != "auto":
                raise ValueError("workspace must be 'auto', None or a tensor")
            if y_dev.dtype in DTYPES and mode not in MX_MODES:
                need = qmm_quantized_matmul_workspace_size(M, K, N, transpose, bits, y_dev.dtype)
                if need > 0:
                    ws = _matmul_workspace(x_dev.device, need)
        elif workspace is not None:
            _cuda(workspace)
            ws = workspace
        # keep the tensors alive as long as the call may run
        self._keep = (x_host, x_dev, wq, scales, biases, y_dev, y_host, ws)
        xh, yh = _p(x_host), _p(y_host)
        self._fn = lib().qmm_quantized_matmul_host
        if x_host.is_pinned() and y_host.is_pinned():
            with torch.cuda.device(x_dev.device):
                xm, ym = lib().qmm_mapped_pointer(xh), lib().qmm_mapped_pointer(yh)
            if xm and ym:
                xh, yh = xm, ym
                self._fn = lib().qmm_quantized_matmul_mapped
        self._args = (xh, _p(x_dev), M, K, _p(wq), _p(scales), _p(biases),
                      _dtype(y_dev), N, int(bool(transpose)), group_size, bits, _mode(mode),
                      _p(y_dev), yh, _p(ws),
                      ws.numel() * ws.element_size() if ws is not None else 0,
                      _stream(x_dev.device))

    def __call__(self):
        st = self._fn(*self._args)
        if st != 0:
            _check(st)


def qmm_quantized_matmul_host(x_host, x_dev, wq, scales, biases, y_dev, y_host,
                              transpose: bool = True, group_size: int = 64, bits: int = 4,
                              mode: str = "affine", workspace="auto"):
    """x_host -> x_dev, ``x_dev @ W`` -> y_dev, y_dev -> y_host, enqueued on the
    current stream (one C call; see HostMatmul for the repeated form)."""
    HostMatmul(x_host, x_dev, wq, scales, biases, y_dev, y_host, transpose, group_size, bits,
               mode, workspace)()
    return y_host


def qmm_quantized_dense(x, wq, scales, biases, bias=0, transpose: bool = True,
                        group_size: int = 64, bits: int = 4, mode: str = "affine",
                        out: Optional[torch.Tensor] = None, workspace="auto"):
    """Dense layer ``x @ W (+ bias)`` on a quantized weight (Emily.Quantization.Layers,
    ``quantized_dense``): ``bias`` is a number, or a tensor of the output
    features' length in the scales dtype, or a tensor of one element (taken as
    a number).  The bias is added inside the product before rounding."""
    _cuda(x, wq, scales, biases, out)
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    N = wq.shape[-2] if transpose else wq.shape[-1] * 32 // bits
    odt = x.dtype if mode in MX_MODES else scales.dtype
    bias_t, bias_v = None, 0.0
    if isinstance(bias, torch.Tensor):
        if bias.numel() == 1:
            bias_v = float(bias.reshape(()).item())
        else:
            if bias.numel() != N or bias.dtype != odt:
                raise ValueError(f"bias must hold {N} values of dtype {odt}")
            bias_t = bias.reshape(-1)
            _cuda(bias_t)
    else:
        bias_v = float(bias)
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=odt, device=x.device)
    ws = None
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError("workspace must be 'auto', None or a tensor")
        need = 0 if mode in MX_MODES else qmm_quantized_matmul_workspace_size(
            M, K, N, transpose, bits, odt)
        if need > 0:
            ws = _matmul_workspace(x.device, need)
    elif workspace is not None:
        _cuda(workspace)
        ws = workspace
    _check(lib().qmm_quantized_dense(_p(x), M, K, _p(wq), _p(scales), _p(biases),
                                     _dtype(out), N, int(bool(transpose)), group_size, bits,
                                     _mode(mode), _p(bias_t), bias_v, _p(out), _p(ws),
                                     ws.numel() * ws.element_size() if ws is not None else 0,
                                     _stream(x.device)))
    return out


def qmm_qqmm(x, w, w_scales=None, group_size: Optional[int] = None, bits: Optional[int] = None,
             mode: str = "nvfp4", out: Optional[torch.Tensor] = None,
             workspace: Optional[torch.Tensor] = None):
    """mlx-rs ``qqmm``: ``Q(x) @ Q(W).T`` with x quantized on the fly; ``w`` is
    the packed weight with ``w_scales``, or a dense weight (quantized first
    when ``w_scales`` is None).  Modes "nvfp4" (default) and "mxfp8"; group
    size and bits default to the mode's."""
    if mode not in ("nvfp4", "mxfp8"):
        raise ValueError("qqmm supports modes nvfp4 and mxfp8")
    gs_d, bits_d = MX_MODES[mode]
    group_size = gs_d if group_size is None else group_size
    bits = bits_d if bits is None else bits
    if w_scales is None:
        w, w_scales, _ = qmm_quantize(w, group_size, bits, mode)
    _cuda(x, w, w_scales, out, workspace)
    K = x.shape[-1]
    M = x.numel() // K if K else 0
    N = w.shape[-2]
    if out is None:
        out = torch.empty(tuple(x.shape[:-1]) + (N,), dtype=x.dtype, device=x.device)
    need = int(lib().qmm_qqmm_workspace_size(M, K, group_size, bits, _dtype(x)))
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().qmm_qqmm(_p(x), M, K, _dtype(x), _p(w), _p(w_scales), N, group_size, bits,
                          _mode(mode), _p(out), _p(workspace), ws_bytes, _stream(x.device)))
    return out


def qmm_gather_qmm_workspace_size(batch: int, M: int, K: int, n_experts: int,
                                  dtype=torch.bfloat16) -> int:
    return int(lib().qmm_gather_qmm_workspace_size(batch, M, K, n_experts, DTYPES[dtype]))


def _gather_shapes(x, wq, lhs_indices, rhs_indices, transpose, bits):
    """Sizes of a gather_qmm call, and the index arrays stretched to the
    broadcast batch (the C ABI takes arrays of length batch)."""
    for t in (lhs_indices, rhs_indices):
        if t is not None and t.dtype != torch.int32:
            raise ValueError("indices must be int32")
    x_batch, M, K = x.shape
    n_experts = wq.shape[0]
    N = wq.shape[1] if transpose else wq.shape[2] * 32 // bits
    sizes = [t.numel() for t in (lhs_indices, rhs_indices) if t is not None]
    if lhs_indices is None:
        sizes.append(x_batch)
    if rhs_indices is None:
        sizes.append(n_experts)
    # Broadcast of the batch sizes (a size of 1 stretches to the other).
    others = {n for n in sizes if n != 1}
    if len(others) > 1:
        raise ValueError(f"batch sizes {sizes} do not broadcast")
    batch = others.pop() if others else 1
    if lhs_indices is not None:
        lhs_indices = lhs_indices.reshape(-1).expand(batch).contiguous()
    if rhs_indices is not None:
        rhs_indices = rhs_indices.reshape(-1).expand(batch).contiguous()
    return x_batch, M, K, n_experts, N, batch, lhs_indices, rhs_indices


def qmm_gather_qmm(x, wq, scales, biases, lhs_indices=None, rhs_indices=None,
                   transpose: bool = True, group_size: int = 64, bits: int = 4,
                   mode: str = "affine", sorted_indices: bool = False,
                   workspace: Optional[torch.Tensor] = None,
                   out: Optional[torch.Tensor] = None):
    """Mixture-of-experts quantized matmul: x [x_batch, M, K], experts stacked
    on wq's leading axis; returns y [batch, M, N]."""
    _cuda(x, wq, scales, biases, lhs_indices, rhs_indices, workspace, out)
    x_batch, M, K, n_experts, N, batch, lhs_indices, rhs_indices = _gather_shapes(
        x, wq, lhs_indices, rhs_indices, transpose, bits)
    if out is None:
        out = torch.empty((batch, M, N), dtype=scales.dtype, device=x.device)
    need = qmm_gather_qmm_workspace_size(batch, M, K, n_experts, scales.dtype)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check(lib().qmm_gather_qmm(_p(x), x_batch, M, K, _p(wq), _p(scales), _p(biases),
                                _dtype(scales), n_experts, N, _p(lhs_indices), _p(rhs_indices),
                                batch, int(bool(transpose)), group_size, bits, _mode(mode),
                                int(bool(sorted_indices)), _p(out), _p(workspace), ws_bytes,
                                _stream(x.device)))
    return out


def qmm_gather_qmm_static(x, wq, scales, biases, lhs_indices=None, rhs_indices=None,
                          transpose: bool = True, group_size: int = 64, bits: int = 4,
                          mode: str = "affine", sorted_indices: bool = False,
                          out: Optional[torch.Tensor] = None):
    """gather_qmm on the library's built-in scratch (no workspace argument).
    Calls whose work overlaps in time on one device race on that scratch."""
    _cuda(x, wq, scales, biases, lhs_indices, rhs_indices, out)
    x_batch, M, K, n_experts, N, batch, lhs_indices, rhs_indices = _gather_shapes(
        x, wq, lhs_indices, rhs_indices, transpose, bits)
    if out is None:
        out = torch.empty((batch, M, N), dtype=scales.dtype, device=x.device)
    _check(lib().qmm_gather_qmm_static(_p(x), x_batch, M, K, _p(wq), _p(scales), _p(biases),
                                       _dtype(scales), n_experts, N, _p(lhs_indices),
                                       _p(rhs_indices), batch, int(bool(transpose)), group_size,
                                       bits, _mode(mode), int(bool(sorted_indices)), _p(out),
                                       _stream(x.device)))
    return out


def qmm_device_status(reset: bool = True, device=None):
    """Synchronise the current stream and raise if a kernel recorded an error."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check(lib().qmm_device_status(_stream(dev), int(bool(reset))))


def qmm_set_path(path: str = "auto"):
    _check(lib().qmm_set_path(PATHS[path]))
    _mm_ws_size.clear()


def qmm_set_wait_limit_ns(ns: int = 0):
    """Limit of the kernels' bounded waits on the current device (0: the 2 s
    default).  For tests of the failure path."""
    _check(lib().qmm_set_wait_limit_ns(int(ns)))


FAULTS = {"none": 0, "streamk_no_publish": 1}


def qmm_inject_fault(fault: str = "none"):
    """Host-side fault injection for tests (see include/qmm.h)."""
    _check(lib().qmm_inject_fault(FAULTS[fault]))


def qmm_launch_count() -> int:
    """Kernels launched through libqmm by this process so far."""
    return int(lib().qmm_launch_count())


def qmm_version() -> int:
    return int(lib().qmm_version())
