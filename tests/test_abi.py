"""C-ABI checks that need no GPU: the library loads, exports every function
declared in include/qmm.h, and rejects invalid arguments before launching."""
import ctypes
import re
from pathlib import Path

import pytest

from quantized_matmul_03_b200 import binding

HEADER = Path(__file__).resolve().parents[1] / "include" / "qmm.h"


@pytest.fixture(scope="module")
def L():
    from quantized_matmul_03_b200 import build
    build.build()
    return binding.lib()


def declared_functions():
    text = HEADER.read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(qmm_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("qmm_quantize", "qmm_dequantize", "qmm_quantized_matmul", "qmm_gather_qmm",
              "qmm_gather_qmm_workspace_size", "qmm_status_string", "qmm_device_status"):
        assert n in names


def test_library_exports_every_declared_function(L):
    missing = [n for n in declared_functions() if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings(L):
    for code, name in binding.STATUS_NAMES.items():
        assert L.qmm_status_string(code).decode() == name
    assert L.qmm_version() >= 100


FAKE = ctypes.c_void_p(0x10000)        # aligned, never dereferenced: calls fail first
MISALIGNED = ctypes.c_void_p(0x10004)
NULL = ctypes.c_void_p(0)


def q(L, **kw):
    a = dict(w=FAKE, dtype=1, rows=4, cols=128, gs=64, bits=4, mode=b"affine",
             wq=FAKE, s=FAKE, b=FAKE)
    a.update(kw)
    return L.qmm_quantize(a["w"], a["dtype"], a["rows"], a["cols"], a["gs"], a["bits"],
                          a["mode"], a["wq"], a["s"], a["b"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(bits=5), 1), (dict(bits=16), 1),
    (dict(gs=48), 1), (dict(gs=16), 1), (dict(cols=96), 1), (dict(cols=0), 1),
    (dict(rows=-1), 1), (dict(mode=b"nvfp4"), 1), (dict(mode=b"mxfp4"), 1),
    (dict(mode=b"mxfp8", gs=32), 1), (dict(mode=b"mxfp4", gs=32), 1),
    (dict(mode=b"bogus"), 1), (dict(dtype=7), 1),
    (dict(w=NULL), 1), (dict(wq=MISALIGNED), 1), (dict(b=NULL), 1),
])
def test_quantize_rejects_before_launch(L, kw, status):
    assert q(L, **kw) == status
    assert L.qmm_last_error()


def test_quantize_zero_rows_is_a_noop(L):
    assert q(L, rows=0, w=NULL, wq=NULL, s=NULL, b=NULL) == 0


def mm(L, **kw):
    a = dict(x=FAKE, M=2, K=128, wq=FAKE, s=FAKE, b=FAKE, dtype=1, N=64, tr=1, gs=64,
             bits=4, mode=None, y=FAKE)
    a.update(kw)
    return L.qmm_quantized_matmul(a["x"], a["M"], a["K"], a["wq"], a["s"], a["b"], a["dtype"],
                                  a["N"], a["tr"], a["gs"], a["bits"], a["mode"], a["y"], NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(K=96), 1), (dict(tr=0, N=96), 1), (dict(K=0), 1), (dict(M=-1), 1),
    (dict(b=NULL), 1), (dict(x=MISALIGNED), 1), (dict(y=NULL), 1),
    (dict(mode=b"nvfp4"), 1), (dict(mode=b"nvfp4", gs=16), 1), (dict(bits=5), 1),
    (dict(gs=256), 1),
])
def test_matmul_rejects_before_launch(L, kw, status):
    # (microscaled modes: a group size or bits other than the mode's, or a
    # non-NULL biases pointer, are invalid arguments)
    assert mm(L, **kw) == status


def test_matmul_empty_is_a_noop(L):
    assert mm(L, M=0, x=NULL, y=NULL) == 0
    assert mm(L, N=0, x=NULL, y=NULL) == 0


def test_set_path(L):
    assert L.qmm_set_path(7) == 1
    assert L.qmm_set_path(0) == 0


def mmws(L, ws=NULL, ws_bytes=0, **kw):
    a = dict(x=FAKE, M=2, K=128, wq=FAKE, s=FAKE, b=FAKE, dtype=1, N=64, tr=1, gs=64,
             bits=4, mode=None, y=FAKE)
    a.update(kw)
    return L.qmm_quantized_matmul_ws(a["x"], a["M"], a["K"], a["wq"], a["s"], a["b"], a["dtype"],
                                     a["N"], a["tr"], a["gs"], a["bits"], a["mode"], a["y"],
                                     ws, ws_bytes, NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(K=96), 1), (dict(tr=0, N=96), 1), (dict(b=NULL), 1), (dict(x=MISALIGNED), 1),
    (dict(mode=b"nvfp4"), 1), (dict(bits=7), 1),
])
def test_matmul_ws_rejects_like_the_plain_call(L, kw, status):
    assert mmws(L, **kw) == status


def test_matmul_ws_checks_workspace_alignment(L):
    assert mmws(L, ws=ctypes.c_void_p(0x10080), ws_bytes=1 << 20) == 6  # QMM_ERR_WORKSPACE
    assert mmws(L, M=0, x=NULL, y=NULL) == 0


def test_matmul_workspace_size(L):
    """Stream-K (and so a workspace) only for narrow tiles (at most 64
    activation rows) when the problem has fewer 128-feature tiles than SMs."""
    ws = lambda M, K, N, tr=1, bits=4, dt=1: int(L.qmm_quantized_matmul_workspace_size(
        M, K, N, tr, bits, dt))
    need = ws(16, 4096, 4096)
    assert need > 4096                          # flags, then one partial slot per SM
    assert ws(64, 4096, 4096) == need and ws(1, 4096, 4096, tr=0) == need
    assert ws(4, 4096, 4096) == 0               # decode rows go to the SIMT decode kernel
    assert ws(1, 4096, 4096, bits=8) == 0       # (8-bit codes too)
    assert ws(1, 4096, 4096, bits=3) > 4096     # 3/6-bit rows: the tensor-core GEMM, split
    assert ws(4, 4096, 14336, bits=6) > 4096
    assert ws(4, 4096, 4096, bits=2) >= 4096 + 48 * 4096   # 2-bit rows: the decode tensor-core kernel
    assert ws(128, 4096, 4096) == 0             # wide tiles keep whole tiles
    assert ws(64, 4096, 14336 * 4) == 0         # at least one full wave of tiles
    assert ws(16, 4096, 4096, dt=0) == 0        # f32 has no tensor-core path
    assert ws(16, 4000, 4096) == 0              # K not a multiple of the k-block


def test_fault_injection_rejects_unknown_values(L):
    assert L.qmm_inject_fault(99) == 1
    assert L.qmm_inject_fault(0) == 0


def mmhost(L, xh=FAKE, yh=FAKE, **kw):
    a = dict(x=FAKE, M=2, K=128, wq=FAKE, s=FAKE, b=FAKE, dtype=1, N=64, tr=1, gs=64,
             bits=4, mode=None, y=FAKE)
    a.update(kw)
    return L.qmm_quantized_matmul_host(xh, a["x"], a["M"], a["K"], a["wq"], a["s"], a["b"],
                                       a["dtype"], a["N"], a["tr"], a["gs"], a["bits"], a["mode"],
                                       a["y"], yh, NULL, 0, NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(xh=NULL), 1), (dict(yh=NULL), 1), (dict(K=96), 1), (dict(b=NULL), 1),
    (dict(x=MISALIGNED), 1), (dict(bits=7), 1), (dict(mode=b"nvfp4"), 1),
])
def test_matmul_host_rejects_before_any_copy(L, kw, status):
    """The host-buffer entry checks every argument (and that the host buffers
    are given) before it enqueues a copy: these calls touch no device."""
    assert mmhost(L, **kw) == status


def test_matmul_host_empty_is_a_noop(L):
    assert mmhost(L, M=0, x=NULL, y=NULL, xh=NULL, yh=NULL) == 0


def mmmapped(L, xm=FAKE, ym=FAKE, **kw):
    a = dict(x=FAKE, M=2, K=128, wq=FAKE, s=FAKE, b=FAKE, dtype=1, N=64, tr=1, gs=64,
             bits=4, mode=None, y=FAKE)
    a.update(kw)
    return L.qmm_quantized_matmul_mapped(xm, a["x"], a["M"], a["K"], a["wq"], a["s"], a["b"],
                                         a["dtype"], a["N"], a["tr"], a["gs"], a["bits"],
                                         a["mode"], a["y"], ym, NULL, 0, NULL)


@pytest.mark.parametrize("kw,status", [
    (dict(xm=NULL), 1), (dict(ym=NULL), 1), (dict(K=96), 1), (dict(b=NULL), 1),
    (dict(x=MISALIGNED), 1), (dict(bits=7), 1),
])
def test_matmul_mapped_rejects_before_any_copy(L, kw, status):
    """The mapped entry checks its mappings and every argument before it
    enqueues anything."""
    assert mmmapped(L, **kw) == status


def test_matmul_mapped_empty_is_a_noop(L):
    assert mmmapped(L, M=0, x=NULL, y=NULL, xm=NULL, ym=NULL) == 0


def test_mapped_pointer_of_ordinary_memory_is_null(L):
    """Pageable host memory (and NULL) has no device mapping."""
    buf = ctypes.create_string_buffer(256)
    assert L.qmm_mapped_pointer(ctypes.addressof(buf)) is None
    assert L.qmm_mapped_pointer(None) is None
