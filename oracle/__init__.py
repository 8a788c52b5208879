"""CPU oracle for group-wise affine quantization and the quantized matmuls.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  It is
plain and slow on purpose, shares no code with the CUDA library, and never
imports it.

Parity status per function (what pins it is in ``tests/test_oracle_pins.py``):

  quantize            pinned: hand-packed words, on-grid round trip, brute-force
                      nearest-code search, the error bound of mlx-rs
                      ``test_quantize_dequantize``, the doctest shapes.
  dequantize          pinned: on-grid round trip, hand-packed words, bounds.
  quantized_matmul    pinned: reduces to a library float64 matmul when the
                      weight is exactly on the grid (both layouts), one-hot
                      rows, the doctest shapes, the mlx-rs
                      ``test_quantized_matmul`` bound.
  quantized_dense     pinned: a zero bias gives quantized_matmul exactly; a
                      one-hot row gives a column of the dequantized weight plus
                      the bias; a constant-bias tensor equals the number form.
  qqmm                pinned: the dequantized operands' library matmul on
                      values already on both grids, exact in float64; a
                      weight given dense equals the weight quantized first.
  gather_qmm          pinned: the two cases of mlx-rs ``test_gather_qmm``
                      against an independent indexed dense product.
"""
from .ref import (  # noqa: F401
    DTYPE_TAG,
    dequantize,
    MX_MODES,
    dequantize_f32,
    encode_elements,
    gather_qmm,
    qqmm,
    quantize,
    quantized_dense,
    quantized_matmul,
    round_to_dtype,
    unpack_codes,
)
