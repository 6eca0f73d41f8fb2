"""CPU oracle for the packed INT-b quantizer and the fused linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.
"""
from .quant import (  # noqa: F401
    MAX_BITS,
    MIN_BITS,
    QLINEAR_ABS_TOL,
    QLINEAR_REL_TOL,
    check_qlinear,
    dequantize,
    pack,
    packed_row_bytes,
    qlinear_ref,
    qlinear_rows_ref,
    qmax,
    quality,
    quantize,
    quantize_pack,
    qlinear_rms_ref,
    rms_scale,
    row_scales,
    unpack,
    unpadded_row_bytes,
)
