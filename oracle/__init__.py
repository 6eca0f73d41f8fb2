"""CPU oracle for the packed INT-b quantizer and the fused linear layer.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.
"""
from .quant import (  # noqa: F401
    MAX_BITS,
    MIN_BITS,
    PAIR_GROUP,
    QLINEAR_ABS_TOL,
    QLINEAR_REL_TOL,
    check_qlinear,
    dequantize,
    dequantize_groups,
    group_count,
    group_scale_of_weight,
    group_scales,
    pack,
    pack_paired,
    pair_halves,
    packed_row_bytes,
    qlinear_groups_ref,
    qlinear_ref,
    qlinear_rows_ref,
    qmax,
    quality,
    quantize,
    quantize_groups,
    quantize_pack,
    qlinear_rms_ref,
    rms_scale,
    row_scales,
    unpack,
    unpack_paired,
    unpadded_row_bytes,
)
from .fp8 import (  # noqa: F401
    E4M3_MAX,
    FP8_MAX_BITS,
    e4m3_round,
    fp8_input_error_bound,
    qlinear_fp8_ref,
    quantize_x_fp8,
)
