"""Host-side checks of the C ABI: the library loads, exports every symbol the
header declares, and rejects bad arguments before launching anything.

No call here reaches a CUDA kernel (every argument set is invalid), so these
run without a GPU.
"""
import ctypes
import os
import re

import pytest

import mixed_precision_weight_row_b200 as mpw
import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "mpw.h")

A16 = 0x10000          # fake, 16-byte aligned "device" addresses (never dereferenced)
A16B = 0x20000
ODD = 0x10001


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MPW_API\s+[\w\s\*]+?\b(mpw_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("mpw_quantize_pack", "mpw_unpack", "mpw_dequantize", "mpw_qlinear",
                 "mpw_qlinear_path", "mpw_recipe_run", "mpw_packed_row_bytes",
                 "mpw_status_str", "mpw_version", "mpw_device_error", "mpw_repack",
                 "mpw_qlinear_ex", "mpw_qlinear_ws", "mpw_qlinear_workspace_bytes",
                 "mpw_recipe_run_ws", "mpw_recipe_workspace_bytes", "mpw_qlinear_flags"):
        assert want in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(mpw.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings():
    for st in range(0, 10):
        assert mpw.status_str(st) and mpw.status_str(st) != "unknown status"
    assert mpw.status_str(99) == "unknown status"


@pytest.mark.parametrize("bits", list(range(4, 16)))
def test_packed_row_bytes_matches_oracle(bits):
    for K in (1, 2, 31, 32, 33, 127, 128, 129, 4096, 5120, 17408, 100001):
        assert mpw.packed_row_bytes(K, bits) == oracle.packed_row_bytes(K, bits)


def test_packed_row_bytes_invalid():
    assert mpw.packed_row_bytes(10, 3) == 0
    assert mpw.packed_row_bytes(10, 16) == 0
    assert mpw.packed_row_bytes(0, 8) == 0
    assert mpw.packed_row_bytes(-5, 8) == 0


def test_quantize_pack_validation():
    L = mpw.lib
    assert L.mpw_quantize_pack(A16, 4, 4, 3, A16B, A16, 0, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_quantize_pack(A16, 4, 4, 16, A16B, A16, 0, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_quantize_pack(0, 4, 4, 5, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, 4, 4, 5, 0, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, 4, 4, 5, A16B, 0, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, 0, 4, 5, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, 4, 0, 5, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, -1, 4, 5, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_pack(A16, 4, 4, 5, A16B + 8, A16, 0, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_quantize_pack(A16 + 2, 4, 4, 5, A16B, A16, 0, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_quantize_pack(A16, 4, 4, 5, A16B, A16, ODD, 0) == mpw.MPW_E_MISALIGNED


def test_unpack_and_dequantize_validation():
    L = mpw.lib
    assert L.mpw_unpack(A16, 4, 4, 2, A16B, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_unpack(0, 4, 4, 5, A16B, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_unpack(A16, 4, 4, 5, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_unpack(A16 + 4, 4, 4, 5, A16B, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_unpack(A16, 4, 4, 5, ODD, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_dequantize(A16, A16B, 4, 4, 17, A16, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_dequantize(A16, 0, 4, 4, 5, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_dequantize(A16, A16B, 4, 0, 5, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_dequantize(A16, A16B + 1, 4, 4, 5, A16, 0) == mpw.MPW_E_MISALIGNED


def test_qlinear_validation():
    L = mpw.lib
    assert L.mpw_qlinear(A16, A16B, A16, 3, 1, 4, 4, A16, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_qlinear(0, A16B, A16, 5, 1, 4, 4, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear(A16, A16B, A16, 5, 0, 4, 4, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear(A16, A16B, A16, 5, 1, 0, 4, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear(A16, A16B, A16, 5, 1, 4, 0, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear(A16, A16B, A16, 5, 1, 4, 4, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear(A16, A16B + 8, A16, 5, 1, 4, 4, A16, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_qlinear(ODD, A16B, A16, 5, 1, 4, 4, A16, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_qlinear_path(A16, A16B, A16, 5, 1, 4, 4, A16, 7, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_path(A16, A16B, A16, 5, 1, 4, 4, A16, -1, 0) == mpw.MPW_E_INVALID_ARG


def test_repack_validation():
    L = mpw.lib
    assert L.mpw_repack(A16, 4, 64, 3, 0, 1, A16B, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_repack(0, 4, 64, 5, 0, 1, A16B, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_repack(A16, 4, 64, 5, 0, 1, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_repack(A16, 4, 48, 5, 0, 1, A16B, 0) == mpw.MPW_E_INVALID_ARG      # K % 32 != 0
    assert L.mpw_repack(A16, 0, 64, 5, 0, 1, A16B, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_repack(A16, 4, 64, 5, 1, 1, A16B, 0) == mpw.MPW_E_INVALID_ARG      # same layout
    assert L.mpw_repack(A16, 4, 64, 5, 0, 2, A16B, 0) == mpw.MPW_E_INVALID_ARG      # unknown layout
    assert L.mpw_repack(A16, 4, 64, 5, -1, 1, A16B, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_repack(A16 + 8, 4, 64, 5, 0, 1, A16B, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_repack(A16, 4, 64, 5, 0, 1, A16B + 4, 0) == mpw.MPW_E_MISALIGNED
    # partial overlap (in place is allowed, a shifted copy is not)
    assert L.mpw_repack(A16, 4, 64, 5, 0, 1, A16 + 16, 0) == mpw.MPW_E_INVALID_ARG


def test_qlinear_ex_validation():
    L = mpw.lib
    assert L.mpw_qlinear_ex(A16, A16B, A16, 5, 2, 1, 4, 64, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_ex(A16, A16B, A16, 5, -1, 1, 4, 64, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_ex(A16, A16B, A16, 5, 1, 1, 4, 48, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_ex(A16 + 2, A16B, A16, 5, 1, 1, 4, 64, A16, 0, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_qlinear_ex(A16, A16B, A16, 5, 1, 1, 4, 64, A16, 3, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_ex(A16, A16B, A16, 2, 1, 1, 4, 64, A16, 0, 0) == mpw.MPW_E_UNSUPPORTED_BITS


def test_qlinear_flags_validation():
    L = mpw.lib
    # unknown flag bits are an argument error; the usual checks still apply
    assert L.mpw_qlinear_flags(A16, A16B, A16, 5, 1, 1, 4, 64, A16, 0, 2, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_flags(A16, A16B, A16, 5, 1, 1, 4, 64, A16, 0, 0x80000000, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_flags(A16, A16B, A16, 3, 1, 1, 4, 64, A16, 0, mpw.X_READY, 0) == \
        mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_qlinear_flags(A16 + 2, A16B, A16, 5, 1, 1, 4, 64, A16, 0, mpw.X_READY, 0) == \
        mpw.MPW_E_MISALIGNED
    assert L.mpw_qlinear_flags(A16, A16B, A16, 5, 1, 1, 4, 48, A16, 0, mpw.X_READY, 0) == mpw.MPW_E_INVALID_ARG
    # y_unshared needs x_ready; bit 2 is not a flag
    assert L.mpw_qlinear_flags(A16, A16B, A16, 5, 1, 1, 4, 64, A16, 0, mpw.Y_UNSHARED, 0) == \
        mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_flags(A16, A16B, A16, 5, 1, 1, 4, 64, A16, 0, 4, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_flags(A16, A16B, A16, 3, 1, 1, 4, 64, A16, 0, mpw.X_READY | mpw.Y_UNSHARED, 0) == \
        mpw.MPW_E_UNSUPPORTED_BITS


def test_binding_rejects_x_ready_with_workspace():
    import torch

    x = torch.zeros((1, 64), dtype=torch.bfloat16)
    p = torch.zeros((4, mpw.packed_row_bytes(64, 5)), dtype=torch.uint8)
    s = torch.ones((4,), dtype=torch.float32)
    with pytest.raises(ValueError):
        mpw.qlinear(x, p, s, 5, x_ready=True, use_workspace=True)
    with pytest.raises(ValueError):
        mpw.qlinear(x, p, s, 5, y_unshared=True)


def test_qlinear_ws_validation():
    L = mpw.lib
    # a workspace must be 16-byte aligned; argument errors come first
    assert L.mpw_qlinear_ws(A16, A16B, A16, 5, 0, 1, 4, 64, A16, 0, A16 + 8, 4096, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_qlinear_ws(A16, A16B, A16, 3, 0, 1, 4, 64, A16, 0, A16, 4096, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_qlinear_ws(0, A16B, A16, 5, 0, 1, 4, 64, A16, 0, A16, 4096, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_qlinear_workspace_bytes(3, 0, 1, 4, 64) == 0
    assert L.mpw_qlinear_workspace_bytes(5, 2, 1, 4, 64) == 0
    assert L.mpw_qlinear_workspace_bytes(5, 0, 33, 4, 64) == 0      # not a decode call


def test_recipe_run_ws_validation():
    L = mpw.lib
    slots = (ctypes.c_void_p * 3)(A16, A16B, A16 + 0x100)
    good = (A16, A16B, 8, 64, 6, 0, 1, 0)
    assert L.mpw_recipe_run_ws(_layers(good), 1, slots, 3, 1, A16 + 4, 4096, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_recipe_run_ws(_layers(good), 0, slots, 3, 1, A16, 4096, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_workspace_bytes(_layers(good), 0, 1) == 0
    assert L.mpw_recipe_workspace_bytes(_layers(good), 1, 33) == 0


def _layers(*specs):
    arr = (mpw._Linear * len(specs))()
    for i, s in enumerate(specs):
        arr[i] = mpw._Linear(*s)
    return arr


def test_recipe_run_validation():
    L = mpw.lib
    slots = (ctypes.c_void_p * 3)(A16, A16B, A16 + 0x100)
    good = (A16, A16B, 8, 8, 6, 0, 1, 0)
    assert L.mpw_recipe_run(_layers(good), 0, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers(good), 1, slots, 3, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers(good), 1, slots, 3, 33, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 8, 3, 0, 1, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 8, 6, 0, 0, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 8, 6, 0, 3, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 8, 6, -1, 1, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((0, A16B, 8, 8, 6, 0, 1, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16 + 4, A16B, 8, 8, 6, 0, 1, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_MISALIGNED
    # an invalid entry anywhere in the list rejects the whole call before any launch
    assert L.mpw_recipe_run(_layers(good, (A16, A16B, 8, 0, 6, 1, 2, 0)), 2, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    nulls = (ctypes.c_void_p * 3)(A16, 0, A16B)
    assert L.mpw_recipe_run(_layers(good), 1, nulls, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    # layouts: unknown value, reserved field, K % 32 for paired, x alignment for paired
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 64, 6, 0, 1, 0, 2, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 64, 6, 0, 1, 0, 0, 1)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 48, 6, 0, 1, 0, 1, 0)), 1, slots, 3, 1, 0) == mpw.MPW_E_INVALID_ARG
    odd_slots = (ctypes.c_void_p * 3)(A16 + 2, A16B, A16 + 0x100)
    assert L.mpw_recipe_run(_layers((A16, A16B, 8, 64, 6, 0, 1, 0, 1, 0)), 1, odd_slots, 3, 1, 0) == mpw.MPW_E_MISALIGNED


def test_device_error_rejects_null():
    assert mpw.lib.mpw_device_error(None) == mpw.MPW_E_INVALID_ARG


def test_binding_rejects_host_tensors():
    import torch

    W = torch.zeros((4, 8), dtype=torch.float32)
    with pytest.raises(ValueError):
        mpw.quantize_pack(W, 5)
    with pytest.raises(TypeError):
        mpw.quantize_pack(W.double(), 5)


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "mixed_precision_weight_row_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".h", ".cuh")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_group_entry_points_validation():
    """Group-wise scales: the group size, shapes, layout and alignment are
    checked before anything is launched."""
    L = mpw.lib
    qg = L.mpw_quantize_pack_groups
    assert qg(A16, 4, 256, 3, 128, A16B, A16, 0, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    for bad_group in (0, 16, 48, 96, 2048, -128):
        assert qg(A16, 4, 256, 5, bad_group, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG, bad_group
    assert qg(0, 4, 256, 5, 128, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert qg(A16, 0, 256, 5, 128, A16B, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert qg(A16, 4, 256, 5, 128, A16B + 8, A16, 0, 0) == mpw.MPW_E_MISALIGNED
    assert qg(A16, 4, 256, 5, 128, A16B, A16 + 2, 0, 0) == mpw.MPW_E_MISALIGNED
    ql = L.mpw_qlinear_groups
    # x, packed, scales, bits, group, layout, M, N, K, y, stream
    assert ql(A16, A16B, A16, 16, 128, 0, 1, 16, 256, A16, 0, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    for bad_group in (32, 64, 100, 2048):
        assert ql(A16, A16B, A16, 5, bad_group, 0, 1, 16, 256, A16, 0, 0) == mpw.MPW_E_INVALID_ARG, bad_group
    assert ql(A16, A16B, A16, 5, 128, 2, 1, 16, 256, A16, 0, 0) == mpw.MPW_E_INVALID_ARG      # layout
    assert ql(A16, A16B, A16, 5, 128, 0, 0, 16, 256, A16, 0, 0) == mpw.MPW_E_INVALID_ARG      # M
    assert ql(A16, A16B, A16, 5, 128, 0, 1, 16, 250, A16, 0, 0) == mpw.MPW_E_INVALID_ARG      # K % 8
    assert ql(A16, A16B, A16, 5, 128, 1, 1, 16, 264, A16, 0, 0) == mpw.MPW_E_INVALID_ARG      # paired K % 32
    assert ql(A16 + 8, A16B, A16, 5, 128, 0, 1, 16, 256, A16, 0, 0) == mpw.MPW_E_MISALIGNED  # x 16-byte
    assert ql(0, A16B, A16, 5, 128, 0, 1, 16, 256, A16, 0, 0) == mpw.MPW_E_INVALID_ARG
    assert ql(A16, A16B, A16, 5, 128, 0, 1, 16, 256, A16, 2, 0) == mpw.MPW_E_INVALID_ARG   # y_unshared alone
    assert ql(A16, A16B, A16, 5, 128, 0, 1, 16, 256, A16, 4, 0) == mpw.MPW_E_INVALID_ARG   # unknown flag


def test_fp8_entry_points_validation():
    L = mpw.lib
    # x, M, K, xq, sx, stream
    assert L.mpw_quantize_x_fp8(0, 4, 64, A16B, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_x_fp8(A16, 0, 64, A16B, A16, 0) == mpw.MPW_E_INVALID_ARG
    assert L.mpw_quantize_x_fp8(A16, 4, 72, A16B, A16, 0) == mpw.MPW_E_INVALID_ARG     # K % 16
    assert L.mpw_quantize_x_fp8(A16 + 2, 4, 64, A16B, A16, 0) == mpw.MPW_E_MISALIGNED
    assert L.mpw_quantize_x_fp8(A16, 4, 64, A16B + 8, A16, 0) == mpw.MPW_E_MISALIGNED
    q8 = L.mpw_qlinear_fp8
    # xq, sx, packed, scales, bits, layout, M, N, K, y, stream
    for b in (3, 6, 8, 15):
        assert q8(A16, A16, A16B, A16, b, 0, 4, 16, 64, A16, 0) == mpw.MPW_E_UNSUPPORTED_BITS
    assert q8(A16, A16, A16B, A16, 5, 0, 4, 16, 72, A16, 0) == mpw.MPW_E_INVALID_ARG      # K % 16
    assert q8(A16, A16, A16B, A16, 5, 1, 4, 16, 80, A16, 0) == mpw.MPW_E_INVALID_ARG      # paired K % 32
    assert q8(A16, A16, A16B, A16, 5, 2, 4, 16, 64, A16, 0) == mpw.MPW_E_INVALID_ARG      # layout
    assert q8(A16 + 8, A16, A16B, A16, 5, 0, 4, 16, 64, A16, 0) == mpw.MPW_E_MISALIGNED
    assert q8(A16, A16, A16B + 8, A16, 5, 0, 4, 16, 64, A16, 0) == mpw.MPW_E_MISALIGNED
    assert q8(0, A16, A16B, A16, 5, 0, 4, 16, 64, A16, 0) == mpw.MPW_E_INVALID_ARG
