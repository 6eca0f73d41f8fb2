"""Packed INT-b weight rows and the fused dequantize-linear layer on B200.

Thin Python binding over ``libmpw.so`` (C ABI declared in ``include/mpw.h``).
This module only marshals arguments: it checks tensor dtypes, devices and
shapes, allocates outputs with torch when the caller does not pass them, and
forwards raw device pointers and the current CUDA stream.  Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback, and
the first call raises ImportError if the library has not been built.

Build: ``python -m mixed_precision_weight_row_b200.build``.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

__all__ = [
    "MPWError", "LIB_PATH", "lib", "packed_row_bytes", "quantize_pack", "unpack",
    "dequantize", "repack", "qlinear", "Linear", "recipe_run", "device_error", "status_str", "allocate_bits", "allocation_frontier",
    "recipe_plan", "save_packed", "load_packed", "Pass", "pass_dependencies",
    "LAYOUTS", "workspace", "qlinear_workspace_bytes", "quantize_pack_groups", "qlinear_groups",
    "gather_shards", "quantize_x_fp8", "qlinear_fp8",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmpw.so")

MPW_OK = 0
MPW_E_INVALID_ARG = 1
MPW_E_UNSUPPORTED_BITS = 2
MPW_E_MISALIGNED = 3
MPW_E_CUDA = 4
MPW_E_NONFINITE = 5
MPW_E_TIMEOUT = 6
MPW_E_SCRATCH_LIMIT = 7
MPW_E_IO = 8
MPW_E_FORMAT = 9
MPW_E_UNSUPPORTED = 10

PATHS = {"auto": 0, "gemv": 1, "gemm": 2}
# Packed layouts (mpw_layout): the canonical stream and its paired-halves
# re-ordering, which the decode kernels read fastest (K % 32 == 0).
LAYOUTS = {"canonical": 0, "paired": 1}
# mpw_qlinear_flags: x was written before the launch preceding the run of
# flagged calls
X_READY = 1
# with X_READY: no other call of the run, nor the launch before it, touches y
Y_UNSHARED = 2


class MPWError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_str(status)} (status {status})")


class _FileMatrix(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("bits", ctypes.c_int32),
        ("layout", ctypes.c_int32),
        ("packed", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
    ]


class _Linear(ctypes.Structure):
    _fields_ = [
        ("packed", ctypes.c_void_p),
        ("scales", ctypes.c_void_p),
        ("N", ctypes.c_int64),
        ("K", ctypes.c_int64),
        ("bits", ctypes.c_int32),
        ("in_slot", ctypes.c_int32),
        ("out_slot", ctypes.c_int32),
        ("norm_input", ctypes.c_int32),
        ("layout", ctypes.c_int32),
        ("reserved", ctypes.c_int32),
    ]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -m mixed_precision_weight_row_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, c_int = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int
    L.mpw_status_str.argtypes = [c_int]
    L.mpw_status_str.restype = ctypes.c_char_p
    L.mpw_version.argtypes = []
    L.mpw_version.restype = c_int
    L.mpw_packed_row_bytes.argtypes = [i64, c_int]
    L.mpw_packed_row_bytes.restype = ctypes.c_size_t
    L.mpw_quantize_pack.argtypes = [vp, i64, i64, c_int, vp, vp, vp, vp]
    L.mpw_quantize_pack.restype = c_int
    L.mpw_unpack.argtypes = [vp, i64, i64, c_int, vp, vp]
    L.mpw_unpack.restype = c_int
    L.mpw_dequantize.argtypes = [vp, vp, i64, i64, c_int, vp, vp]
    L.mpw_dequantize.restype = c_int
    L.mpw_qlinear.argtypes = [vp, vp, vp, c_int, i64, i64, i64, vp, vp]
    L.mpw_qlinear.restype = c_int
    L.mpw_qlinear_path.argtypes = [vp, vp, vp, c_int, i64, i64, i64, vp, c_int, vp]
    L.mpw_qlinear_path.restype = c_int
    L.mpw_qlinear_ex.argtypes = [vp, vp, vp, c_int, c_int, i64, i64, i64, vp, c_int, vp]
    L.mpw_qlinear_ex.restype = c_int
    L.mpw_repack.argtypes = [vp, i64, i64, c_int, c_int, c_int, vp, vp]
    L.mpw_repack.restype = c_int
    L.mpw_qlinear_workspace_bytes.argtypes = [c_int, c_int, i64, i64, i64]
    L.mpw_qlinear_workspace_bytes.restype = ctypes.c_size_t
    L.mpw_qlinear_ws.argtypes = [vp, vp, vp, c_int, c_int, i64, i64, i64, vp, c_int, vp, ctypes.c_size_t, vp]
    L.mpw_qlinear_ws.restype = c_int
    L.mpw_qlinear_flags.argtypes = [vp, vp, vp, c_int, c_int, i64, i64, i64, vp, c_int, ctypes.c_uint, vp]
    L.mpw_qlinear_flags.restype = c_int
    L.mpw_allocate_bits.argtypes = [vp, vp, vp, i64, ctypes.c_uint64, c_int, vp, vp]
    L.mpw_allocate_bits.restype = c_int
    L.mpw_allocate_frontier.argtypes = [vp, vp, vp, i64, c_int, vp, vp, i64, ctypes.POINTER(i64)]
    L.mpw_allocate_frontier.restype = c_int
    L.mpw_recipe_plan.argtypes = [ctypes.POINTER(_Linear), i64, ctypes.POINTER(vp), i64, i64,
                                  ctypes.POINTER(ctypes.c_uint32)]
    L.mpw_recipe_plan.restype = c_int
    L.mpw_file_write.argtypes = [ctypes.c_char_p, ctypes.POINTER(_FileMatrix), i64]
    L.mpw_file_write.restype = c_int
    L.mpw_file_count.argtypes = [ctypes.c_char_p, ctypes.POINTER(i64)]
    L.mpw_file_count.restype = c_int
    L.mpw_file_info.argtypes = [ctypes.c_char_p, i64, ctypes.POINTER(i64), ctypes.POINTER(i64), ctypes.POINTER(i32),
                                ctypes.POINTER(i32)]
    L.mpw_file_info.restype = c_int
    L.mpw_file_read.argtypes = [ctypes.c_char_p, i64, vp, vp]
    L.mpw_file_read.restype = c_int
    L.mpw_recipe_workspace_bytes.argtypes = [ctypes.POINTER(_Linear), i64, i64]
    L.mpw_recipe_workspace_bytes.restype = ctypes.c_size_t
    L.mpw_recipe_run_ws.argtypes = [ctypes.POINTER(_Linear), i64, ctypes.POINTER(vp), i64, i64, vp,
                                    ctypes.c_size_t, vp]
    L.mpw_recipe_run_ws.restype = c_int
    L.mpw_qlinear_noalloc.argtypes = [vp, vp, vp, c_int, c_int, i64, i64, i64, vp, vp]
    L.mpw_qlinear_noalloc.restype = c_int
    L.mpw_recipe_run.argtypes = [ctypes.POINTER(_Linear), i64, ctypes.POINTER(vp), i64, i64, vp]
    L.mpw_recipe_run.restype = c_int
    L.mpw_pass_create.argtypes = [ctypes.POINTER(_Linear), i64, ctypes.POINTER(vp), i64, i64, ctypes.POINTER(vp)]
    L.mpw_pass_create.restype = c_int
    L.mpw_pass_run.argtypes = [vp, vp]
    L.mpw_pass_run.restype = c_int
    L.mpw_pass_info.argtypes = [vp, ctypes.POINTER(i64)]
    L.mpw_pass_info.restype = c_int
    L.mpw_pass_destroy.argtypes = [vp]
    L.mpw_pass_destroy.restype = None
    L.mpw_pass_dependencies.argtypes = [ctypes.POINTER(_Linear), i64, ctypes.POINTER(vp), i64, i64,
                                        ctypes.POINTER(i32), ctypes.POINTER(i32), i64]
    L.mpw_pass_dependencies.restype = c_int
    L.mpw_quantize_pack_groups.argtypes = [vp, i64, i64, c_int, i64, vp, vp, vp, vp]
    L.mpw_quantize_pack_groups.restype = c_int
    L.mpw_qlinear_groups.argtypes = [vp, vp, vp, c_int, i64, c_int, i64, i64, i64, vp, ctypes.c_uint, vp]
    L.mpw_qlinear_groups.restype = c_int
    L.mpw_quantize_x_fp8.argtypes = [vp, i64, i64, vp, vp, vp]
    L.mpw_quantize_x_fp8.restype = c_int
    L.mpw_qlinear_fp8.argtypes = [vp, vp, vp, vp, c_int, c_int, i64, i64, i64, vp, vp]
    L.mpw_qlinear_fp8.restype = c_int
    L.mpw_gather_shards.argtypes = [vp, i64, i64, i64, i64, vp, vp]
    L.mpw_gather_shards.restype = c_int
    L.mpw_device_error.argtypes = [ctypes.POINTER(i32)]
    L.mpw_device_error.restype = c_int
    return L


class _Lib:
    """libmpw.so, opened on first use.  The build step imports this package
    before the library exists, so the import itself does not open it; the
    first call raises ImportError if the library has not been built."""

    _handle = None

    def __getattr__(self, name):
        if _Lib._handle is None:
            _Lib._handle = _load()
        return getattr(_Lib._handle, name)


lib = _Lib()


def status_str(status: int) -> str:
    return lib.mpw_status_str(int(status)).decode()


def _check(status: int, where: str) -> None:
    if status != MPW_OK:
        raise MPWError(status, where)


def _stream(stream=None) -> int:
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _need(t, dtype, name, ndim=None):
    import torch

    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims")


# Decode workspaces (see mpw_qlinear_workspace_bytes in mpw.h), one per
# (device, stream): zero-filled when created, grown by replacement.  Calls on
# one stream are ordered, so they may share it.
_workspaces = {}


def workspace(nbytes: int, stream=None):
    """A zero-filled decode workspace of at least ``nbytes`` for this stream."""
    import torch

    if nbytes <= 0:
        return None
    dev = torch.cuda.current_device()
    key = (dev, _stream(stream))
    ws = _workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        size = max(int(nbytes), 1 << 20, 0 if ws is None else 2 * ws.numel())
        ws = torch.zeros(size, dtype=torch.uint8, device=f"cuda:{dev}")
        _workspaces[key] = ws
    return ws


def qlinear_workspace_bytes(bits: int, M: int, N: int, K: int, layout: str = "canonical") -> int:
    return int(lib.mpw_qlinear_workspace_bytes(int(bits), LAYOUTS[layout], int(M), int(N), int(K)))


def packed_row_bytes(K: int, bits: int) -> int:
    """16 * ceil(K * bits / 128); 0 if bits is outside 4..15 or K < 1."""
    return int(lib.mpw_packed_row_bytes(int(K), int(bits)))


def quantize_pack(W, bits: int, packed=None, scales=None, nonfinite_flag=None, stream=None):
    """W fp32 [N, K] (CUDA) -> (packed uint8 [N, row_bytes], scales fp32 [N])."""
    import torch

    _need(W, torch.float32, "W", 2)
    N, K = W.shape
    rb = packed_row_bytes(K, bits)
    if packed is None:
        packed = torch.empty((N, max(rb, 16)), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((N,), dtype=torch.float32, device=W.device)
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.float32, "scales")
    flag = 0 if nonfinite_flag is None else nonfinite_flag.data_ptr()
    _check(lib.mpw_quantize_pack(W.data_ptr(), N, K, int(bits), packed.data_ptr(), scales.data_ptr(),
                                 flag, _stream(stream)), "mpw_quantize_pack")
    return packed, scales


def unpack(packed, K: int, bits: int, codes=None, stream=None):
    """packed uint8 [N, row_bytes] -> codes int16 [N, K]."""
    import torch

    _need(packed, torch.uint8, "packed", 2)
    N = packed.shape[0]
    if codes is None:
        codes = torch.empty((N, K), dtype=torch.int16, device=packed.device)
    _need(codes, torch.int16, "codes")
    _check(lib.mpw_unpack(packed.data_ptr(), N, int(K), int(bits), codes.data_ptr(), _stream(stream)),
           "mpw_unpack")
    return codes


def dequantize(packed, scales, K: int, bits: int, out=None, stream=None):
    """(packed, scales) -> fl32(q * s) as fp32 [N, K]."""
    import torch

    _need(packed, torch.uint8, "packed", 2)
    _need(scales, torch.float32, "scales", 1)
    N = packed.shape[0]
    if out is None:
        out = torch.empty((N, K), dtype=torch.float32, device=packed.device)
    _need(out, torch.float32, "out")
    _check(lib.mpw_dequantize(packed.data_ptr(), scales.data_ptr(), N, int(K), int(bits), out.data_ptr(),
                              _stream(stream)), "mpw_dequantize")
    return out


def repack(packed, K: int, bits: int, layout_in: str = "canonical", layout_out: str = "paired", out=None,
           stream=None):
    """Re-order packed rows between layouts; ``out=packed`` runs in place."""
    import torch

    _need(packed, torch.uint8, "packed", 2)
    if out is None:
        out = torch.empty_like(packed)
    _need(out, torch.uint8, "out", 2)
    if out.shape != packed.shape:
        raise ValueError("out must have the shape of packed")
    if packed.shape[1] != packed_row_bytes(K, bits):
        raise ValueError("packed rows must be exactly packed_row_bytes(K, bits) long")
    _check(lib.mpw_repack(packed.data_ptr(), packed.shape[0], int(K), int(bits), LAYOUTS[layout_in],
                          LAYOUTS[layout_out], out.data_ptr(), _stream(stream)), "mpw_repack")
    return out


def qlinear(x, packed, scales, bits: int, y=None, path: str = "auto", layout: str = "canonical",
            stream=None, use_workspace: bool = False, x_ready: bool = False, y_unshared: bool = False):
    """y = x @ (q * s)^T with x bf16 [M, K]; returns y bf16 [M, N].

    With ``use_workspace`` the decode path (M <= 32) gets this stream's
    workspace and runs the stream-K kernel; without it (the default, faster
    on every measured shape) the per-tile kernel.  ``x_ready`` states that x
    was written before the launch that precedes the current run of x_ready
    calls on the stream (MPW_QLINEAR_X_READY in mpw.h); it cannot be combined
    with a workspace.  ``y_unshared`` (only with ``x_ready``) states that no
    other call of that run, nor the launch before it, reads or writes y
    (MPW_QLINEAR_Y_UNSHARED)."""
    import torch

    if x_ready and use_workspace:
        raise ValueError("x_ready cannot be combined with use_workspace")
    if y_unshared and not x_ready:
        raise ValueError("y_unshared needs x_ready")
    _need(x, torch.bfloat16, "x", 2)
    _need(packed, torch.uint8, "packed", 2)
    _need(scales, torch.float32, "scales", 1)
    M, K = x.shape
    N = packed.shape[0]
    if scales.shape[0] != N:
        raise ValueError("scales must have one entry per packed row")
    if packed.shape[1] != packed_row_bytes(K, bits):
        raise ValueError("packed rows must be exactly packed_row_bytes(K, bits) long")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, "y")
    if x_ready:
        _check(lib.mpw_qlinear_flags(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), int(bits),
                                     LAYOUTS[layout], M, N, K, y.data_ptr(), PATHS[path],
                                     X_READY | (Y_UNSHARED if y_unshared else 0),
                                     _stream(stream)), "mpw_qlinear_flags")
        return y
    ws, ws_bytes = None, 0
    if use_workspace:
        need = qlinear_workspace_bytes(bits, min(M, 32), N, K, layout) if M <= 32 or path == "gemv" else 0
        if M > 32 and path == "gemv":
            need = max(need, qlinear_workspace_bytes(bits, M % 32 or 32, N, K, layout))
        ws = workspace(need, stream)
        ws_bytes = 0 if ws is None else ws.numel()
    _check(lib.mpw_qlinear_ws(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), int(bits), LAYOUTS[layout],
                              M, N, K, y.data_ptr(), PATHS[path], None if ws is None else ws.data_ptr(),
                              ws_bytes, _stream(stream)), "mpw_qlinear")
    return y


def quantize_pack_groups(W, bits: int, group: int, packed=None, scales=None, nonfinite_flag=None, stream=None):
    """W fp32 [N, K] (CUDA) -> (packed uint8 [N, row_bytes], scales fp32
    [N, ceil(K / group)]): one scale per ``group`` consecutive weights of a
    row (mpw_quantize_pack_groups)."""
    import torch

    _need(W, torch.float32, "W", 2)
    N, K = W.shape
    rb = packed_row_bytes(K, bits)
    G = -(-K // int(group)) if group > 0 else 0
    if packed is None:
        packed = torch.empty((N, max(rb, 16)), dtype=torch.uint8, device=W.device)
    if scales is None:
        scales = torch.empty((N, max(G, 1)), dtype=torch.float32, device=W.device)
    _need(packed, torch.uint8, "packed")
    _need(scales, torch.float32, "scales")
    flag = 0 if nonfinite_flag is None else nonfinite_flag.data_ptr()
    _check(lib.mpw_quantize_pack_groups(W.data_ptr(), N, K, int(bits), int(group), packed.data_ptr(),
                                        scales.data_ptr(), flag, _stream(stream)), "mpw_quantize_pack_groups")
    return packed, scales


def qlinear_groups(x, packed, scales, bits: int, group: int, y=None, layout: str = "canonical", stream=None,
                   x_ready: bool = False, y_unshared: bool = False):
    """y = x @ (q * s_group)^T with group scales [N, ceil(K / group)]
    (mpw_qlinear_groups); x bf16 [M, K] -> y bf16 [M, N].  ``x_ready`` and
    ``y_unshared`` as for qlinear."""
    import torch

    _need(x, torch.bfloat16, "x", 2)
    _need(packed, torch.uint8, "packed", 2)
    _need(scales, torch.float32, "scales", 2)
    M, K = x.shape
    N = packed.shape[0]
    if scales.shape[0] != N or scales.shape[1] != -(-K // int(group)):
        raise ValueError("scales must be [N, ceil(K / group)]")
    if packed.shape[1] != packed_row_bytes(K, bits):
        raise ValueError("packed rows must be exactly packed_row_bytes(K, bits) long")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, "y")
    if y_unshared and not x_ready:
        raise ValueError("y_unshared needs x_ready")
    flags = (X_READY if x_ready else 0) | (Y_UNSHARED if y_unshared else 0)
    _check(lib.mpw_qlinear_groups(x.data_ptr(), packed.data_ptr(), scales.data_ptr(), int(bits), int(group),
                                  LAYOUTS[layout], M, N, K, y.data_ptr(), flags, _stream(stream)),
           "mpw_qlinear_groups")
    return y


def quantize_x_fp8(x, xq=None, sx=None, stream=None):
    """x bf16 [M, K] -> (xq uint8 [M, K] of E4M3 codes, sx fp32 [M]): the
    per-token activations of the FP8 prefill (mpw_quantize_x_fp8)."""
    import torch

    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    if xq is None:
        xq = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty((M,), dtype=torch.float32, device=x.device)
    _need(xq, torch.uint8, "xq", 2)
    _need(sx, torch.float32, "sx", 1)
    _check(lib.mpw_quantize_x_fp8(x.data_ptr(), M, K, xq.data_ptr(), sx.data_ptr(), _stream(stream)),
           "mpw_quantize_x_fp8")
    return xq, sx


def qlinear_fp8(x, packed, scales, bits: int, y=None, layout: str = "canonical", xq=None, sx=None, stream=None):
    """FP8 (E4M3) prefill linear for 4- and 5-bit codes (mpw_qlinear_fp8):
    quantizes x per token unless (xq, sx) are given, then y bf16 [M, N]."""
    import torch

    _need(packed, torch.uint8, "packed", 2)
    _need(scales, torch.float32, "scales", 1)
    if xq is None or sx is None:
        xq, sx = quantize_x_fp8(x, stream=stream)
    M, K = xq.shape
    N = packed.shape[0]
    if packed.shape[1] != packed_row_bytes(K, bits):
        raise ValueError("packed rows must be exactly packed_row_bytes(K, bits) long")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=packed.device)
    _need(y, torch.bfloat16, "y")
    _check(lib.mpw_qlinear_fp8(xq.data_ptr(), sx.data_ptr(), packed.data_ptr(), scales.data_ptr(), int(bits),
                               LAYOUTS[layout], M, N, K, y.data_ptr(), _stream(stream)), "mpw_qlinear_fp8")
    return y


def gather_shards(blocks, world: int, M: int, Nl: int, N: int, y=None, stream=None):
    """Gathered outputs of an N-sharded linear, bf16 [world * M * Nl] rank
    after rank, -> y bf16 [M, N] (mpw_gather_shards; see shard.py)."""
    import torch

    _need(blocks, torch.bfloat16, "blocks")
    if blocks.numel() != world * M * Nl:
        raise ValueError("blocks must hold world * M * Nl values")
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=blocks.device)
    _need(y, torch.bfloat16, "y", 2)
    _check(lib.mpw_gather_shards(blocks.data_ptr(), int(world), int(M), int(Nl), int(N), y.data_ptr(),
                                 _stream(stream)), "mpw_gather_shards")
    return y


ALLOC_MODES = {"native": 0, "full": 1}


def allocate_bits(sensitivity, shapes, budget_bytes: int, mode: str = "full"):
    """Per-matrix bit widths under a byte budget (mpw_allocate_bits, host
    only): sensitivity per matrix, shapes as (N, K) pairs; returns (bits,
    total bytes)."""
    import numpy as np

    sens = np.ascontiguousarray(sensitivity, dtype=np.float64)
    sh = np.ascontiguousarray(shapes, dtype=np.int64).reshape(-1, 2)
    if sens.ndim != 1 or sens.shape[0] != sh.shape[0]:
        raise ValueError("one sensitivity per (N, K) shape")
    n_rows = np.ascontiguousarray(sh[:, 0])
    k_cols = np.ascontiguousarray(sh[:, 1])
    bits = np.zeros(sens.shape[0], dtype=np.int32)
    total = ctypes.c_uint64(0)
    _check(lib.mpw_allocate_bits(sens.ctypes.data, n_rows.ctypes.data, k_cols.ctypes.data, sens.shape[0],
                                 int(budget_bytes), ALLOC_MODES[mode], bits.ctypes.data, ctypes.byref(total)),
           "mpw_allocate_bits")
    return bits.tolist(), int(total.value)


def allocation_frontier(sensitivity, shapes, mode: str = "full"):
    """(bytes, total loss) after each upgrade of the unbounded water filling
    (mpw_allocate_frontier, host only)."""
    import numpy as np

    sens = np.ascontiguousarray(sensitivity, dtype=np.float64)
    sh = np.ascontiguousarray(shapes, dtype=np.int64).reshape(-1, 2)
    if sens.ndim != 1 or sens.shape[0] != sh.shape[0]:
        raise ValueError("one sensitivity per (N, K) shape")
    n_rows = np.ascontiguousarray(sh[:, 0])
    k_cols = np.ascontiguousarray(sh[:, 1])
    n = ctypes.c_int64(0)
    _check(lib.mpw_allocate_frontier(sens.ctypes.data, n_rows.ctypes.data, k_cols.ctypes.data, sens.shape[0],
                                     ALLOC_MODES[mode], None, None, 0, ctypes.byref(n)), "mpw_allocate_frontier")
    nbytes = np.zeros(n.value, dtype=np.uint64)
    loss = np.zeros(n.value, dtype=np.float64)
    _check(lib.mpw_allocate_frontier(sens.ctypes.data, n_rows.ctypes.data, k_cols.ctypes.data, sens.shape[0],
                                     ALLOC_MODES[mode], nbytes.ctypes.data, loss.ctypes.data, n.value,
                                     ctypes.byref(n)), "mpw_allocate_frontier")
    return [int(v) for v in nbytes], loss.tolist()


@dataclass
class Linear:
    """One quantized linear of a recipe stack (see mpw_linear in mpw.h)."""
    packed: object
    scales: object
    N: int
    K: int
    bits: int
    in_slot: int
    out_slot: int
    norm_input: bool = False
    layout: str = "canonical"


def save_packed(path: str, matrices) -> None:
    """Write packed matrices to a file (mpw_file_write).  ``matrices``: items
    (packed uint8 [N, row_bytes], scales fp32 [N], bits, K, layout), tensors
    on any device (copied to the host)."""
    import torch

    keep = []
    arr = (_FileMatrix * len(matrices))()
    for i, (packed, scales, bits, K, layout) in enumerate(matrices):
        p = packed.detach().to("cpu").contiguous()
        s_ = scales.detach().to("cpu", torch.float32).contiguous()
        if p.dtype != torch.uint8 or p.dim() != 2 or p.shape[1] != packed_row_bytes(K, bits):
            raise ValueError("packed rows must be uint8 [N, packed_row_bytes(K, bits)]")
        if s_.dim() != 1 or s_.shape[0] != p.shape[0]:
            raise ValueError("scales must have one entry per packed row")
        keep += [p, s_]
        arr[i] = _FileMatrix(p.shape[0], int(K), int(bits), LAYOUTS[layout], p.data_ptr(), s_.data_ptr())
    _check(lib.mpw_file_write(os.fsencode(path), arr, len(matrices)), "mpw_file_write")


def load_packed(path: str, device=None):
    """Read every matrix of a file written by save_packed (mpw_file_read
    checks the checksums): a list of dicts with packed, scales, bits, K, N,
    layout; tensors on ``device`` (host if None)."""
    import torch

    n = ctypes.c_int64(0)
    _check(lib.mpw_file_count(os.fsencode(path), ctypes.byref(n)), "mpw_file_count")
    out = []
    for i in range(n.value):
        N, K, b, lay = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int32(), ctypes.c_int32()
        _check(lib.mpw_file_info(os.fsencode(path), i, ctypes.byref(N), ctypes.byref(K), ctypes.byref(b),
                                 ctypes.byref(lay)), "mpw_file_info")
        packed = torch.empty((N.value, packed_row_bytes(K.value, b.value)), dtype=torch.uint8)
        scales = torch.empty((N.value,), dtype=torch.float32)
        _check(lib.mpw_file_read(os.fsencode(path), i, packed.data_ptr(), scales.data_ptr()), "mpw_file_read")
        layout = [k for k, v in LAYOUTS.items() if v == lay.value][0]
        if device is not None:
            packed, scales = packed.to(device), scales.to(device)
        out.append({"packed": packed, "scales": scales, "bits": b.value, "K": K.value, "N": N.value,
                    "layout": layout})
    return out


def recipe_plan(layers, slots, M: int):
    """The MPW_QLINEAR_* flags recipe_run launches each linear with (host
    only; slot addresses are compared, never read)."""
    arr = (_Linear * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = _Linear(L.packed.data_ptr(), L.scales.data_ptr(), int(L.N), int(L.K), int(L.bits),
                         int(L.in_slot), int(L.out_slot), int(bool(L.norm_input)), LAYOUTS[L.layout], 0)
    ptrs = (ctypes.c_void_p * len(slots))(*[s.data_ptr() for s in slots])
    flags = (ctypes.c_uint32 * len(layers))()
    _check(lib.mpw_recipe_plan(arr, len(layers), ptrs, len(slots), int(M), flags), "mpw_recipe_plan")
    return list(flags)


def _addr(t) -> int:
    return t if isinstance(t, int) else t.data_ptr()


def _linear_array(layers):
    arr = (_Linear * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = _Linear(_addr(L.packed), _addr(L.scales), int(L.N), int(L.K), int(L.bits),
                         int(L.in_slot), int(L.out_slot), int(bool(L.norm_input)), LAYOUTS[L.layout], 0)
    return arr


def pass_dependencies(layers, slots, M: int = 1):
    """For every linear, the earlier linears the planned pass makes it wait
    for (mpw_pass_dependencies; host only, slot addresses are compared, never
    read).  ``slots`` may be tensors or plain integer addresses."""
    arr = _linear_array(layers)
    addr = [s if isinstance(s, int) else s.data_ptr() for s in slots]
    ptrs = (ctypes.c_void_p * len(slots))(*addr)
    offsets = (ctypes.c_int32 * (len(layers) + 1))()
    st = lib.mpw_pass_dependencies(arr, len(layers), ptrs, len(slots), int(M), offsets, None, 0)
    need = offsets[len(layers)]
    if st != MPW_OK and not (st == MPW_E_INVALID_ARG and need > 0):
        _check(st, "mpw_pass_dependencies")
    deps = (ctypes.c_int32 * max(need, 1))()
    _check(lib.mpw_pass_dependencies(arr, len(layers), ptrs, len(slots), int(M), offsets, deps, need),
           "mpw_pass_dependencies")
    return [list(deps[offsets[i]:offsets[i + 1]]) for i in range(len(layers))]


class Pass:
    """A decode pass planned once and run as one persistent kernel per call
    (mpw_pass_create / mpw_pass_run).  Holds references to the layers' and
    slots' tensors, whose pointers the plan records.  Raises MPWError with
    MPW_E_UNSUPPORTED when the pass does not take these linears."""

    def __init__(self, layers, slots, M: int = 1):
        arr = _linear_array(layers)
        ptrs = (ctypes.c_void_p * len(slots))(*[s.data_ptr() for s in slots])
        h = ctypes.c_void_p()
        _check(lib.mpw_pass_create(arr, len(layers), ptrs, len(slots), int(M), ctypes.byref(h)), "mpw_pass_create")
        self._h = h
        self._keep = (list(layers), list(slots))

    def run(self, stream=None) -> None:
        if not self._h:
            raise ValueError("pass already closed")
        _check(lib.mpw_pass_run(self._h, _stream(stream)), "mpw_pass_run")

    def info(self) -> dict:
        v = (ctypes.c_int64 * 4)()
        _check(lib.mpw_pass_info(self._h, v), "mpw_pass_info")
        return {"grid": v[0], "stages": v[1], "items": v[2], "smem_bytes": v[3]}

    def close(self) -> None:
        """Free the plan (the caller makes sure its last run has completed)."""
        if self._h:
            lib.mpw_pass_destroy(self._h)
            self._h = ctypes.c_void_p()
            self._keep = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def recipe_run(layers, slots, M: int, stream=None, use_workspace: bool = False):
    """Launch every linear of ``layers`` in order (one kernel each)."""
    arr = (_Linear * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = _Linear(L.packed.data_ptr(), L.scales.data_ptr(), int(L.N), int(L.K), int(L.bits),
                         int(L.in_slot), int(L.out_slot), int(bool(L.norm_input)), LAYOUTS[L.layout], 0)
    ptrs = (ctypes.c_void_p * len(slots))(*[s.data_ptr() for s in slots])
    ws, ws_bytes = None, 0
    if use_workspace:
        ws = workspace(int(lib.mpw_recipe_workspace_bytes(arr, len(layers), int(M))), stream)
        ws_bytes = 0 if ws is None else ws.numel()
    _check(lib.mpw_recipe_run_ws(arr, len(layers), ptrs, len(slots), int(M),
                                 None if ws is None else ws.data_ptr(), ws_bytes, _stream(stream)),
           "mpw_recipe_run")


def device_error() -> int:
    """Synchronise; return and clear the library's device-side error word."""
    code = ctypes.c_int32(0)
    st = lib.mpw_device_error(ctypes.byref(code))
    if st not in (MPW_OK, MPW_E_TIMEOUT):
        _check(st, "mpw_device_error")
    return int(code.value)
