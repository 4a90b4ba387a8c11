"""Scaled FP8 casting on NVIDIA B200 (sm_100a): Python binding of libfp8q.

The compute path is the C-ABI library ``libfp8q.so`` (hand-written CUDA
kernels, declared in ``include/fp8q.h``).  This module only marshals
arguments: it turns torch tensors into device pointers, sizes, dtype codes and
the current CUDA stream, checks that output buffers are large enough and on
the same device, and raises :class:`Fp8qError` on a non-zero status.  torch
is used for device memory and streams only.  There is no CPU fallback: if the
library is missing or a tensor is not on a CUDA device, the call fails.

Entry points with the C names (caller-provided outputs, nothing allocated):
    fp8q_per_token_group_quant, fp8q_cast_per_channel, fp8q_cast_per_tensor,
    fp8q_block_dequant, fp8q_block_dequant_grouped, fp8q_cast_from_fp8

fp8-compressed collectives (ColossalAI all_gather_fp8 / all_to_all_fp8 /
all_to_all_single_fp8): each rank packs [scale_inv | fp8 payload] records
with libfp8q, torch.distributed moves the bytes, and libfp8q dequantises
every received record; no arithmetic runs outside the library.

fp8 matrix products on the tensor cores (tcgen05):
    fp8q_scaled_mm            ColossalAI _LinearFp8.forward (torch._scaled_mm,
                              per-tensor scales)
    fp8q_scaled_mm_blockwise  DeepEP per-token activations x DeepSeek-V3
                              128 x 128 block-scaled weight

Allocating helpers named after the functions on the pages:
    per_token_cast_to_fp8   (DeepEP "5 Utils")
    per_token_cast_back     (DeepEP "5 Utils", the named inverse)
    cast_to_fp8, cast_from_fp8   (ColossalAI colossalai/quantization/fp8.py)
    weight_dequant          (DeepSeek-V3 fp8_cast_bf16 blog)
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Sequence, Tuple

import torch

__all__ = [
    "E4M3FN", "E5M2", "F32", "F16", "BF16",
    "GRAN_TENSOR", "GRAN_ROW", "GRAN_GROUP", "GRAN_BLOCK", "SCALE_IEEE", "SCALE_TORCH",
    "Fp8qError", "lib", "lib_path",
    "fp8q_per_token_group_quant", "fp8q_cast_per_channel", "fp8q_cast_per_tensor",
    "fp8q_per_token_group_quant_ex", "fp8q_cast_per_channel_ex", "fp8q_cast_per_tensor_ex",
    "fp8q_cast_per_tensor_workspace_bytes", "fp8q_cast_per_tensor_noalloc", "fp8q_block_dequant", "fp8q_block_dequant_grouped",
    "fp8q_cast_from_fp8", "fp8q_cast_pipeline", "fp8q_cast_from_pipeline", "fp8q_status_string", "fp8q_version",
    "fp8q_tensor_amax", "fp8q_cast_per_tensor_with_amax", "allreduce_amax_bits", "cast_to_fp8_sharded",
    "per_token_cast_to_fp8", "per_token_cast_back", "cast_to_fp8", "cast_from_fp8", "weight_dequant",
    "cast_to_fp8_pipeline", "cast_from_fp8_pipeline",
    "RECORD_HEADER_BYTES", "record_bytes", "fp8q_record_bytes", "fp8q_pack_record", "fp8q_unpack_records",
    "RECORD_PACKED4", "RECORD_ALIGNED16", "fp8q_record_bytes_ex", "fp8q_pack_record_ex", "fp8q_unpack_records_ex",
    "exchange_records", "exchange_records_all_to_all", "exchange_payload_all_to_all", "all_gather_fp8", "all_to_all_fp8", "all_to_all_single_fp8",
    "fp8q_scaled_mm", "fp8q_scaled_mm_blockwise", "scaled_mm", "scaled_mm_blockwise", "linear_fp8",
    "linear_fp8_blockwise", "fp8q_transpose_fp8", "fp8q_sum_rows", "transpose_fp8", "fp8q_scaled_mm_ex",
    "K_MAJOR", "MN_MAJOR", "fp8q_scaled_mm_wait_test",
]

E4M3FN, E5M2 = 0, 1
F32, F16, BF16 = 0, 1, 2
GRAN_TENSOR, GRAN_ROW, GRAN_GROUP, GRAN_BLOCK = 0, 1, 2, 3
SCALE_IEEE, SCALE_TORCH = 0, 1
K_MAJOR, MN_MAJOR = 0, 1
RECORD_PACKED4, RECORD_ALIGNED16 = 4, 16     # fp8q_record_layout: the page's 4-byte header / 16-byte aligned

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libfp8q.so")

_DTYPE_CODE = {torch.float32: F32, torch.float16: F16, torch.bfloat16: BF16}
_CODE_DTYPE = {v: k for k, v in _DTYPE_CODE.items()}
_FP8_DTYPES = {torch.float8_e4m3fn: E4M3FN, torch.float8_e5m2: E5M2}
_FMT_DTYPE = {E4M3FN: torch.float8_e4m3fn, E5M2: torch.float8_e5m2}


class Fp8qError(RuntimeError):
    """A libfp8q call returned a non-zero fp8q_status."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {fp8q_status_string(status)}")


class _BlockDesc(ctypes.Structure):
    _fields_ = [("w", ctypes.c_void_p), ("scale_inv", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("M", ctypes.c_int64), ("N", ctypes.c_int64)]


_lock = threading.Lock()
_lib: Optional[ctypes.CDLL] = None


def lib_path() -> str:
    return _LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libfp8q.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise ImportError(
                    f"libfp8q.so not found at {_LIB_PATH}; build it with "
                    "`python -m dequantisation_fp8q_token_b200.build` (needs nvcc)")
            L = ctypes.CDLL(_LIB_PATH)
            p, i64, i32, st = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int
            L.fp8q_status_string.restype = ctypes.c_char_p
            L.fp8q_status_string.argtypes = [st]
            L.fp8q_version.restype = i32
            L.fp8q_version.argtypes = []
            L.fp8q_per_token_group_quant.restype = st
            L.fp8q_per_token_group_quant.argtypes = [p, i32, i64, i64, i32, i32, p, p, p]
            L.fp8q_cast_per_channel.restype = st
            L.fp8q_cast_per_channel.argtypes = [p, i32, i64, i64, i32, p, p, p]
            L.fp8q_cast_per_tensor_workspace_bytes.restype = ctypes.c_size_t
            L.fp8q_cast_per_tensor_workspace_bytes.argtypes = []
            L.fp8q_cast_per_tensor.restype = st
            L.fp8q_cast_per_tensor.argtypes = [p, i32, i64, i32, p, p, p, ctypes.c_size_t, p]
            L.fp8q_block_dequant.restype = st
            L.fp8q_block_dequant.argtypes = [p, i32, i64, i64, p, i32, i32, p, p]
            L.fp8q_block_dequant_grouped.restype = st
            L.fp8q_block_dequant_grouped.argtypes = [ctypes.POINTER(_BlockDesc), i32, i32, i32, i32, p]
            L.fp8q_cast_from_fp8.restype = st
            L.fp8q_cast_from_fp8.argtypes = [p, i32, i64, i64, p, i32, i32, i32, p, p]
            L.fp8q_tensor_amax.restype = st
            L.fp8q_tensor_amax.argtypes = [p, i32, i64, p, p, ctypes.c_size_t, p]
            L.fp8q_cast_per_tensor_with_amax.restype = st
            L.fp8q_cast_per_tensor_with_amax.argtypes = [p, i32, i64, i32, p, p, p, i32, p]
            L.fp8q_cast_pipeline.restype = st
            L.fp8q_cast_pipeline.argtypes = [p, i32, i64, p, p, p, p, ctypes.c_size_t, i32, p]
            L.fp8q_cast_from_pipeline.restype = st
            L.fp8q_cast_from_pipeline.argtypes = [p, i64, p, p, i32, p, p]
            L.fp8q_per_token_group_quant_ex.restype = st
            L.fp8q_per_token_group_quant_ex.argtypes = [p, i32, i64, i64, i32, i32, p, p, i32, p]
            L.fp8q_cast_per_channel_ex.restype = st
            L.fp8q_cast_per_channel_ex.argtypes = [p, i32, i64, i64, i32, p, p, i32, p]
            L.fp8q_cast_per_tensor_ex.restype = st
            L.fp8q_cast_per_tensor_ex.argtypes = [p, i32, i64, i32, p, p, p, ctypes.c_size_t, i32, p]
            L.fp8q_record_bytes.restype = ctypes.c_size_t
            L.fp8q_record_bytes.argtypes = [i64]
            L.fp8q_pack_record.restype = st
            L.fp8q_pack_record.argtypes = [p, i32, i64, i32, p, p, ctypes.c_size_t, i32, p]
            L.fp8q_unpack_records.restype = st
            L.fp8q_unpack_records.argtypes = [p, i32, i64, i32, i32, p, p]
            L.fp8q_record_bytes_ex.restype = ctypes.c_size_t
            L.fp8q_record_bytes_ex.argtypes = [i64, i32]
            L.fp8q_pack_record_ex.restype = st
            L.fp8q_pack_record_ex.argtypes = [p, i32, i64, i32, p, p, ctypes.c_size_t, i32, i32, p]
            L.fp8q_unpack_records_ex.restype = st
            L.fp8q_unpack_records_ex.argtypes = [p, i32, i64, i32, i32, p, i32, p]
            L.fp8q_scaled_mm.restype = st
            L.fp8q_scaled_mm.argtypes = [p, i32, p, i32, i64, i64, i64, p, p, p, i32, p, p, p]
            L.fp8q_scaled_mm_wait_test.restype = st
            L.fp8q_scaled_mm_wait_test.argtypes = [p, p, i64, i64, i64, p, p, p, p, ctypes.c_uint64, i32, p]
            L.fp8q_scaled_mm_blockwise_wait_test.restype = st
            L.fp8q_scaled_mm_blockwise_wait_test.argtypes = [p, p, p, p, i64, i64, i64, p, p, ctypes.c_uint64, i32, p]
            L.fp8q_scaled_mm_ex.restype = st
            L.fp8q_scaled_mm_ex.argtypes = [p, i32, i32, p, i32, i32, i64, i64, i64, p, p, p, i32, p, p, p]
            L.fp8q_transpose_fp8.restype = st
            L.fp8q_transpose_fp8.argtypes = [p, i64, i64, p, i64, p]
            L.fp8q_sum_rows.restype = st
            L.fp8q_sum_rows.argtypes = [p, i32, i64, i64, p, p]
            L.fp8q_scaled_mm_blockwise.restype = st
            L.fp8q_scaled_mm_blockwise.argtypes = [p, i32, p, p, i32, p, i64, i64, i64, p, i32, p, p, p]
            _lib = L
    return _lib


def fp8q_status_string(status: int) -> str:
    return lib().fp8q_status_string(int(status)).decode()


def fp8q_version() -> int:
    return int(lib().fp8q_version())


def fp8q_cast_per_tensor_workspace_bytes() -> int:
    return int(lib().fp8q_cast_per_tensor_workspace_bytes())


# ---------------------------------------------------------------------------
# marshalling helpers
# ---------------------------------------------------------------------------
def _check(status: int, what: str) -> None:
    if status != 0:
        raise Fp8qError(status, what)


def _dev_ptr(t: Optional[torch.Tensor], name: str, device=None) -> Optional[int]:
    """Device pointer of a contiguous CUDA tensor (None for an empty tensor)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (libfp8q takes device pointers)")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


# The current device and its current stream's raw handle, read the cheap way where this torch
# build has it (the public torch.cuda.current_stream builds a Stream object: ~2 us of the ~12 us a
# call costs on the host, against ~0.1 us for the raw handle).
_current_device = getattr(torch._C, "_cuda_getDevice", None) or torch.cuda.current_device
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device) -> int:
    """The raw stream handle for a call on `device`.  The library sizes its launches (and picks
    the allocation-free cast's scratch) from the CURRENT device, so a tensor on any other device
    is refused before anything is enqueued."""
    cur = None
    if device is not None and device.type == "cuda":
        cur = _current_device()
        if device.index is not None and device.index != cur:
            raise ValueError(f"tensors are on {device} but the current device is cuda:{cur}; "
                             f"call under torch.cuda.device({device.index})")
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(cur if cur is not None else _current_device())
        return torch.cuda.current_stream(device).cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _dtype_code(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DTYPE_CODE:
        raise TypeError(f"{name}: only float32, float16 and bfloat16 are allowed, got {t.dtype}")
    return _DTYPE_CODE[t.dtype]


def _is_byte_tensor(t: torch.Tensor) -> bool:
    return t.dtype == torch.uint8 or t.dtype in _FP8_DTYPES


def _need(t: torch.Tensor, numel: int, name: str, byte: bool = False, dtype=None) -> None:
    if byte and not _is_byte_tensor(t):
        raise TypeError(f"{name} must be uint8 or a float8 dtype, got {t.dtype}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements, needs {numel}")


def _rule_of(rule) -> int:
    if isinstance(rule, str):
        return {"ieee": SCALE_IEEE, "torch": SCALE_TORCH}[rule]
    return int(rule)


def _fmt_of(fmt) -> int:
    if isinstance(fmt, str):
        return {"e4m3": E4M3FN, "e4m3fn": E4M3FN, "e5m2": E5M2}[fmt]
    if isinstance(fmt, torch.dtype):
        return _FP8_DTYPES[fmt]
    return int(fmt)


# ---------------------------------------------------------------------------
# C entry points (caller-provided outputs)
# ---------------------------------------------------------------------------
def fp8q_per_token_group_quant(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                               group: int = 128, fmt=E4M3FN, stream=None) -> None:
    """DeepEP per_token_cast_to_fp8 into q[m, n] (uint8/fp8) and scale_inv[m, n/group] (fp32)."""
    fp8q_per_token_group_quant_ex(x, q, scale_inv, group, fmt, SCALE_IEEE, stream)


def fp8q_per_token_group_quant_ex(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                                  group: int = 128, fmt=E4M3FN, rule=SCALE_IEEE, stream=None) -> None:
    """fp8q_per_token_group_quant with a scale rule ("ieee" or "torch")."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D [m, n]")
    m, n = x.shape
    dev = x.device
    if group > 0 and n % group == 0:
        _need(q, m * n, "q", byte=True)
        _need(scale_inv, m * (n // group), "scale_inv", dtype=torch.float32)
    _check(lib().fp8q_per_token_group_quant_ex(
        _dev_ptr(x, "x"), _dtype_code(x, "x"), m, n, group, _fmt_of(fmt),
        _dev_ptr(q, "q", dev), _dev_ptr(scale_inv, "scale_inv", dev), _rule_of(rule), _stream(stream, dev)),
        "fp8q_per_token_group_quant")


def fp8q_cast_per_channel(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                          fmt=E4M3FN, stream=None) -> None:
    """ColossalAI cast_to_fp8(per_channel_scale=True): one scale per row of x[rows, cols]."""
    fp8q_cast_per_channel_ex(x, q, scale_inv, fmt, SCALE_IEEE, stream)


def fp8q_cast_per_channel_ex(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                             fmt=E4M3FN, rule=SCALE_IEEE, stream=None) -> None:
    """fp8q_cast_per_channel with a scale rule ("ieee" or "torch")."""
    x2 = x.reshape(-1, x.shape[-1]) if x.dim() != 2 else x
    rows, cols = x2.shape
    dev = x.device
    _need(q, rows * cols, "q", byte=True)
    _need(scale_inv, max(rows, 1), "scale_inv", dtype=torch.float32)
    _check(lib().fp8q_cast_per_channel_ex(
        _dev_ptr(x2, "x"), _dtype_code(x, "x"), rows, cols, _fmt_of(fmt),
        _dev_ptr(q, "q", dev), _dev_ptr(scale_inv, "scale_inv", dev), _rule_of(rule), _stream(stream, dev)),
        "fp8q_cast_per_channel")


def fp8q_cast_per_tensor(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                         workspace: torch.Tensor, fmt=E4M3FN, stream=None) -> None:
    """ColossalAI cast_to_fp8 per-tensor branch; workspace of fp8q_cast_per_tensor_workspace_bytes()."""
    fp8q_cast_per_tensor_ex(x, q, scale_inv, workspace, fmt, SCALE_IEEE, stream)


def fp8q_cast_per_tensor_ex(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                            workspace: torch.Tensor, fmt=E4M3FN, rule=SCALE_IEEE, stream=None) -> None:
    """fp8q_cast_per_tensor with a scale rule ("ieee" or "torch")."""
    dev = x.device
    n = x.numel()
    _need(q, n, "q", byte=True)
    _need(scale_inv, 1, "scale_inv", dtype=torch.float32)
    wbytes = workspace.numel() * workspace.element_size()
    _check(lib().fp8q_cast_per_tensor_ex(
        _dev_ptr(x, "x"), _dtype_code(x, "x"), n, _fmt_of(fmt), _dev_ptr(q, "q", dev),
        _dev_ptr(scale_inv, "scale_inv", dev), _dev_ptr(workspace, "workspace", dev), wbytes,
        _rule_of(rule), _stream(stream, dev)), "fp8q_cast_per_tensor")


def fp8q_cast_per_tensor_noalloc(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor,
                                 fmt=E4M3FN, stream=None) -> None:
    """Per-tensor cast with the library's own static scratch (no workspace argument).

    For callers that cannot allocate device memory.  Calls that overlap on the
    GPU share the scratch and race; the first call on a device sets it up."""
    L = lib()
    f = L.fp8q_cast_per_tensor_noalloc
    if f.argtypes is None:
        p = ctypes.c_void_p
        f.restype = ctypes.c_int
        f.argtypes = [p, ctypes.c_int, ctypes.c_int64, ctypes.c_int, p, p, p]
    dev = x.device
    n = x.numel()
    _need(q, n, "q", byte=True)
    _need(scale_inv, 1, "scale_inv", dtype=torch.float32)
    _check(f(_dev_ptr(x, "x"), _dtype_code(x, "x"), n, _fmt_of(fmt), _dev_ptr(q, "q", dev),
             _dev_ptr(scale_inv, "scale_inv", dev), _stream(stream, dev)), "fp8q_cast_per_tensor_noalloc")


def fp8q_tensor_amax(x: torch.Tensor, amax_bits: torch.Tensor, workspace: torch.Tensor, stream=None) -> None:
    """amax_bits[0] (int32) = fp32 bit pattern of max |x| over this tensor (a shard)."""
    dev = x.device
    _need(amax_bits, 1, "amax_bits", dtype=torch.int32)
    wbytes = workspace.numel() * workspace.element_size()
    _check(lib().fp8q_tensor_amax(_dev_ptr(x, "x"), _dtype_code(x, "x"), x.numel(),
                                  _dev_ptr(amax_bits, "amax_bits", dev), _dev_ptr(workspace, "workspace", dev),
                                  wbytes, _stream(stream, dev)), "fp8q_tensor_amax")


def fp8q_cast_per_tensor_with_amax(x: torch.Tensor, amax_bits: torch.Tensor, q: torch.Tensor,
                                   scale_inv: torch.Tensor, fmt=E4M3FN, rule=SCALE_IEEE, stream=None) -> None:
    """Per-tensor cast of x with the amax given as fp32 bits in amax_bits[0] (device int32)."""
    dev = x.device
    n = x.numel()
    _need(q, n, "q", byte=True)
    _need(scale_inv, 1, "scale_inv", dtype=torch.float32)
    _need(amax_bits, 1, "amax_bits", dtype=torch.int32)
    _check(lib().fp8q_cast_per_tensor_with_amax(
        _dev_ptr(x, "x"), _dtype_code(x, "x"), n, _fmt_of(fmt), _dev_ptr(amax_bits, "amax_bits", dev),
        _dev_ptr(q, "q", dev), _dev_ptr(scale_inv, "scale_inv", dev), _rule_of(rule), _stream(stream, dev)),
        "fp8q_cast_per_tensor_with_amax")


def allreduce_amax_bits(amax_bits: torch.Tensor, group=None) -> None:
    """The exchange step of a sharded per-tensor cast: an integer MAX of the
    ranks' amax bit patterns (int32, sign bit clear), in place.  Integer max
    orders fp32 magnitudes and keeps a NaN from any rank, whatever the
    backend's float max would do with NaN.  A no-op without a process group."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax_bits, op=dist.ReduceOp.MAX, group=group)


def cast_to_fp8_sharded(x_local: torch.Tensor, fp8_format: str = "e4m3", group=None,
                        rule=SCALE_IEEE) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-tensor cast of a tensor whose shards live on the ranks of `group`:
    local amax, a 4-byte all-reduce (MAX) across ranks, then the cast with the
    global amax.  Each rank gets its slice of the one-tensor cast's bytes and
    the shared scale_inv."""
    f = _fmt_of(fp8_format)
    dev = x_local.device
    amax = torch.empty((1,), dtype=torch.int32, device=dev)
    ws = _workspace(dev)
    fp8q_tensor_amax(x_local, amax, ws)
    allreduce_amax_bits(amax, group)
    q = torch.empty(x_local.shape, dtype=_FMT_DTYPE[f], device=dev)
    s = torch.empty((1,), dtype=torch.float32, device=dev)
    fp8q_cast_per_tensor_with_amax(x_local, amax, q, s, f, rule)
    return q, s


def fp8q_cast_pipeline(x: torch.Tensor, q: torch.Tensor, scale_inv: torch.Tensor, fmt_tag: torch.Tensor,
                       workspace: torch.Tensor, rule=SCALE_IEEE, stream=None) -> None:
    """ColossalAI cast_to_fp8_pipeline: format chosen by the amax, written to fmt_tag (int32 [1])."""
    dev = x.device
    n = x.numel()
    _need(q, n, "q", byte=True)
    _need(scale_inv, 1, "scale_inv", dtype=torch.float32)
    _need(fmt_tag, 1, "fmt_tag", dtype=torch.int32)
    wbytes = workspace.numel() * workspace.element_size()
    _check(lib().fp8q_cast_pipeline(
        _dev_ptr(x, "x"), _dtype_code(x, "x"), n, _dev_ptr(q, "q", dev), _dev_ptr(scale_inv, "scale_inv", dev),
        _dev_ptr(fmt_tag, "fmt_tag", dev), _dev_ptr(workspace, "workspace", dev), wbytes, _rule_of(rule),
        _stream(stream, dev)), "fp8q_cast_pipeline")


def fp8q_cast_from_pipeline(q: torch.Tensor, scale_inv: torch.Tensor, fmt_tag: torch.Tensor, y: torch.Tensor,
                            stream=None) -> None:
    """ColossalAI cast_from_fp8_pipeline into y (its dtype), reading the format tag on the device."""
    dev = q.device
    n = q.numel()
    _need(q, n, "q", byte=True)
    _need(y, n, "y")
    _need(scale_inv, 1, "scale_inv", dtype=torch.float32)
    _need(fmt_tag, 1, "fmt_tag", dtype=torch.int32)
    _check(lib().fp8q_cast_from_pipeline(
        _dev_ptr(q, "q"), n, _dev_ptr(scale_inv, "scale_inv", dev), _dev_ptr(fmt_tag, "fmt_tag", dev),
        _dtype_code(y, "y"), _dev_ptr(y, "y", dev), _stream(stream, dev)), "fp8q_cast_from_pipeline")


def fp8q_block_dequant(w: torch.Tensor, scale_inv: torch.Tensor, y: torch.Tensor, block: int = 128,
                       fmt=E4M3FN, stream=None) -> None:
    """DeepSeek-V3 weight_dequant of w[M, N] with scale_inv[ceil(M/B), ceil(N/B)] into y[M, N]."""
    if w.dim() != 2:
        raise ValueError("w must be 2-D [M, N]")
    M, N = w.shape
    dev = w.device
    if block > 0:
        _need(w, M * N, "w", byte=True)
        _need(scale_inv, -(-M // block) * -(-N // block), "scale_inv", dtype=torch.float32)
        _need(y, M * N, "y")
    _check(lib().fp8q_block_dequant(
        _dev_ptr(w, "w"), _fmt_of(fmt), M, N, _dev_ptr(scale_inv, "scale_inv", dev), block,
        _dtype_code(y, "y"), _dev_ptr(y, "y", dev), _stream(stream, dev)), "fp8q_block_dequant")


def fp8q_block_dequant_grouped(ws: Sequence[torch.Tensor], scale_invs: Sequence[torch.Tensor],
                               ys: Sequence[torch.Tensor], block: int = 128, fmt=E4M3FN,
                               stream=None) -> None:
    """Many block dequantisations in one launch (shared block, format and output dtype)."""
    n = len(ws)
    if not (len(scale_invs) == len(ys) == n):
        raise ValueError("ws, scale_invs and ys must have the same length")
    if n == 0:
        return
    dev = ws[0].device
    yt = _dtype_code(ys[0], "y")
    arr = (_BlockDesc * n)()
    for i, (w, s, y) in enumerate(zip(ws, scale_invs, ys)):
        if w.dim() != 2:
            raise ValueError("each w must be 2-D")
        M, N = w.shape
        if _dtype_code(y, "y") != yt:
            raise TypeError("all outputs must share one dtype")
        if block > 0:
            _need(w, M * N, "w", byte=True)
            _need(s, -(-M // block) * -(-N // block), "scale_inv", dtype=torch.float32)
            _need(y, M * N, "y")
        arr[i] = _BlockDesc(_dev_ptr(w, "w", dev), _dev_ptr(s, "scale_inv", dev), _dev_ptr(y, "y", dev), M, N)
    _check(lib().fp8q_block_dequant_grouped(arr, n, _fmt_of(fmt), block, yt, _stream(stream, dev)),
           "fp8q_block_dequant_grouped")


def _granule_count(gran: int, rows: int, cols: int, gb: int) -> int:
    if gran == GRAN_TENSOR:
        return 1
    if gran == GRAN_ROW:
        return rows
    if gran == GRAN_GROUP:
        return rows * (cols // gb) if gb > 0 else 0
    return -(-rows // gb) * -(-cols // gb) if gb > 0 else 0


def fp8q_cast_from_fp8(q: torch.Tensor, scale_inv: torch.Tensor, y: torch.Tensor, gran: int,
                       group_or_block: int = 0, fmt=None, stream=None) -> None:
    """ColossalAI cast_from_fp8 / DeepEP per_token_cast_back into y (dtype of y)."""
    if fmt is None:
        fmt = _FP8_DTYPES.get(q.dtype, E4M3FN)
    q2 = q.reshape(-1, q.shape[-1]) if q.dim() != 2 else q
    rows, cols = q2.shape if q.dim() > 0 else (1, 1)
    dev = q.device
    _need(q, rows * cols, "q", byte=True)
    _need(y, rows * cols, "y")
    if gran in (GRAN_TENSOR, GRAN_ROW, GRAN_GROUP, GRAN_BLOCK):
        _need(scale_inv, _granule_count(gran, rows, cols, group_or_block), "scale_inv", dtype=torch.float32)
    _check(lib().fp8q_cast_from_fp8(
        _dev_ptr(q2, "q"), _fmt_of(fmt), rows, cols, _dev_ptr(scale_inv, "scale_inv", dev), gran,
        group_or_block, _dtype_code(y, "y"), _dev_ptr(y, "y", dev), _stream(stream, dev)),
        "fp8q_cast_from_fp8")


# ---------------------------------------------------------------------------
# allocating helpers named after the pages' functions
# ---------------------------------------------------------------------------
_ws_cache = {}


def _workspace(device: torch.device) -> torch.Tensor:
    key = (device.type, device.index)
    w = _ws_cache.get(key)
    if w is None:
        w = torch.empty(fp8q_cast_per_tensor_workspace_bytes(), dtype=torch.uint8, device=device)
        _ws_cache[key] = w
    return w


def per_token_cast_to_fp8(x: torch.Tensor, group: int = 128, fmt=E4M3FN, rule=SCALE_IEEE
                          ) -> Tuple[torch.Tensor, torch.Tensor]:
    """DeepEP per_token_cast_to_fp8: returns (q [m, n] float8, scale_inv [m, n/group] fp32).
    rule="torch" reproduces the bytes torch itself computes for the page's code on a GPU."""
    m, n = x.shape
    f = _fmt_of(fmt)
    q = torch.empty((m, n), dtype=_FMT_DTYPE[f], device=x.device)
    s = torch.empty((m, n // group if group > 0 else 0), dtype=torch.float32, device=x.device)
    fp8q_per_token_group_quant_ex(x, q, s, group, f, rule)
    return q, s


def per_token_cast_back(q: torch.Tensor, scale_inv: torch.Tensor, dtype=torch.bfloat16,
                        group: int = 128) -> torch.Tensor:
    """Inverse of per_token_cast_to_fp8: y = dtype(scale_inv[r, c/group] * float(q))."""
    y = torch.empty(q.shape, dtype=dtype, device=q.device)
    fp8q_cast_from_fp8(q, scale_inv, y, GRAN_GROUP, group)
    return y


def cast_to_fp8(inp: torch.Tensor, fp8_format: str = "e4m3", per_channel_scale: bool = False,
                rule=SCALE_IEEE) -> Tuple[torch.Tensor, torch.Tensor]:
    """ColossalAI cast_to_fp8: (q with inp's shape, scale_inv).  scale_inv has shape [rows]
    (per-channel; [1] for an empty input) or [1] (per-tensor)."""
    f = _fmt_of(fp8_format)
    q = torch.empty(inp.shape, dtype=_FMT_DTYPE[f], device=inp.device)
    if per_channel_scale:
        rows = inp.numel() // inp.shape[-1] if inp.dim() > 0 and inp.shape[-1] > 0 else 0
        s = torch.empty((max(rows, 1) if inp.numel() == 0 else rows,), dtype=torch.float32, device=inp.device)
        fp8q_cast_per_channel_ex(inp.reshape(-1, inp.shape[-1]) if inp.dim() != 2 else inp, q, s, f, rule)
    else:
        s = torch.empty((1,), dtype=torch.float32, device=inp.device)
        fp8q_cast_per_tensor_ex(inp, q, s, _workspace(inp.device), f, rule)
    return q, s


def cast_from_fp8(inp: torch.Tensor, scale_inv: torch.Tensor, ret_type: torch.dtype,
                  per_channel_scale: bool = False) -> torch.Tensor:
    """ColossalAI cast_from_fp8 (row r scaled by scale_inv[r] in the per-channel case)."""
    if inp.dtype not in _FP8_DTYPES:
        raise TypeError("Only float8_e4m3fn and float8_e5m2 are allowed.")
    y = torch.empty(inp.shape, dtype=ret_type, device=inp.device)
    fp8q_cast_from_fp8(inp, scale_inv, y, GRAN_ROW if per_channel_scale else GRAN_TENSOR, 0,
                       _FP8_DTYPES[inp.dtype])
    return y


def weight_dequant(x: torch.Tensor, s: torch.Tensor, block_size: int = 128,
                   dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """DeepSeek-V3 weight_dequant: y[M, N] = dtype(float(x) * s[i/B, j/B])."""
    if not (x.is_contiguous() and s.is_contiguous()):
        raise ValueError("Input tensors must be contiguous")
    if x.dim() != 2 or s.dim() != 2:
        raise ValueError("Input tensors must have 2 dimensions")
    y = torch.empty(x.shape, dtype=dtype, device=x.device)
    fp8q_block_dequant(x, s, y, block_size, _FP8_DTYPES.get(x.dtype, E4M3FN))
    return y


def cast_to_fp8_pipeline(x: torch.Tensor, rule=SCALE_IEEE) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """ColossalAI cast_to_fp8_pipeline: returns (codes uint8 with x's shape, scale_inv [1], fmt_tag int32 [1])."""
    q = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    s = torch.empty((1,), dtype=torch.float32, device=x.device)
    tag = torch.empty((1,), dtype=torch.int32, device=x.device)
    fp8q_cast_pipeline(x, q, s, tag, _workspace(x.device), rule)
    return q, s, tag


def cast_from_fp8_pipeline(q: torch.Tensor, scale_inv: torch.Tensor, fmt_tag: torch.Tensor,
                           dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """ColossalAI cast_from_fp8_pipeline: y = dtype(scale_inv * float(q)) in the tagged format."""
    y = torch.empty(q.shape, dtype=dtype, device=q.device)
    fp8q_cast_from_pipeline(q, scale_inv, fmt_tag, y)
    return y


# ---------------------------------------------------------------------------
# fp8-compressed collectives: [scale_inv | fp8 payload] records
# ---------------------------------------------------------------------------
RECORD_HEADER_BYTES = 16


def _layout_of(layout) -> int:
    if layout not in (RECORD_PACKED4, RECORD_ALIGNED16):
        raise ValueError("record layout must be RECORD_PACKED4 (4) or RECORD_ALIGNED16 (16)")
    return int(layout)


def record_bytes(numel: int, layout: int = RECORD_ALIGNED16) -> int:
    """Size of one record: RECORD_ALIGNED16, a 16-byte header (fp32 scale_inv,
    then zeros) and the fp8 payload padded with zeros to a multiple of 16
    bytes; RECORD_PACKED4, the page's own layout, the 4-byte scale then the
    codes.  The same arithmetic as fp8q_record_bytes_ex, on the host, so that
    buffers can be sized without loading the library."""
    if numel < 0:
        raise ValueError("numel must be >= 0")
    if _layout_of(layout) == RECORD_PACKED4:
        return 4 + numel
    return RECORD_HEADER_BYTES + -(-numel // 16) * 16


def fp8q_record_bytes(numel: int) -> int:
    return int(lib().fp8q_record_bytes(int(numel)))


def fp8q_record_bytes_ex(numel: int, layout: int = RECORD_ALIGNED16) -> int:
    return int(lib().fp8q_record_bytes_ex(int(numel), int(layout)))


def fp8q_pack_record(x: torch.Tensor, record: torch.Tensor, workspace: torch.Tensor, fmt=E5M2,
                     rule=SCALE_IEEE, stream=None) -> None:
    """Per-tensor cast of x into one record (uint8, record_bytes(x.numel()) bytes)."""
    fp8q_pack_record_ex(x, record, workspace, fmt, rule, RECORD_ALIGNED16, stream)


def fp8q_pack_record_ex(x: torch.Tensor, record: torch.Tensor, workspace: torch.Tensor, fmt=E5M2,
                        rule=SCALE_IEEE, layout: int = RECORD_ALIGNED16, stream=None) -> None:
    """Per-tensor cast of x into one record of the given layout (uint8, record_bytes(numel, layout))."""
    dev = x.device
    n = x.numel()
    _need(record, record_bytes(n, layout), "record", byte=True)
    wbytes = workspace.numel() * workspace.element_size()
    _check(lib().fp8q_pack_record_ex(
        _dev_ptr(x, "x"), _dtype_code(x, "x"), n, _fmt_of(fmt), _dev_ptr(record, "record", dev),
        _dev_ptr(workspace, "workspace", dev), wbytes, _rule_of(rule), _layout_of(layout), _stream(stream, dev)),
        "fp8q_pack_record_ex")


def fp8q_unpack_records(records: torch.Tensor, count: int, numel: int, y: torch.Tensor, fmt=E5M2,
                        stream=None) -> None:
    """Dequantise `count` back-to-back records of `numel` codes into y[count * numel] (dtype of y)."""
    fp8q_unpack_records_ex(records, count, numel, y, fmt, RECORD_ALIGNED16, stream)


def fp8q_unpack_records_ex(records: torch.Tensor, count: int, numel: int, y: torch.Tensor, fmt=E5M2,
                           layout: int = RECORD_ALIGNED16, stream=None) -> None:
    """Dequantise `count` back-to-back records of the given layout into y[count * numel]."""
    dev = records.device
    _need(records, count * record_bytes(numel, layout), "records", byte=True)
    _need(y, count * numel, "y")
    _check(lib().fp8q_unpack_records_ex(
        _dev_ptr(records, "records"), int(count), int(numel), _fmt_of(fmt), _dtype_code(y, "y"),
        _dev_ptr(y, "y", dev), _layout_of(layout), _stream(stream, dev)), "fp8q_unpack_records_ex")


def exchange_records(combined: torch.Tensor, group=None) -> None:
    """The all-gather step: combined is uint8 [world * R]; this rank's record
    sits at slot `rank` and every other slot is filled from its rank, in
    place.  Only bytes move; a no-op without a process group."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return
    world = dist.get_world_size(group)
    if world == 1:
        return
    slots = combined.view(world, -1)
    mine = slots[dist.get_rank(group)]
    dist.all_gather_into_tensor(combined, mine, group=group)


def exchange_records_all_to_all(recv: torch.Tensor, send: torch.Tensor, group=None) -> None:
    """The all-to-all step: send is uint8 [world * R] with the record for rank
    j at slot j; afterwards recv slot i holds rank i's record for this rank.
    Needs an initialised process group."""
    import torch.distributed as dist
    dist.all_to_all_single(recv, send, group=group)


def exchange_payload_all_to_all(recv_q: torch.Tensor, q: torch.Tensor, scales: torch.Tensor,
                                scale_inv: torch.Tensor, group=None) -> None:
    """The exchange of all_to_all_single_fp8: equal chunks of this rank's
    codes q go to the ranks (recv_q chunk i from rank i), and every rank's
    one scale_inv is all-gathered into scales[world].  Needs an initialised
    process group."""
    import torch.distributed as dist
    dist.all_to_all_single(recv_q, q, group=group)
    dist.all_gather_into_tensor(scales, scale_inv, group=group)


def _world_rank(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def all_gather_fp8(output_list, input_: torch.Tensor, group=None, fp8_format: str = "e5m2",
                   rule=SCALE_IEEE, layout: int = RECORD_ALIGNED16) -> None:
    """ColossalAI all_gather_fp8 (and all_gather_fp8_lagacy): every rank casts
    its tensor with its own per-tensor scale into a record, one all-gather
    moves the records, and each output_list[r] receives rank r's tensor
    dequantised with rank r's scale, in input_'s dtype.  output_list may
    also be one contiguous tensor [world, *input_.shape].  layout
    RECORD_PACKED4 puts the page's own bytes on the wire (4-byte scale, then
    the codes; numel a multiple of 4 when there is more than one rank)."""
    world, rank = _world_rank(group)
    dev = input_.device
    n = input_.numel()
    f = _fmt_of(fp8_format)
    R = record_bytes(n, layout)
    combined = torch.empty(world * R, dtype=torch.uint8, device=dev)
    fp8q_pack_record_ex(input_, combined[rank * R:(rank + 1) * R], _workspace(dev), f, rule, layout)
    exchange_records(combined, group)
    if isinstance(output_list, torch.Tensor):
        if output_list.numel() != world * n or not output_list.is_contiguous():
            raise ValueError("the output tensor must be contiguous with world * input_.numel() elements")
        fp8q_unpack_records_ex(combined, world, n, output_list, f, layout)
        return
    if len(output_list) != world:
        raise ValueError(f"output_list has {len(output_list)} tensors, the group has {world} ranks")
    for r, out in enumerate(output_list):
        fp8q_unpack_records_ex(combined[r * R:(r + 1) * R], 1, n, out, f, layout)


def all_to_all_fp8(output_list, input_list, group=None, fp8_format: str = "e5m2", rule=SCALE_IEEE) -> None:
    """ColossalAI all_to_all_fp8: input_list[j] (for rank j) is cast with its
    own per-tensor scale; output_list[i] receives rank i's tensor for this
    rank, dequantised with the scale rank i used.  All tensors have one
    numel and dtype."""
    world, _ = _world_rank(group)
    if len(input_list) != world or len(output_list) != world:
        raise ValueError("input_list and output_list need one tensor per rank")
    n = input_list[0].numel()
    if any(t.numel() != n for t in input_list) or any(t.numel() != n for t in output_list):
        raise ValueError("every tensor must have the same numel")
    dev = input_list[0].device
    f = _fmt_of(fp8_format)
    R = record_bytes(n)
    send = torch.empty(world * R, dtype=torch.uint8, device=dev)
    ws = _workspace(dev)
    for j, t in enumerate(input_list):
        fp8q_pack_record(t, send[j * R:(j + 1) * R], ws, f, rule)
    recv = send
    if world > 1:
        recv = torch.empty_like(send)
        exchange_records_all_to_all(recv, send, group)
    for i, out in enumerate(output_list):
        fp8q_unpack_records(recv[i * R:(i + 1) * R], 1, n, out, f)


def all_to_all_single_fp8(output: torch.Tensor, input: torch.Tensor, group=None, fp8_format: str = "e5m2",
                          rule=SCALE_IEEE) -> None:
    """ColossalAI all_to_all_single_fp8 with equal splits: the whole input is
    cast with ONE per-tensor scale, its world equal chunks along dim 0 go to
    the ranks, the scales are all-gathered, and chunk i of output is rank
    i's chunk dequantised with rank i's scale, in input's dtype."""
    world, _ = _world_rank(group)
    if input.shape[0] % world:
        raise ValueError("dim 0 must split evenly across the ranks")
    if output.shape != input.shape or output.dtype != input.dtype or not output.is_contiguous():
        raise ValueError("output must be a contiguous tensor of input's shape and dtype")
    dev = input.device
    f = _fmt_of(fp8_format)
    n = input.numel()
    c = n // world
    q = torch.empty(n, dtype=torch.uint8, device=dev)
    s = torch.empty(1, dtype=torch.float32, device=dev)
    fp8q_cast_per_tensor_ex(input, q, s, _workspace(dev), f, rule)
    qr, scales = q, s
    if world > 1:
        qr = torch.empty_like(q)
        scales = torch.empty(world, dtype=torch.float32, device=dev)
        exchange_payload_all_to_all(qr, q, scales, s, group)
    # chunk i with scale i: a block edge above any size gives one scale per chunk
    ws_, ss, ys = [], [], []
    flat = output.view(-1)
    cols = 4096
    for i in range(world):
        body, tail = divmod(c, cols)
        base = i * c
        if body:
            ws_.append(qr[base:base + body * cols].view(body, cols))
            ss.append(scales[i:i + 1])
            ys.append(flat[base:base + body * cols])
        if tail:
            ws_.append(qr[base + body * cols:base + c].view(1, tail))
            ss.append(scales[i:i + 1])
            ys.append(flat[base + body * cols:base + c])
    fp8q_block_dequant_grouped(ws_, ss, ys, block=1 << 30, fmt=f)


# ---------------------------------------------------------------------------
# fp8 matrix products (tensor cores)
# ---------------------------------------------------------------------------
def _mm_operands(a: torch.Tensor, b: torch.Tensor, out: torch.Tensor, bias, fa, fb):
    if a.dim() != 2 or b.dim() != 2:
        raise ValueError("a must be [M, K] and b [N, K] (the weight as stored)")
    M, K = a.shape
    N, K2 = b.shape
    if K != K2:
        raise ValueError(f"a has K = {K} but b has K = {K2}")
    _need(a, M * K, "a", byte=True)
    _need(b, N * K, "b", byte=True)
    _need(out, M * N, "out")
    if bias is not None:
        _need(bias, N, "bias", dtype=out.dtype)
    fa = _fmt_of(fa) if fa is not None else _FP8_DTYPES.get(a.dtype, E4M3FN)
    fb = _fmt_of(fb) if fb is not None else _FP8_DTYPES.get(b.dtype, E4M3FN)
    return M, N, K, fa, fb


def _status_word(status: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if status is not None and (status.dtype not in (torch.int32, torch.uint32) or status.numel() < 1):
        raise TypeError("status must be a CUDA int32 or uint32 tensor of at least one element")
    return status


def fp8q_scaled_mm(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                   out: torch.Tensor, bias: Optional[torch.Tensor] = None, fa=None, fb=None,
                   status: Optional[torch.Tensor] = None, stream=None) -> None:
    """ColossalAI linear_fp8 forward product, torch._scaled_mm(a, b.t(), scale_a, scale_b, bias):
    out[M, N] = T(acc * scale_a[0] * scale_b[0] + bias) with a [M, K] and b [N, K] fp8 codes
    (formats from their float8 dtypes, or fa / fb), scale_a / scale_b fp32 [1] on the device.
    `status`: optional int32/uint32 [1] device word that the kernel ORs a nonzero code into if
    one of its bounded internal waits runs out."""
    M, N, K, fa, fb = _mm_operands(a, b, out, bias, fa, fb)
    dev = a.device
    _need(scale_a, 1, "scale_a", dtype=torch.float32)
    _need(scale_b, 1, "scale_b", dtype=torch.float32)
    _check(lib().fp8q_scaled_mm(
        _dev_ptr(a, "a", dev), fa, _dev_ptr(b, "b", dev), fb, M, N, K,
        _dev_ptr(scale_a, "scale_a", dev), _dev_ptr(scale_b, "scale_b", dev), _dev_ptr(bias, "bias", dev),
        _dtype_code(out, "out"), _dev_ptr(out, "out", dev), _dev_ptr(_status_word(status), "status", dev),
        _stream(stream, dev)), "fp8q_scaled_mm")


WAIT_PRODUCER, WAIT_MMA, WAIT_EPILOGUE, WAIT_DRAIN = 1, 2, 4, 8      # status bits of the products


def fp8q_scaled_mm_wait_test(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                             out: torch.Tensor, status: torch.Tensor, wait_limit_ns: int, stall_kb: int = -1,
                             stream=None) -> None:
    """Test of the products' bounded waits: fp8q_scaled_mm (e4m3fn operands, bf16 out, no bias)
    with every internal wait bounded by wait_limit_ns; stall_kb >= 0 leaves out the copies of that
    k-block of each CTA's first tile, so that its waits run out and WAIT_* bits land in `status`."""
    M, N, K, _, _ = _mm_operands(a, b, out, None, E4M3FN, E4M3FN)
    dev = a.device
    _need(scale_a, 1, "scale_a", dtype=torch.float32)
    _need(scale_b, 1, "scale_b", dtype=torch.float32)
    if out.dtype != torch.bfloat16:
        raise TypeError("out must be bf16")
    if status is None:
        raise TypeError("status is required")
    _check(lib().fp8q_scaled_mm_wait_test(
        _dev_ptr(a, "a", dev), _dev_ptr(b, "b", dev), M, N, K,
        _dev_ptr(scale_a, "scale_a", dev), _dev_ptr(scale_b, "scale_b", dev), _dev_ptr(out, "out", dev),
        _dev_ptr(_status_word(status), "status", dev), int(wait_limit_ns), int(stall_kb),
        _stream(stream, dev)), "fp8q_scaled_mm_wait_test")


def fp8q_scaled_mm_blockwise_wait_test(a: torch.Tensor, scale_a: torch.Tensor, b: torch.Tensor,
                                       scale_b: torch.Tensor, out: torch.Tensor, status: torch.Tensor,
                                       wait_limit_ns: int, stall_kb: int = -1, stream=None) -> None:
    """The bounded-wait test of the fine-grained product: fp8q_scaled_mm_blockwise (e4m3fn operands,
    bf16 out, no bias) with every internal wait bounded by wait_limit_ns; stall_kb >= 0 leaves out
    the copies of that k-block of each CTA's first tile."""
    M, N, K, _, _ = _mm_operands(a, b, out, None, E4M3FN, E4M3FN)
    dev = a.device
    kb = -(-K // 128)
    _need(scale_a, M * kb, "scale_a", dtype=torch.float32)
    _need(scale_b, -(-N // 128) * kb, "scale_b", dtype=torch.float32)
    if out.dtype != torch.bfloat16:
        raise TypeError("out must be bf16")
    if status is None:
        raise TypeError("status is required")
    _check(lib().fp8q_scaled_mm_blockwise_wait_test(
        _dev_ptr(a, "a", dev), _dev_ptr(scale_a, "scale_a", dev), _dev_ptr(b, "b", dev),
        _dev_ptr(scale_b, "scale_b", dev), M, N, K, _dev_ptr(out, "out", dev),
        _dev_ptr(_status_word(status), "status", dev), int(wait_limit_ns), int(stall_kb),
        _stream(stream, dev)), "fp8q_scaled_mm_blockwise_wait_test")


def fp8q_scaled_mm_blockwise(a: torch.Tensor, scale_a: torch.Tensor, b: torch.Tensor, scale_b: torch.Tensor,
                             out: torch.Tensor, bias: Optional[torch.Tensor] = None, fa=None, fb=None,
                             status: Optional[torch.Tensor] = None, stream=None) -> None:
    """Per-token activations a [M, K] with scale_a [M, ceil(K/128)] (per_token_cast_to_fp8) times
    a weight b [N, K] with scale_b [ceil(N/128), ceil(K/128)] (one scale_inv per 128 x 128 block):
    out[M, N] = T(sum_kb scale_a[m, kb] * scale_b[n/128, kb] * acc_kb + bias)."""
    M, N, K, fa, fb = _mm_operands(a, b, out, bias, fa, fb)
    dev = a.device
    kb = -(-K // 128)
    _need(scale_a, M * kb, "scale_a", dtype=torch.float32)
    _need(scale_b, -(-N // 128) * kb, "scale_b", dtype=torch.float32)
    _check(lib().fp8q_scaled_mm_blockwise(
        _dev_ptr(a, "a", dev), fa, _dev_ptr(scale_a, "scale_a", dev), _dev_ptr(b, "b", dev), fb,
        _dev_ptr(scale_b, "scale_b", dev), M, N, K, _dev_ptr(bias, "bias", dev), _dtype_code(out, "out"),
        _dev_ptr(out, "out", dev), _dev_ptr(_status_word(status), "status", dev), _stream(stream, dev)),
        "fp8q_scaled_mm_blockwise")


def _operand_layout(t: torch.Tensor, name: str):
    """(storage tensor, layout) of a 2-D fp8 operand given as [rows, k]: K_MAJOR when its rows
    are contiguous, MN_MAJOR when it is the transpose of a contiguous [k, rows] matrix."""
    if t.is_contiguous():
        return t, K_MAJOR
    if t.t().is_contiguous():
        return t.t(), MN_MAJOR
    raise ValueError(f"{name} must be row-major or the transpose of a row-major matrix")


def scaled_mm(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
              bias: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """torch._scaled_mm(a, b, scale_a, scale_b, bias, out_dtype): out[M, N] = a[M, K] @ b[K, N] with
    per-tensor scales.  Each operand may be row-major or the transpose of a row-major matrix (as
    ColossalAI passes w_fp8.t()); neither is copied."""
    if a.dim() != 2 or b.dim() != 2:
        raise ValueError("a and b must be 2-D")
    A, la = _operand_layout(a, "a")                  # a as [M, K]
    B, lb = _operand_layout(b.t(), "b")              # b^T as [N, K]
    out = torch.empty((a.shape[0], b.shape[1]), dtype=out_dtype, device=a.device)
    fp8q_scaled_mm_ex(A, B, scale_a, scale_b, out, bias, a_layout=la, b_layout=lb)
    return out


def scaled_mm_blockwise(a: torch.Tensor, scale_a: torch.Tensor, w: torch.Tensor, scale_w: torch.Tensor,
                        bias: Optional[torch.Tensor] = None, out_dtype: torch.dtype = torch.bfloat16) -> torch.Tensor:
    """a [M, K] fp8 with per-token-group scale_a times the weight w [N, K] fp8 with 128 x 128 block
    scale_w; returns out [M, N] of out_dtype."""
    out = torch.empty((a.shape[0], w.shape[0]), dtype=out_dtype, device=a.device)
    fp8q_scaled_mm_blockwise(a, scale_a, w, scale_w, out, bias)
    return out


def fp8q_scaled_mm_ex(a: torch.Tensor, b: torch.Tensor, scale_a: torch.Tensor, scale_b: torch.Tensor,
                      out: torch.Tensor, bias: Optional[torch.Tensor] = None, a_layout: int = K_MAJOR,
                      b_layout: int = K_MAJOR, fa=None, fb=None, status: Optional[torch.Tensor] = None,
                      stream=None) -> None:
    """fp8q_scaled_mm with an operand layout each: A is stored [M, K] (K_MAJOR) or [K, M]
    (MN_MAJOR), B is stored [N, K] (K_MAJOR) or [K, N] (MN_MAJOR); out is [M, N]."""
    if a.dim() != 2 or b.dim() != 2:
        raise ValueError("a and b must be 2-D")
    M, K = (a.shape[1], a.shape[0]) if a_layout == MN_MAJOR else tuple(a.shape)
    N, K2 = (b.shape[1], b.shape[0]) if b_layout == MN_MAJOR else tuple(b.shape)
    if K != K2:
        raise ValueError(f"a has K = {K} but b has K = {K2}")
    _need(a, M * K, "a", byte=True)
    _need(b, N * K, "b", byte=True)
    _need(out, M * N, "out")
    if bias is not None:
        _need(bias, N, "bias", dtype=out.dtype)
    _need(scale_a, 1, "scale_a", dtype=torch.float32)
    _need(scale_b, 1, "scale_b", dtype=torch.float32)
    fa = _fmt_of(fa) if fa is not None else _FP8_DTYPES.get(a.dtype, E4M3FN)
    fb = _fmt_of(fb) if fb is not None else _FP8_DTYPES.get(b.dtype, E4M3FN)
    dev = a.device
    _check(lib().fp8q_scaled_mm_ex(
        _dev_ptr(a, "a", dev), fa, int(a_layout), _dev_ptr(b, "b", dev), fb, int(b_layout), M, N, K,
        _dev_ptr(scale_a, "scale_a", dev), _dev_ptr(scale_b, "scale_b", dev), _dev_ptr(bias, "bias", dev),
        _dtype_code(out, "out"), _dev_ptr(out, "out", dev), _dev_ptr(_status_word(status), "status", dev),
        _stream(stream, dev)), "fp8q_scaled_mm_ex")


def fp8q_transpose_fp8(src: torch.Tensor, dst: torch.Tensor, ld: Optional[int] = None, stream=None) -> None:
    """dst[c, r] = src[r, c] (fp8 codes), zero for rows <= r < ld; dst holds [cols, ld]."""
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    rows, cols = src.shape
    ld = rows if ld is None else int(ld)
    dev = src.device
    _need(src, rows * cols, "src", byte=True)
    _need(dst, cols * ld, "dst", byte=True)
    _check(lib().fp8q_transpose_fp8(_dev_ptr(src, "src", dev), rows, cols, _dev_ptr(dst, "dst", dev), ld,
                                    _stream(stream, dev)), "fp8q_transpose_fp8")


def fp8q_sum_rows(x: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """out[c] = sum over rows of x[r, c] in fp32, in a fixed order, stored in x's dtype."""
    if x.dim() != 2:
        raise ValueError("x must be 2-D")
    rows, cols = x.shape
    dev = x.device
    _need(out, cols, "out", dtype=x.dtype)
    _check(lib().fp8q_sum_rows(_dev_ptr(x, "x", dev), _dtype_code(x, "x"), rows, cols, _dev_ptr(out, "out", dev),
                               _stream(stream, dev)), "fp8q_sum_rows")


def transpose_fp8(src: torch.Tensor, pad_to: int = 1) -> torch.Tensor:
    """The .t().contiguous() of an fp8 matrix, with the new rows zero-padded to a multiple of pad_to."""
    rows, cols = src.shape
    ld = -(-rows // pad_to) * pad_to
    dst = torch.empty((cols, ld), dtype=src.dtype, device=src.device)
    fp8q_transpose_fp8(src, dst, ld)
    return dst


class _LinearFp8(torch.autograd.Function):
    """ColossalAI _LinearFp8: forward casts input and weight to e4m3 with one scale each and
    multiplies them; backward casts the output gradient to e5m2 with one scale and takes the
    input gradient g @ w and the weight gradient g^T @ x as two more scaled products, reading the
    weight, g and x where they lie (MN-major operands, no transposed copies); the bias gradient is
    the column sum of g.  All arithmetic runs in libfp8q.  As for torch._scaled_mm, the input's
    last dimension and the weight's first must be multiples of 16."""

    @staticmethod
    def forward(ctx, x: torch.Tensor, w: torch.Tensor, bias: Optional[torch.Tensor]) -> torch.Tensor:
        if x.dtype not in (torch.bfloat16, torch.float16) or x.dtype != w.dtype:
            raise TypeError("Only float16 and bfloat16 are allowed.")
        if bias is not None and bias.dtype != x.dtype:
            raise TypeError("Bias should have the same dtype as input.")
        x = x.contiguous()
        w = w.contiguous()
        ctx.x_shape = x.shape
        ctx.has_bias = bias is not None
        x2 = x.reshape(-1, x.shape[-1])
        x_fp8, sx = cast_to_fp8(x2, "e4m3")
        w_fp8, sw = cast_to_fp8(w, "e4m3")
        ctx.save_for_backward(x_fp8, w_fp8, sx, sw)
        out = torch.empty((x2.shape[0], w.shape[0]), dtype=x.dtype, device=x.device)
        fp8q_scaled_mm(x_fp8, w_fp8, sx, sw, out, bias)
        return out.reshape(*x.shape[:-1], w.shape[0])

    @staticmethod
    def backward(ctx, out_grad: torch.Tensor):
        x_fp8, w_fp8, sx, sw = ctx.saved_tensors
        g = out_grad.contiguous().reshape(-1, out_grad.shape[-1])
        T, N = g.shape
        K = w_fp8.shape[1]
        g_fp8, sg = cast_to_fp8(g, "e5m2")
        dt = out_grad.dtype
        # x_grad[T, K] = g[T, N] @ w[N, K]: A = g (k = n contiguous), B = w read as [k = n][K]
        x_grad = torch.empty((T, K), dtype=dt, device=g.device)
        fp8q_scaled_mm_ex(g_fp8, w_fp8, sg, sw, x_grad, a_layout=K_MAJOR, b_layout=MN_MAJOR)
        # w_grad[N, K] = g^T[N, T] @ x[T, K]: both operands read as [k = t][.], any token count
        w_grad = torch.empty((N, K), dtype=dt, device=g.device)
        fp8q_scaled_mm_ex(g_fp8, x_fp8, sg, sx, w_grad, a_layout=MN_MAJOR, b_layout=MN_MAJOR)
        bias_grad = None
        if ctx.has_bias:
            bias_grad = torch.empty((N,), dtype=dt, device=g.device)
            fp8q_sum_rows(g, bias_grad)
        return x_grad.reshape(ctx.x_shape), w_grad, bias_grad


def linear_fp8(input: torch.Tensor, weight: torch.Tensor, bias: Optional[torch.Tensor] = None) -> torch.Tensor:
    """ColossalAI linear_fp8: per-tensor e4m3 casts of input and weight (cast_to_fp8), then the
    scaled product with the input's dtype as output dtype; differentiable (see _LinearFp8)."""
    return _LinearFp8.apply(input, weight, bias)


def linear_fp8_blockwise(input: torch.Tensor, weight: torch.Tensor, weight_scale_inv: torch.Tensor,
                         bias: Optional[torch.Tensor] = None) -> torch.Tensor:
    """A linear layer on a DeepSeek-V3-style fp8 weight [N, K] with its 128 x 128 block scale_inv:
    the input is quantised per token (per_token_cast_to_fp8, 1 x 128 groups), then multiplied
    without dequantising either operand; the output has the input's dtype."""
    x = input.contiguous().reshape(-1, input.shape[-1])
    q, s = per_token_cast_to_fp8(x)
    out = torch.empty((x.shape[0], weight.shape[0]), dtype=input.dtype, device=input.device)
    fp8q_scaled_mm_blockwise(q, s, weight, weight_scale_inv, out, bias)
    return out.reshape(*input.shape[:-1], weight.shape[0])
