"""Python binding of the B200 block-scaled FP4 library (libfp4.so).

Argument marshalling only: every step of the quantise / dequantise / scale
search path runs in the library's CUDA kernels.  PyTorch supplies device
memory and streams.  There is no CPU fallback: if libfp4.so is missing the
import of the entry points fails with an error saying how to build it.

Low-level functions carry the C names of include/fp4.h and take torch
tensors for the pointers; the snake-case helpers below them allocate the
outputs and return them.
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import re

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfp4.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "fp4.h")

# fp4_status / fp4_dtype / fp4_format values (include/fp4.h).
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_RANGE, ERR_WORKSPACE, ERR_CUDA = range(8)
F32, BF16 = 0, 1
NVFP4, MXFP4 = 0, 1

_lib = None


class FP4Error(RuntimeError):
    def __init__(self, status: int, where: str = ""):
        self.status = int(status)
        msg = lib().fp4_status_string(self.status).decode()
        super().__init__(f"{where}: {msg} (status {self.status})" if where else msg)


def lib() -> ctypes.CDLL:
    """The loaded libfp4.so (built by __graft_entry__.build() or
    `python -m block_scaled_fp4_reduce_b200.build`)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built; run `python -m block_scaled_fp4_reduce_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        sig = {
            "fp4_status_string": (ctypes.c_char_p, [I]),
            "fp4_version": (I, []),
            "fp4_workspace_bytes": (SZ, [I, I64, I64]),
            "fp4_tensor_amax": (I, [P, I, I64, P, P, SZ, P, P]),
            "fp4_nvfp4_quantize": (I, [P, I, I64, I64, P, P, P, P, SZ, P, P]),
            "fp4_nvfp4_quantize_with_amax": (I, [P, I, I64, I64, P, P, P, P, P, P]),
            "fp4_nvfp4_quantize_noalloc": (I, [P, I, I64, I64, P, P, P, P, P]),
            "fp4_mxfp4_quantize": (I, [P, I, I64, I64, P, P, P, P]),
            "fp4_mxfp4_quantize_ceil": (I, [P, I, I64, I64, P, P, P, P]),
            "fp4_nvfp4_quantize_four_over_six": (I, [P, I, I64, I64, P, P, P, P, P, SZ, P, P]),
            "fp4_dequantize": (I, [I, P, P, P, I64, I64, P, I, P]),
            "fp4_scale_search": (I, [P, I, I64, I64, P, P, P, P, P, SZ, P, P]),
            "fp4_scale_search_with_amax": (I, [P, I, I64, I64, P, P, P, P, P, P, P]),
            "fp4_e2m1_round": (I, [P, P, I64, P]),
            "fp4_e2m1_roundtrip": (I, [P, P, I64, P]),
            "fp4_nv_encode_quotient": (I, [P, P, P, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def declared_entry_points() -> list[str]:
    """Names of the functions include/fp4.h declares."""
    with open(HEADER_PATH) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return sorted(set(re.findall(r"\b(fp4_[a-z0-9_]+)\s*\(", text)))


# ---------------------------------------------------------------- helpers --

def _p(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"fp32 or bf16 tensor required, got {t.dtype}")


def _shape2(x: torch.Tensor):
    if not x.is_contiguous():
        raise ValueError("contiguous row-major tensor required")
    if x.dim() == 1:
        return 1, x.shape[0]
    return x.numel() // x.shape[-1] if x.shape[-1] else 0, x.shape[-1]


def _check(st: int, where: str):
    if st != OK:
        raise FP4Error(st, where)


# -------------------------------------------------------- C-ABI wrappers ---

def fp4_tensor_amax(x, amax, workspace, status, stream=None) -> int:
    return lib().fp4_tensor_amax(_p(x), _dtype_code(x), x.numel(), _p(amax), _p(workspace),
                                 workspace.numel() * workspace.element_size(), _p(status), _stream(stream))


def fp4_nvfp4_quantize(x, packed, scales, global_scale, workspace, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_nvfp4_quantize(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales), _p(global_scale),
                                    _p(workspace), workspace.numel() * workspace.element_size(),
                                    _p(status), _stream(stream))


def fp4_nvfp4_quantize_with_amax(x, amax, packed, scales, global_scale, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_nvfp4_quantize_with_amax(_p(x), _dtype_code(x), R, C, _p(amax), _p(packed), _p(scales),
                                              _p(global_scale), _p(status), _stream(stream))


def fp4_nvfp4_quantize_noalloc(x, packed, scales, global_scale, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_nvfp4_quantize_noalloc(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales),
                                            _p(global_scale), _p(status), _stream(stream))


def fp4_mxfp4_quantize(x, packed, scales, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_mxfp4_quantize(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales), _p(status),
                                    _stream(stream))


def fp4_mxfp4_quantize_ceil(x, packed, scales, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_mxfp4_quantize_ceil(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales), _p(status),
                                         _stream(stream))


def fp4_nvfp4_quantize_four_over_six(x, packed, scales, global_scale, block_loss, workspace, status,
                                     stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_nvfp4_quantize_four_over_six(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales),
                                                  _p(global_scale), _p(block_loss), _p(workspace),
                                                  workspace.numel() * workspace.element_size(),
                                                  _p(status), _stream(stream))


def fp4_dequantize(fmt, packed, scales, global_scale, rows, cols, y, stream=None) -> int:
    return lib().fp4_dequantize(fmt, _p(packed), _p(scales), _p(global_scale), rows, cols, _p(y),
                                _dtype_code(y), _stream(stream))


def fp4_scale_search(x, packed, scales, global_scale, block_loss, workspace, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_scale_search(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales), _p(global_scale),
                                  _p(block_loss), _p(workspace), workspace.numel() * workspace.element_size(),
                                  _p(status), _stream(stream))


def fp4_scale_search_with_amax(x, amax, packed, scales, global_scale, block_loss, status, stream=None) -> int:
    R, C = _shape2(x)
    return lib().fp4_scale_search_with_amax(_p(x), _dtype_code(x), R, C, _p(amax), _p(packed), _p(scales),
                                            _p(global_scale), _p(block_loss), _p(status), _stream(stream))


def fp4_e2m1_round(v, codes, stream=None) -> int:
    return lib().fp4_e2m1_round(_p(v), _p(codes), v.numel(), _stream(stream))


def fp4_e2m1_roundtrip(v, out, stream=None) -> int:
    return lib().fp4_e2m1_roundtrip(_p(v), _p(out), v.numel(), _stream(stream))


def fp4_nv_encode_quotient(x, d, codes, stream=None) -> int:
    return lib().fp4_nv_encode_quotient(_p(x), _p(d), _p(codes), x.numel(), _stream(stream))


# ------------------------------------------------- allocating helpers ------

@dataclasses.dataclass
class Quantized:
    """Packed codes [R, C/2], block scales [R, C/G] (uint8), the NVFP4 global
    scale g (fp32 [1], None for MXFP4) and the device status word."""
    fmt: int
    packed: torch.Tensor
    scales: torch.Tensor
    global_scale: torch.Tensor | None
    status: torch.Tensor
    rows: int
    cols: int
    block_loss: torch.Tensor | None = None

    def check(self, where: str = "fp4"):
        st = int(self.status.item())
        if st != OK:
            raise FP4Error(st, where)
        return self


def workspace_for(x: torch.Tensor) -> torch.Tensor:
    """A zero-filled workspace (the library keeps its counter word at zero)."""
    n = lib().fp4_workspace_bytes(NVFP4, *_shape2(x))
    return torch.zeros(n, dtype=torch.uint8, device=x.device)


def new_status(device) -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


def nvfp4_quantize(x: torch.Tensor, workspace=None, status=None, stream=None) -> Quantized:
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else workspace_for(x)
    st = status if status is not None else new_status(dev)
    _check(fp4_nvfp4_quantize(x, packed, scales, g, ws, st, stream), "fp4_nvfp4_quantize")
    return Quantized(NVFP4, packed, scales, g, st, R, C)


def mxfp4_quantize(x: torch.Tensor, status=None, stream=None) -> Quantized:
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 32), dtype=torch.uint8, device=dev)
    st = status if status is not None else new_status(dev)
    _check(fp4_mxfp4_quantize(x, packed, scales, st, stream), "fp4_mxfp4_quantize")
    return Quantized(MXFP4, packed, scales, None, st, R, C)


def mxfp4_quantize_ceil(x: torch.Tensor, status=None, stream=None) -> Quantized:
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 32), dtype=torch.uint8, device=dev)
    st = status if status is not None else new_status(dev)
    _check(fp4_mxfp4_quantize_ceil(x, packed, scales, st, stream), "fp4_mxfp4_quantize_ceil")
    return Quantized(MXFP4, packed, scales, None, st, R, C)


def nvfp4_quantize_four_over_six(x: torch.Tensor, with_loss: bool = True, workspace=None, status=None,
                                 stream=None) -> Quantized:
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    loss = torch.empty((R, C // 16), dtype=torch.float32, device=dev) if with_loss else None
    ws = workspace if workspace is not None else workspace_for(x)
    st = status if status is not None else new_status(dev)
    _check(fp4_nvfp4_quantize_four_over_six(x, packed, scales, g, loss, ws, st, stream),
           "fp4_nvfp4_quantize_four_over_six")
    return Quantized(NVFP4, packed, scales, g, st, R, C, block_loss=loss)


def dequantize(q: Quantized, out_dtype=torch.bfloat16, out=None, stream=None) -> torch.Tensor:
    y = out if out is not None else torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.packed.device)
    _check(fp4_dequantize(q.fmt, q.packed, q.scales, q.global_scale, q.rows, q.cols, y, stream),
           "fp4_dequantize")
    return y


def scale_search(x: torch.Tensor, with_loss: bool = True, workspace=None, status=None, stream=None) -> Quantized:
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    loss = torch.empty((R, C // 16), dtype=torch.float32, device=dev) if with_loss else None
    ws = workspace if workspace is not None else workspace_for(x)
    st = status if status is not None else new_status(dev)
    _check(fp4_scale_search(x, packed, scales, g, loss, ws, st, stream), "fp4_scale_search")
    return Quantized(NVFP4, packed, scales, g, st, R, C, block_loss=loss)


def tensor_amax(x: torch.Tensor, workspace=None, status=None, stream=None):
    dev = x.device
    a = torch.empty(1, dtype=torch.float32, device=dev)
    ws = workspace if workspace is not None else workspace_for(x)
    st = status if status is not None else new_status(dev)
    _check(fp4_tensor_amax(x, a, ws, st, stream), "fp4_tensor_amax")
    return a, st


def e2m1_round(v: torch.Tensor, stream=None) -> torch.Tensor:
    codes = torch.empty(v.shape, dtype=torch.uint8, device=v.device)
    _check(fp4_e2m1_round(v, codes, stream), "fp4_e2m1_round")
    return codes


def e2m1_roundtrip(v: torch.Tensor, stream=None) -> torch.Tensor:
    out = torch.empty((v.numel(), 2), dtype=torch.float32, device=v.device)
    _check(fp4_e2m1_roundtrip(v, out, stream), "fp4_e2m1_roundtrip")
    return out


def nv_encode_quotient(x: torch.Tensor, d: torch.Tensor, stream=None) -> torch.Tensor:
    codes = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    _check(fp4_nv_encode_quotient(x, d, codes, stream), "fp4_nv_encode_quotient")
    return codes
