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
OK, ERR_INVALID_ARG, ERR_SHAPE, ERR_ALIGN, ERR_NONFINITE, ERR_RANGE, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT = range(9)
F32, BF16 = 0, 1
NVFP4, MXFP4 = 0, 1
MX_FLOOR, MX_CEIL = 0, 1
# fp4_gemm_kernel
GEMM_AUTO, GEMM_CTA, GEMM_CTA_PAIR = 0, 1, 2

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
            "fp4_scale_search_grid": (I, [P, I, I64, I64, I, I, I, P, P, P, P, P, SZ, P, P]),
            "fp4_e2m1_round": (I, [P, P, I64, P]),
            "fp4_e2m1_roundtrip": (I, [P, P, I64, P]),
            "fp4_nv_encode_quotient": (I, [P, P, P, I64, P]),
            "fp4_test_bounded_wait": (I, [ctypes.c_uint32, P, P, P]),
            "fp4_grouped_workspace_bytes": (SZ, [I]),
            "fp4_nvfp4_quantize_grouped": (I, [P, I, I, P, SZ, P, P]),
            "fp4_tensor_amax_grouped": (I, [P, I, I, P, SZ, P, P]),
            "fp4_nvfp4_quantize_grouped_with_amax": (I, [P, I, I, P, P, P]),
            "fp4_mxfp4_quantize_grouped": (I, [P, I, I, P, P]),
            "fp4_mxfp4_quantize_ceil_grouped": (I, [P, I, I, P, P]),
            "fp4_dequantize_grouped": (I, [I, P, I, I, P]),
            "fp4_grouped_plan": (I, [P, I, I64, I, P, P, P, P, I]),
            "fp4_set_launch_unit_limit": (I, [I64]),
            "fp4_mma_scales_bytes": (SZ, [I64, I64]),
            "fp4_scales_to_mma_layout": (I, [P, I64, I64, P, P]),
            "fp4_nvfp4_gemm": (I, [P, P, P, P, P, P, I64, I64, I64, P, P, P]),
            "fp4_nvfp4_gemm_ex": (I, [P, P, P, P, P, P, I64, I64, I64, P, I, P, P]),
            "fp4_nvfp4_quantize_padded": (I, [P, I, I64, I64, P, P, P, P, SZ, P, P]),
            "fp4_nvfp4_quantize_padded_with_amax": (I, [P, I, I64, I64, P, P, P, P, P, P]),
            "fp4_mxfp4_quantize_padded": (I, [P, I, I64, I64, I, P, P, P, P]),
            "fp4_dequantize_padded": (I, [I, P, P, P, I64, I64, P, I, P]),
            "fp4_nvfp4_quantize_columns": (I, [P, I, I64, I64, P, P, P, P, SZ, P, P]),
            "fp4_nvfp4_quantize_columns_with_amax": (I, [P, I, I64, I64, P, P, P, P, P, P]),
            "fp4_mxfp4_quantize_columns": (I, [P, I, I64, I64, I, P, P, P, P]),
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


class QuantItem(ctypes.Structure):
    """struct fp4_quant_item (include/fp4.h)."""
    _fields_ = [("x", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64),
                ("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p)]


class DequantItem(ctypes.Structure):
    """struct fp4_dequant_item (include/fp4.h)."""
    _fields_ = [("packed", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("y", ctypes.c_void_p), ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


def quant_items(xs, packed, scales, global_scales=None):
    """A ctypes array of fp4_quant_item for matching lists of tensors."""
    arr = (QuantItem * len(xs))()
    for i, x in enumerate(xs):
        R, C = _shape2(x)
        arr[i] = QuantItem(_p(x), R, C, _p(packed[i]), _p(scales[i]),
                           _p(global_scales[i]) if global_scales is not None else None)
    return arr


def dequant_items(qs, ys):
    arr = (DequantItem * len(qs))()
    for i, (q, y) in enumerate(zip(qs, ys)):
        arr[i] = DequantItem(_p(q.packed), _p(q.scales), _p(q.global_scale), _p(y), q.rows, q.cols)
    return arr


def _group_dtype(xs) -> int:
    codes = {_dtype_code(x) for x in xs}
    if len(codes) > 1:
        raise TypeError("all matrices of a grouped call share one dtype")
    return codes.pop() if codes else BF16


def fp4_nvfp4_quantize_grouped(items, dtype, workspace, status, stream=None) -> int:
    return lib().fp4_nvfp4_quantize_grouped(ctypes.cast(items, ctypes.c_void_p), len(items), dtype,
                                            _p(workspace), workspace.numel() * workspace.element_size(),
                                            _p(status), _stream(stream))


def fp4_tensor_amax_grouped(items, dtype, workspace, status, stream=None) -> int:
    return lib().fp4_tensor_amax_grouped(ctypes.cast(items, ctypes.c_void_p), len(items), dtype,
                                         _p(workspace), workspace.numel() * workspace.element_size(),
                                         _p(status), _stream(stream))


def fp4_nvfp4_quantize_grouped_with_amax(items, dtype, amax_words, status, stream=None) -> int:
    return lib().fp4_nvfp4_quantize_grouped_with_amax(ctypes.cast(items, ctypes.c_void_p), len(items), dtype,
                                                      _p(amax_words), _p(status), _stream(stream))


def tensor_amax_grouped(xs, status=None, stream=None):
    """Per-matrix amax of every matrix in xs: (fp32 [len(xs)] on the device,
    status word)."""
    dev = xs[0].device if xs else torch.device("cuda")
    st = status if status is not None else new_status(dev)
    ws = torch.empty(lib().fp4_grouped_workspace_bytes(len(xs)) // 4, dtype=torch.float32, device=dev)
    items = quant_items(xs, [None] * len(xs), [None] * len(xs))
    _check(fp4_tensor_amax_grouped(items, _group_dtype(xs), ws, st, stream), "fp4_tensor_amax_grouped")
    return ws[:len(xs)], st


def fp4_mxfp4_quantize_grouped(items, dtype, status, ceil=False, stream=None) -> int:
    fn = lib().fp4_mxfp4_quantize_ceil_grouped if ceil else lib().fp4_mxfp4_quantize_grouped
    return fn(ctypes.cast(items, ctypes.c_void_p), len(items), dtype, _p(status), _stream(stream))


def fp4_dequantize_grouped(fmt, items, out_dtype, stream=None) -> int:
    return lib().fp4_dequantize_grouped(fmt, ctypes.cast(items, ctypes.c_void_p), len(items), out_dtype,
                                        _stream(stream))


def grouped_plan(units, max_units, max_entries):
    """The grouped calls' launch plan for items of `units` work units (host
    only): a list of (launch, item, first unit, units) pieces."""
    import numpy as np
    n = len(units)
    u = np.ascontiguousarray(units, dtype=np.int64)
    cap = 2 * n + 16
    while True:
        lo, it = np.zeros(cap, np.int32), np.zeros(cap, np.int32)
        fi, co = np.zeros(cap, np.int64), np.zeros(cap, np.int64)
        k = lib().fp4_grouped_plan(u.ctypes.data if n else None, n, max_units, max_entries, lo.ctypes.data,
                                   it.ctypes.data, fi.ctypes.data, co.ctypes.data, cap)
        if k < 0:
            raise ValueError("fp4_grouped_plan: invalid arguments")
        if k <= cap:
            return list(zip(lo[:k].tolist(), it[:k].tolist(), fi[:k].tolist(), co[:k].tolist()))
        cap = k


def fp4_e2m1_round(v, codes, stream=None) -> int:
    return lib().fp4_e2m1_round(_p(v), _p(codes), v.numel(), _stream(stream))


def fp4_e2m1_roundtrip(v, out, stream=None) -> int:
    return lib().fp4_e2m1_roundtrip(_p(v), _p(out), v.numel(), _stream(stream))


def fp4_nv_encode_quotient(x, d, codes, stream=None) -> int:
    return lib().fp4_nv_encode_quotient(_p(x), _p(d), _p(codes), x.numel(), _stream(stream))


def fp4_test_bounded_wait(tries: int, status, elapsed_ns, stream=None) -> int:
    return lib().fp4_test_bounded_wait(tries, _p(status), _p(elapsed_ns), _stream(stream))


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


def _padded(n: int, group: int) -> int:
    return -(-n // group) * group


def nvfp4_quantize_padded(x: torch.Tensor, workspace=None, status=None, stream=None, amax=None) -> Quantized:
    """NVFP4 of x [R, K] for any K: rows padded with +0 to whole 16-blocks
    (packed [R, ceil(K/16)*8], scales [R, ceil(K/16)]).  With `amax` (a
    device float32 holding the tensor amax) the call skips its own amax
    pass (fp4_nvfp4_quantize_padded_with_amax)."""
    R, K = _shape2(x)
    dev = x.device
    Kp = _padded(K, 16)
    packed = torch.empty((R, Kp // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, Kp // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    st = status if status is not None else new_status(dev)
    if amax is not None:
        _check(lib().fp4_nvfp4_quantize_padded_with_amax(_p(x), _dtype_code(x), R, K, _p(amax), _p(packed),
                                                         _p(scales), _p(g), _p(st), _stream(stream)),
               "fp4_nvfp4_quantize_padded_with_amax")
        return Quantized(NVFP4, packed, scales, g, st, R, K)
    ws = workspace if workspace is not None else workspace_for(x)
    _check(lib().fp4_nvfp4_quantize_padded(_p(x), _dtype_code(x), R, K, _p(packed), _p(scales), _p(g), _p(ws),
                                           ws.numel() * ws.element_size(), _p(st), _stream(stream)),
           "fp4_nvfp4_quantize_padded")
    return Quantized(NVFP4, packed, scales, g, st, R, K)


def mxfp4_quantize_padded(x: torch.Tensor, rule: int = MX_FLOOR, status=None, stream=None) -> Quantized:
    """MXFP4 of x [R, K] for any K: rows padded with +0 to whole 32-blocks."""
    R, K = _shape2(x)
    dev = x.device
    Kp = _padded(K, 32)
    packed = torch.empty((R, Kp // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, Kp // 32), dtype=torch.uint8, device=dev)
    st = status if status is not None else new_status(dev)
    _check(lib().fp4_mxfp4_quantize_padded(_p(x), _dtype_code(x), R, K, rule, _p(packed), _p(scales), _p(st),
                                           _stream(stream)), "fp4_mxfp4_quantize_padded")
    return Quantized(MXFP4, packed, scales, None, st, R, K)


def dequantize_padded(q: Quantized, out_dtype=torch.bfloat16, out=None, stream=None) -> torch.Tensor:
    """Dequantise a padded layout into the logical [q.rows, q.cols]."""
    y = out if out is not None else torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.packed.device)
    _check(lib().fp4_dequantize_padded(q.fmt, _p(q.packed), _p(q.scales), _p(q.global_scale), q.rows, q.cols,
                                       _p(y), _dtype_code(y), _stream(stream)), "fp4_dequantize_padded")
    return y


def nvfp4_quantize_columns(x: torch.Tensor, workspace=None, status=None, stream=None, amax=None) -> Quantized:
    """NVFP4 of W^T for x = W [R, C]: blocks down the columns of W; the
    result describes the logical [C, R] transpose in the padded layout.
    With `amax` (device float32, the amax of W) the call skips its own amax
    pass (fp4_nvfp4_quantize_columns_with_amax)."""
    R, C = _shape2(x)
    dev = x.device
    Rp = _padded(R, 16)
    packed = torch.empty((C, Rp // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((C, Rp // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    st = status if status is not None else new_status(dev)
    if amax is not None:
        _check(lib().fp4_nvfp4_quantize_columns_with_amax(_p(x), _dtype_code(x), R, C, _p(amax), _p(packed),
                                                          _p(scales), _p(g), _p(st), _stream(stream)),
               "fp4_nvfp4_quantize_columns_with_amax")
        return Quantized(NVFP4, packed, scales, g, st, C, R)
    ws = workspace if workspace is not None else workspace_for(x)
    _check(lib().fp4_nvfp4_quantize_columns(_p(x), _dtype_code(x), R, C, _p(packed), _p(scales), _p(g), _p(ws),
                                            ws.numel() * ws.element_size(), _p(st), _stream(stream)),
           "fp4_nvfp4_quantize_columns")
    return Quantized(NVFP4, packed, scales, g, st, C, R)


def mxfp4_quantize_columns(x: torch.Tensor, rule: int = MX_FLOOR, status=None, stream=None) -> Quantized:
    """MXFP4 of W^T for x = W [R, C] (column-wise 32-blocks)."""
    R, C = _shape2(x)
    dev = x.device
    Rp = _padded(R, 32)
    packed = torch.empty((C, Rp // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((C, Rp // 32), dtype=torch.uint8, device=dev)
    st = status if status is not None else new_status(dev)
    _check(lib().fp4_mxfp4_quantize_columns(_p(x), _dtype_code(x), R, C, rule, _p(packed), _p(scales), _p(st),
                                            _stream(stream)), "fp4_mxfp4_quantize_columns")
    return Quantized(MXFP4, packed, scales, None, st, C, R)


def scales_to_mma(scales: torch.Tensor, stream=None) -> torch.Tensor:
    """Block scales [rows, blocks] -> the tiled layout of the tensor-core MMA
    (flat uint8, fp4_mma_scales_bytes long)."""
    rows, nb = scales.shape
    out = torch.empty(lib().fp4_mma_scales_bytes(rows, nb), dtype=torch.uint8, device=scales.device)
    _check(lib().fp4_scales_to_mma_layout(_p(scales), rows, nb, _p(out), _stream(stream)), "fp4_scales_to_mma_layout")
    return out


def nvfp4_gemm(qa: Quantized, qb: Quantized, out=None, status=None, stream=None,
               kernel: int = GEMM_AUTO) -> torch.Tensor:
    """D [M, N] fp32 = g_a g_b A B^T on the tensor cores for NVFP4 A [M, K]
    and B [N, K] (M, N multiples of 128, K of 256; GEMM_CTA_PAIR needs M, N
    multiples of 256)."""
    if qa.fmt != NVFP4 or qb.fmt != NVFP4 or qa.cols != qb.cols:
        raise ValueError("two NVFP4 operands with the same K required")
    M, N, K = qa.rows, qb.rows, qa.cols
    dev = qa.packed.device
    d = out if out is not None else torch.empty((M, N), dtype=torch.float32, device=dev)
    st = status if status is not None else new_status(dev)
    sa, sb = scales_to_mma(qa.scales, stream), scales_to_mma(qb.scales, stream)
    _check(lib().fp4_nvfp4_gemm_ex(_p(qa.packed), _p(sa), _p(qa.global_scale), _p(qb.packed), _p(sb),
                                   _p(qb.global_scale), M, N, K, _p(d), kernel, _p(st), _stream(stream)),
           "fp4_nvfp4_gemm_ex")
    return d


def nvfp4_quantize_grouped(xs, status=None, stream=None) -> list[Quantized]:
    """NVFP4 quantisation of every matrix in xs, each with its own g, in a
    few launches (bit-identical to nvfp4_quantize per matrix)."""
    dev = xs[0].device if xs else torch.device("cuda")
    outs = [(torch.empty((R, C // 2), dtype=torch.uint8, device=dev),
             torch.empty((R, C // 16), dtype=torch.uint8, device=dev),
             torch.empty(1, dtype=torch.float32, device=dev)) for R, C in map(_shape2, xs)]
    st = status if status is not None else new_status(dev)
    ws = torch.empty(lib().fp4_grouped_workspace_bytes(len(xs)), dtype=torch.uint8, device=dev)
    items = quant_items(xs, [o[0] for o in outs], [o[1] for o in outs], [o[2] for o in outs])
    _check(fp4_nvfp4_quantize_grouped(items, _group_dtype(xs), ws, st, stream), "fp4_nvfp4_quantize_grouped")
    return [Quantized(NVFP4, p, s, g, st, *_shape2(x)) for x, (p, s, g) in zip(xs, outs)]


def mxfp4_quantize_grouped(xs, ceil: bool = False, status=None, stream=None) -> list[Quantized]:
    """MXFP4 quantisation of every matrix in xs in a few launches."""
    dev = xs[0].device if xs else torch.device("cuda")
    outs = [(torch.empty((R, C // 2), dtype=torch.uint8, device=dev),
             torch.empty((R, C // 32), dtype=torch.uint8, device=dev)) for R, C in map(_shape2, xs)]
    st = status if status is not None else new_status(dev)
    items = quant_items(xs, [o[0] for o in outs], [o[1] for o in outs])
    _check(fp4_mxfp4_quantize_grouped(items, _group_dtype(xs), st, ceil, stream), "fp4_mxfp4_quantize_grouped")
    return [Quantized(MXFP4, p, s, None, st, *_shape2(x)) for x, (p, s) in zip(xs, outs)]


def dequantize_grouped(qs, out_dtype=torch.bfloat16, outs=None, stream=None) -> list[torch.Tensor]:
    """Dequantise every Quantized in qs (all NVFP4 or all MXFP4)."""
    fmts = {q.fmt for q in qs}
    if len(fmts) > 1:
        raise ValueError("all items of a grouped dequantisation share one format")
    ys = outs if outs is not None else [
        torch.empty((q.rows, q.cols), dtype=out_dtype, device=q.packed.device) for q in qs]
    code = _dtype_code(ys[0]) if ys else (F32 if out_dtype == torch.float32 else BF16)
    _check(fp4_dequantize_grouped(fmts.pop() if fmts else NVFP4, dequant_items(qs, ys), code, stream),
           "fp4_dequantize_grouped")
    return ys


def scale_search(x: torch.Tensor, with_loss: bool = True, workspace=None, status=None, stream=None,
                 grid=None) -> Quantized:
    """MSE scale search; `grid` = (n_cand, p, q) searches the candidates
    (p + k) / q x A_b / (6g), k < n_cand (default: the fixed 64, 147, 210)."""
    R, C = _shape2(x)
    dev = x.device
    packed = torch.empty((R, C // 2), dtype=torch.uint8, device=dev)
    scales = torch.empty((R, C // 16), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    loss = torch.empty((R, C // 16), dtype=torch.float32, device=dev) if with_loss else None
    ws = workspace if workspace is not None else workspace_for(x)
    st = status if status is not None else new_status(dev)
    if grid is None:
        _check(fp4_scale_search(x, packed, scales, g, loss, ws, st, stream), "fp4_scale_search")
    else:
        n_cand, p, q = grid
        _check(lib().fp4_scale_search_grid(_p(x), _dtype_code(x), R, C, int(n_cand), int(p), int(q), _p(packed),
                                           _p(scales), _p(g), _p(loss), _p(ws), ws.numel() * ws.element_size(),
                                           _p(st), _stream(stream)), "fp4_scale_search_grid")
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
