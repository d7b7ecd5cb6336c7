"""CPU oracle for block-scaled FP4 quantisation (test infrastructure).

This package wraps ``fp4_oracle.c`` -- a plain, slow, obviously-correct C
implementation of NVFP4 / MXFP4 quantise, pack, dequantise and the per-block
MSE scale search, written from the pages that define the method ("NVFP4 与
MXFP4 格式", charlestar.github.io, sections 1-8, and "FP4 / NVFP4 数学总结",
devpress.csdn.net, sections 3-10).

TEST INFRASTRUCTURE ONLY: only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py`` may import this package.  The CUDA
library never calls, links or loads it, and it shares no code with it.

Inputs are numpy arrays: ``float32`` for fp32 tensors, ``uint16`` holding
bf16 bit patterns for bf16 tensors.  Contract violations raise
``OracleError`` (a ``ValueError``) carrying the oracle's status value.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp4_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Oracle status values (its own numbering, see fp4_oracle.c).
OK, ERR_ARG, ERR_SHAPE, ERR_NONFINITE, ERR_RANGE = 0, 1, 2, 4, 5
STATUS_NAMES = {OK: "ok", ERR_ARG: "invalid argument", ERR_SHAPE: "shape",
                ERR_NONFINITE: "non-finite input", ERR_RANGE: "global scale out of range"}
F32, BF16 = 0, 1

# gcc flags: IEEE single operations in single precision, no contraction into
# FMA, no fast-math; -O2 only.
CFLAGS = ["-std=c99", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fPIC", "-shared"]


class OracleError(ValueError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"oracle: {STATUS_NAMES.get(status, status)}{': ' + what if what else ''}")


def build(force: bool = False) -> str:
    """Compile liboracle.so next to the source if missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        P, I64, I, F, D = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_double
        sig = {
            "oracle_f32_to_bf16": (ctypes.c_uint16, [F]),
            "oracle_e2m1_decode": (D, [I]),
            "oracle_e2m1_encode": (I, [D, P]),
            "oracle_e2m1_encode_f32": (None, [P, P, I64]),
            "oracle_pack4": (I, [P, I64, P]),
            "oracle_unpack4": (None, [P, I64, P]),
            "oracle_e4m3_value": (D, [I]),
            "oracle_e4m3_decode_byte": (D, [I]),
            "oracle_e4m3_encode": (I, [D]),
            "oracle_e8m0_value": (D, [I]),
            "oracle_tensor_amax": (I, [P, I, I64, P]),
            "oracle_nv_global_scale": (I, [F, P]),
            "oracle_nv_block_scale_code": (I, [F, F]),
            "oracle_nvfp4_quantize_with_g": (I, [P, I, I64, I64, F, P, P]),
            "oracle_nvfp4_quantize": (I, [P, I, I64, I64, P, P, P]),
            "oracle_nvfp4_dequantize": (None, [P, P, F, I64, I64, P]),
            "oracle_mx_block_exponent": (I, [F]),
            "oracle_mxfp4_quantize": (I, [P, I, I64, I64, P, P]),
            "oracle_mx_block_exponent_ceil": (I, [F, P]),
            "oracle_mxfp4_quantize_rule": (I, [P, I, I64, I64, I, P, P]),
            "oracle_nvfp4_quantize_four_over_six": (I, [P, I, I64, I64, P, P, P, P]),
            "oracle_nvfp4_quantize_four_over_six_with_g": (I, [P, I, I64, I64, F, P, P, P]),
            "oracle_mxfp4_dequantize": (None, [P, P, I64, I64, P]),
            "oracle_nv_block_loss": (D, [P, I, F]),
            "oracle_search_candidate_code": (I, [F, F, I]),
            "oracle_nvfp4_scale_search": (I, [P, I, I64, I64, P, P, P, P]),
            "oracle_nvfp4_scale_search_with_g": (I, [P, I, I64, I64, F, P, P, P]),
            "oracle_search_grid_code": (I, [F, F, I, I]),
            "oracle_nvfp4_scale_search_grid": (I, [P, I, I64, I64, I, I, I, P, P, P, P]),
            "oracle_nvfp4_scale_search_grid_with_g": (I, [P, I, I64, I64, F, I, I, I, P, P, P]),
            "oracle_nvfp4_artefact_loss": (I, [P, I, I64, I64, P, P, F, P]),
            "oracle_storage_bytes": (I64, [I64, I64, I64]),
            "oracle_padded_blocks": (I64, [I64, I64, I64]),
            "oracle_padded_storage_bytes": (I64, [I64, I64, I64, I64]),
            "oracle_pad_rows": (I, [P, I, I64, I64, I64, P]),
            "oracle_crop_rows": (I, [P, I64, I64, I64, P]),
            "oracle_transpose": (I, [P, I, I64, I64, P]),
            "oracle_nvfp4_gemm": (I, [P, P, F, P, P, F, I64, I64, I64, P, P]),
            "oracle_scales_mma_layout": (I, [P, I64, I64, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def _input(x: np.ndarray):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError("oracle input must be float32 or uint16 (bf16 bits)")


def _check(st: int, what: str = ""):
    if st != OK:
        raise OracleError(st, what)


# --------------------------------------------------------------------------
# Element and scale codecs
# --------------------------------------------------------------------------

def e2m1_decode(code: int) -> float:
    if not (isinstance(code, (int, np.integer)) and 0 <= int(code) < 16):
        raise OracleError(ERR_ARG, "expected a four-bit code")
    return lib().oracle_e2m1_decode(int(code))


def e2m1_encode(value: float) -> int:
    c = ctypes.c_int()
    _check(lib().oracle_e2m1_encode(float(value), ctypes.byref(c)), "finite input required")
    return c.value


def e2m1_encode_f32(v: np.ndarray) -> np.ndarray:
    """Codes of an fp32 array (0xFF marks a non-finite value)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, np.uint8)
    lib().oracle_e2m1_encode_f32(_ptr(v), _ptr(out), v.size)
    return out


def pack4(codes) -> bytes:
    c = np.ascontiguousarray(np.asarray(codes, dtype=np.int64))
    if c.size % 2:
        raise OracleError(ERR_SHAPE, "odd logical length")
    if c.size and (c.min() < 0 or c.max() > 15):
        raise OracleError(ERR_ARG, "four-bit codes required")
    c8 = c.astype(np.uint8)
    out = np.empty(c.size // 2, np.uint8)
    _check(lib().oracle_pack4(_ptr(c8), c8.size, _ptr(out)))
    return out.tobytes()


def unpack4(data: bytes) -> list:
    b = np.frombuffer(bytes(data), np.uint8).copy()
    out = np.empty(2 * b.size, np.uint8)
    lib().oracle_unpack4(_ptr(b), b.size, _ptr(out))
    return out.tolist()


def e4m3_value(code: int) -> float:
    return lib().oracle_e4m3_value(int(code))


def e4m3_decode_byte(byte: int) -> float:
    return lib().oracle_e4m3_decode_byte(int(byte))


def e4m3_encode(value: float) -> int:
    c = lib().oracle_e4m3_encode(float(value))
    if c < 0:
        raise OracleError(ERR_ARG, "finite non-negative scale required")
    return c


def e8m0_value(byte: int) -> float:
    return lib().oracle_e8m0_value(int(byte))


def f32_to_bf16(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    f = lib().oracle_f32_to_bf16
    return np.array([f(float(t)) for t in v], dtype=np.uint16)


def f32_to_bf16_fast(v: np.ndarray) -> np.ndarray:
    """Vectorised form of the same rounding (ties to even on the upper half),
    for large arrays; checked against ``f32_to_bf16`` in the tests."""
    u = np.ascontiguousarray(v, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = np.isnan(np.ascontiguousarray(v, dtype=np.float32))
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
    return r


def bf16_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------------
# Tensor-level NVFP4 / MXFP4
# --------------------------------------------------------------------------

def tensor_amax(x: np.ndarray) -> float:
    x, dt = _input(x)
    a = ctypes.c_float()
    _check(lib().oracle_tensor_amax(_ptr(x), dt, x.size, ctypes.byref(a)))
    return a.value


def nv_global_scale(amax: float) -> float:
    g = ctypes.c_float()
    _check(lib().oracle_nv_global_scale(float(amax), ctypes.byref(g)))
    return g.value


def nv_block_scale_code(amax_b: float, g: float) -> int:
    return lib().oracle_nv_block_scale_code(float(amax_b), float(g))


def mx_block_exponent(amax_b: float) -> int:
    return lib().oracle_mx_block_exponent(float(amax_b))


def _shape(x: np.ndarray):
    if x.ndim == 1:
        return 1, x.shape[0]
    if x.ndim != 2:
        raise OracleError(ERR_SHAPE, "1-D or 2-D input required")
    return x.shape


def nvfp4_quantize(x: np.ndarray):
    """Returns (packed uint8 [R, C/2], scales uint8 [R, C/16], g float)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    g = ctypes.c_float()
    _check(lib().oracle_nvfp4_quantize(_ptr(x), dt, R, C, _ptr(packed), _ptr(scales), ctypes.byref(g)))
    return packed, scales, g.value


def nvfp4_quantize_with_g(x: np.ndarray, g: float):
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    _check(lib().oracle_nvfp4_quantize_with_g(_ptr(x), dt, R, C, float(g), _ptr(packed), _ptr(scales)))
    return packed, scales


def mxfp4_quantize(x: np.ndarray):
    """Returns (packed uint8 [R, C/2], scales uint8 [R, C/32])."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 32), np.uint8)
    _check(lib().oracle_mxfp4_quantize(_ptr(x), dt, R, C, _ptr(packed), _ptr(scales)))
    return packed, scales


MX_FLOOR, MX_CEIL = 0, 1


def mx_block_exponent_ceil(amax_b: float) -> int:
    e = ctypes.c_int()
    _check(lib().oracle_mx_block_exponent_ceil(float(amax_b), ctypes.byref(e)))
    return e.value


def mxfp4_quantize_rule(x: np.ndarray, rule: int):
    """MXFP4 with scale rule MX_FLOOR (OCP) or MX_CEIL (the page's mx_scale)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 32), np.uint8)
    _check(lib().oracle_mxfp4_quantize_rule(_ptr(x), dt, R, C, int(rule), _ptr(packed), _ptr(scales)))
    return packed, scales


def nvfp4_quantize_four_over_six(x: np.ndarray):
    """Returns (packed, scales, g, block_loss float64)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    g = ctypes.c_float()
    _check(lib().oracle_nvfp4_quantize_four_over_six(_ptr(x), dt, R, C, _ptr(packed), _ptr(scales),
                                                     ctypes.byref(g), _ptr(loss)))
    return packed, scales, g.value, loss


def nvfp4_quantize_four_over_six_with_g(x: np.ndarray, g: float):
    """Four over six at a given global scale.  Returns (packed, scales, loss)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    _check(lib().oracle_nvfp4_quantize_four_over_six_with_g(_ptr(x), dt, R, C, float(g), _ptr(packed),
                                                            _ptr(scales), _ptr(loss)))
    return packed, scales, loss


def nvfp4_dequantize(packed: np.ndarray, scales: np.ndarray, g: float, rows: int, cols: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.empty((rows, cols), np.float32)
    lib().oracle_nvfp4_dequantize(_ptr(packed), _ptr(scales), float(g), rows, cols, _ptr(y))
    return y


def mxfp4_dequantize(packed: np.ndarray, scales: np.ndarray, rows: int, cols: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    y = np.empty((rows, cols), np.float32)
    lib().oracle_mxfp4_dequantize(_ptr(packed), _ptr(scales), rows, cols, _ptr(y))
    return y


# --------------------------------------------------------------------------
# Scale search
# --------------------------------------------------------------------------

def nv_block_loss(xb: np.ndarray, scale_code: int, g: float) -> float:
    xb = np.ascontiguousarray(xb, dtype=np.float32)
    assert xb.size == 16
    return lib().oracle_nv_block_loss(_ptr(xb), int(scale_code), float(g))


def search_candidate_code(amax_b: float, g: float, k: int) -> int:
    return lib().oracle_search_candidate_code(float(amax_b), float(g), int(k))


def nvfp4_scale_search(x: np.ndarray):
    """Brute force over the 64 candidates of every block.
    Returns (packed, scales, g, block_loss float64 [R, C/16])."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    g = ctypes.c_float()
    _check(lib().oracle_nvfp4_scale_search(_ptr(x), dt, R, C, _ptr(packed), _ptr(scales),
                                           ctypes.byref(g), _ptr(loss)))
    return packed, scales, g.value, loss


def search_grid_code(amax_b: float, g: float, num: int, q: int) -> int:
    return lib().oracle_search_grid_code(float(amax_b), float(g), int(num), int(q))


def nvfp4_scale_search_grid(x: np.ndarray, n: int, p: int, q: int):
    """Brute force over the n candidates (p + k) / q x A_b / (6g), k < n,
    of every block.  Returns (packed, scales, g, block_loss)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    g = ctypes.c_float()
    _check(lib().oracle_nvfp4_scale_search_grid(_ptr(x), dt, R, C, int(n), int(p), int(q), _ptr(packed),
                                                _ptr(scales), ctypes.byref(g), _ptr(loss)))
    return packed, scales, g.value, loss


def nvfp4_scale_search_grid_with_g(x: np.ndarray, g: float, n: int, p: int, q: int):
    """The grid search at a given global scale.  Returns (packed, scales,
    block_loss)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    _check(lib().oracle_nvfp4_scale_search_grid_with_g(_ptr(x), dt, R, C, float(g), int(n), int(p), int(q),
                                                       _ptr(packed), _ptr(scales), _ptr(loss)))
    return packed, scales, loss


def nvfp4_scale_search_with_g(x: np.ndarray, g: float):
    """The search at a given global scale (for row samples of a large
    tensor).  Returns (packed, scales, block_loss)."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    _check(lib().oracle_nvfp4_scale_search_with_g(_ptr(x), dt, R, C, float(g), _ptr(packed),
                                                  _ptr(scales), _ptr(loss)))
    return packed, scales, loss


def nvfp4_artefact_loss(x: np.ndarray, packed: np.ndarray, scales: np.ndarray, g: float) -> np.ndarray:
    """Per-block loss (double) of given NVFP4 artefacts against x."""
    x, dt = _input(x)
    R, C = _shape(x)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    loss = np.zeros((R, C // 16), np.float64)
    _check(lib().oracle_nvfp4_artefact_loss(_ptr(x), dt, R, C, _ptr(packed), _ptr(scales),
                                            float(g), _ptr(loss)))
    return loss


def storage_bytes(elements: int, group: int, global_bytes: int) -> int:
    n = lib().oracle_storage_bytes(int(elements), int(group), int(global_bytes))
    if n < 0:
        raise OracleError(ERR_SHAPE, "complete blocks required")
    return n


# --------------------------------------------------------------------------
# Ragged rows and column-wise grouping ("NVFP4 与 MXFP4 格式" sections 6-8)
# --------------------------------------------------------------------------

def padded_cols(cols: int, group: int) -> int:
    """Row length after padding to whole blocks: ceil(cols / G) * G."""
    return -(-int(cols) // group) * group


def padded_blocks(rows: int, cols: int, group: int) -> int:
    return lib().oracle_padded_blocks(int(rows), int(cols), int(group))


def padded_storage_bytes(rows: int, cols: int, group: int, global_bytes: int) -> int:
    n = lib().oracle_padded_storage_bytes(int(rows), int(cols), int(group), int(global_bytes))
    if n < 0:
        raise OracleError(ERR_ARG, "group must be 16 or 32")
    return n


def pad_rows(x: np.ndarray, group: int) -> np.ndarray:
    """x [R, K] with every row padded by +0 to whole blocks of `group`."""
    x, dt = _input(x)
    R, K = _shape(x)
    Kp = padded_cols(K, group)
    out = np.zeros((R, Kp), x.dtype)
    _check(lib().oracle_pad_rows(_ptr(x), dt, R, K, Kp, _ptr(out)))
    return out


def crop_rows(y: np.ndarray, cols: int) -> np.ndarray:
    y = np.ascontiguousarray(y, dtype=np.float32)
    R, Kp = y.shape
    out = np.zeros((R, cols), np.float32)
    _check(lib().oracle_crop_rows(_ptr(y), R, Kp, int(cols), _ptr(out)))
    return out


def transpose(x: np.ndarray) -> np.ndarray:
    x, dt = _input(x)
    R, C = _shape(x)
    out = np.zeros((C, R), x.dtype)
    _check(lib().oracle_transpose(_ptr(x), dt, R, C, _ptr(out)))
    return out


def nvfp4_quantize_padded(x: np.ndarray):
    """NVFP4 of x [R, K] with rows padded by +0 to whole 16-blocks: packed
    [R, ceil(K/16)*8], scales [R, ceil(K/16)], g (pads do not change A)."""
    return nvfp4_quantize(pad_rows(x, 16))


def mxfp4_quantize_padded(x: np.ndarray, rule: int = 0):
    """MXFP4 of x [R, K] with rows padded by +0 to whole 32-blocks."""
    return mxfp4_quantize_rule(pad_rows(x, 32), rule)


def nvfp4_dequantize_padded(packed, scales, g, rows: int, cols: int) -> np.ndarray:
    """Dequantise the padded layout, then crop every row to `cols`."""
    return crop_rows(nvfp4_dequantize(packed, scales, g, rows, padded_cols(cols, 16)), cols)


def mxfp4_dequantize_padded(packed, scales, rows: int, cols: int) -> np.ndarray:
    return crop_rows(mxfp4_dequantize(packed, scales, rows, padded_cols(cols, 32)), cols)


def nvfp4_quantize_columns(x: np.ndarray):
    """NVFP4 of x [R, C] grouped along columns: the padded row-wise
    quantisation of the transpose, packed [C, ceil(R/16)*8]."""
    return nvfp4_quantize_padded(transpose(x))


def mxfp4_quantize_columns(x: np.ndarray, rule: int = 0):
    return mxfp4_quantize_padded(transpose(x), rule)


# --------------------------------------------------------------------------
# The consumer: block-scaled matrix product ("NVFP4 与 MXFP4 格式" section 6)
# --------------------------------------------------------------------------

def nvfp4_gemm(pa, sa, ga, pb, sb, gb, M: int, N: int, K: int):
    """D = A B^T of two NVFP4 operands blocked along K (A [M, K], B [N, K]),
    exact in double; returns (D float64 [M, N], sum of |terms| [M, N])."""
    pa, sa, pb, sb = (np.ascontiguousarray(a, dtype=np.uint8) for a in (pa, sa, pb, sb))
    d = np.zeros((M, N), np.float64)
    mag = np.zeros((M, N), np.float64)
    _check(lib().oracle_nvfp4_gemm(_ptr(pa), _ptr(sa), float(ga), _ptr(pb), _ptr(sb), float(gb), M, N, K,
                                   _ptr(d), _ptr(mag)))
    return d, mag


def scales_mma_layout(scales: np.ndarray) -> np.ndarray:
    """Scale bytes [rows, nb] in the 128-row x 4-block tiled layout of the
    block-scaled tensor-core MMA (flat uint8, zero padded)."""
    s = np.ascontiguousarray(scales, dtype=np.uint8)
    rows, nb = s.shape
    out = np.zeros((-(-rows // 128)) * 128 * (-(-nb // 4)) * 4, np.uint8)
    _check(lib().oracle_scales_mma_layout(_ptr(s), rows, nb, _ptr(out)))
    return out
