"""Host-side checks of the C-ABI library that need no GPU: it builds, loads,
exports every entry point include/fp4.h declares, and rejects bad
arguments synchronously before touching CUDA."""
import ctypes
import os
import subprocess

import pytest

import block_scaled_fp4_reduce_b200 as fp4
from block_scaled_fp4_reduce_b200 import build as fp4_build


@pytest.fixture(scope="module")
def L():
    fp4_build.build()
    return fp4.lib()


def test_exports_every_declared_symbol(L):
    names = fp4.declared_entry_points()
    assert {"fp4_nvfp4_quantize", "fp4_mxfp4_quantize", "fp4_dequantize", "fp4_scale_search"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", fp4.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for n in names:
        assert n in exported, n
        assert getattr(L, n) is not None


def test_library_links_no_oracle_and_loads_without_driver(L):
    out = subprocess.run(["ldd", fp4.LIB_PATH], capture_output=True, text=True).stdout
    assert "oracle" not in out and "libcudart" not in out  # cudart is static


def test_status_strings_and_version(L):
    assert L.fp4_version() >= 100
    for st in range(8):
        assert L.fp4_status_string(st)
    assert L.fp4_status_string(0) == b"ok"
    assert L.fp4_workspace_bytes(fp4.NVFP4, 4096, 4096) >= 4


P = 1 << 20          # a fake, 16-byte aligned "device" address (never dereferenced)
Q = P + 4            # misaligned
WS = 1 << 16


def test_argument_errors_return_before_any_launch(L):
    f = L.fp4_nvfp4_quantize
    assert f(P, fp4.BF16, 4, 24, P, P, P, P, WS, P, None) == fp4.ERR_SHAPE          # cols % 16
    assert f(P, 7, 4, 32, P, P, P, P, WS, P, None) == fp4.ERR_INVALID_ARG           # dtype
    assert f(P, fp4.BF16, -1, 32, P, P, P, P, WS, P, None) == fp4.ERR_INVALID_ARG   # rows < 0
    assert f(P, fp4.BF16, 4, 32, P, P, None, P, WS, P, None) == fp4.ERR_INVALID_ARG # g NULL
    assert f(None, fp4.BF16, 4, 32, P, P, P, P, WS, P, None) == fp4.ERR_INVALID_ARG # x NULL
    assert f(Q, fp4.BF16, 4, 32, P, P, P, P, WS, P, None) == fp4.ERR_ALIGN
    assert f(P, fp4.BF16, 4, 32, Q, P, P, P, WS, P, None) == fp4.ERR_ALIGN
    assert f(P, fp4.BF16, 4, 32, P, P, P, P, 16, P, None) == fp4.ERR_WORKSPACE
    assert f(P, fp4.BF16, 4, 32, P, P, P, None, WS, P, None) == fp4.ERR_WORKSPACE
    assert f(P, fp4.BF16, 1 << 62, 1 << 20, P, P, P, P, WS, P, None) == fp4.ERR_SHAPE  # overflow
    m = L.fp4_mxfp4_quantize
    assert m(P, fp4.BF16, 4, 48, P, P, P, None) == fp4.ERR_SHAPE                   # cols % 32
    assert m(P, fp4.BF16, 4, 64, P, P, None, None) == fp4.ERR_INVALID_ARG          # status NULL
    assert m(Q, fp4.F32, 4, 64, P, P, P, None) == fp4.ERR_ALIGN
    assert m(P, fp4.F32, 0, 64, None, None, P, None) == fp4.OK                      # empty: no work
    d = L.fp4_dequantize
    assert d(5, P, P, P, 4, 32, P, fp4.BF16, None) == fp4.ERR_INVALID_ARG          # format
    assert d(fp4.NVFP4, P, P, None, 4, 32, P, fp4.BF16, None) == fp4.ERR_INVALID_ARG  # NV needs g
    assert d(fp4.MXFP4, P, P, None, 4, 48, P, fp4.BF16, None) == fp4.ERR_SHAPE
    assert d(fp4.NVFP4, P, P, P, 4, 32, Q, fp4.F32, None) == fp4.ERR_ALIGN
    assert d(fp4.MXFP4, P, P, None, 0, 32, P, fp4.F32, None) == fp4.OK
    s = L.fp4_scale_search
    assert s(P, fp4.BF16, 4, 8, P, P, P, None, P, WS, P, None) == fp4.ERR_SHAPE
    assert s(P, fp4.BF16, 4, 16, P, P, P, Q + 1, P, WS, P, None) == fp4.ERR_ALIGN
    a = L.fp4_tensor_amax
    assert a(P, fp4.BF16, 100, None, P, WS, P, None) == fp4.ERR_INVALID_ARG
    assert a(P, fp4.BF16, 100, P, P, 0, P, None) == fp4.ERR_WORKSPACE
    w = L.fp4_nvfp4_quantize_with_amax
    assert w(P, fp4.BF16, 4, 32, None, P, P, P, P, None) == fp4.ERR_INVALID_ARG
    assert w(P, fp4.BF16, 4, 32, Q + 2, P, P, P, P, None) == fp4.ERR_ALIGN
    assert L.fp4_e2m1_round(None, P, 5, None) == fp4.ERR_INVALID_ARG
    assert L.fp4_nv_encode_quotient(P, P, P, -1, None) == fp4.ERR_INVALID_ARG


def test_gemm_argument_errors_return_before_any_launch(L):
    """fp4_nvfp4_gemm_ex: shape, kernel choice, pointers and alignment are
    checked on the host before any CUDA call."""
    f = L.fp4_nvfp4_gemm_ex
    ok = (P, P, P, P, P, P)
    assert f(*ok, 256, 256, 256, P, 7, P, None) == fp4.ERR_INVALID_ARG                  # unknown kernel
    assert f(*ok, 256, 256, 256, P, fp4.GEMM_AUTO, None, None) == fp4.ERR_INVALID_ARG   # no status word
    assert f(*ok, -128, 256, 256, P, fp4.GEMM_AUTO, P, None) == fp4.ERR_INVALID_ARG
    assert f(*ok, 200, 256, 256, P, fp4.GEMM_AUTO, P, None) == fp4.ERR_SHAPE            # M % 128
    assert f(*ok, 256, 256, 320, P, fp4.GEMM_CTA, P, None) == fp4.ERR_SHAPE             # K % 256
    assert f(*ok, 384, 256, 256, P, fp4.GEMM_CTA_PAIR, P, None) == fp4.ERR_SHAPE        # pair: M % 256
    assert f(*ok, 256, 384, 256, P, fp4.GEMM_CTA_PAIR, P, None) == fp4.ERR_SHAPE        # pair: N % 256
    assert f(*ok, 0, 256, 256, P, fp4.GEMM_AUTO, P, None) == fp4.OK                     # empty D
    assert f(P, P, P, None, P, P, 256, 256, 256, P, fp4.GEMM_AUTO, P, None) == fp4.ERR_INVALID_ARG
    assert f(Q, P, P, P, P, P, 256, 256, 256, P, fp4.GEMM_AUTO, P, None) == fp4.ERR_ALIGN
    assert f(*ok, 256, 256, 256, Q, fp4.GEMM_AUTO, P, None) == fp4.ERR_ALIGN           # d


def test_scale_layout_argument_errors(L):
    f = L.fp4_scales_to_mma_layout
    assert f(P, -1, 4, P, None) == fp4.ERR_INVALID_ARG
    assert f(P, 0, 0, P, None) == fp4.OK                   # nothing to write
    assert f(P, 128, 4, None, None) == fp4.ERR_INVALID_ARG
    assert f(P, 128, 4, P + 2, None) == fp4.ERR_ALIGN      # out must be 4-byte aligned
    assert f(P, 128, 5_000_000, P, None) == fp4.ERR_SHAPE  # more scale tiles per band than one grid row
    assert L.fp4_mma_scales_bytes(130, 5) == 256 * 8       # 128-row bands x 4-block tiles, zero padded


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    monkeypatch.setattr(fp4, "_lib", None)
    monkeypatch.setattr(fp4, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="not built"):
        fp4.lib()
