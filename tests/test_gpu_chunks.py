"""Problems split across several launches.  Every call splits work above
2^30 units into launches; the test-only fp4_set_launch_unit_limit lowers
that limit so that small tensors cross the split points: row chunks whose
first element is not 32-byte aligned (ragged rows), MXFP4 dequant units in
pairs, grouped matrices split between launch tables.  Outputs must equal
the oracle bit for bit, as without splitting."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
from test_gpu_parity import assert_same, assert_same_bits, odata
from test_gpu_layouts import check_columns, check_padded, rand

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.fixture
def small_launches():
    assert fp4.lib().fp4_set_launch_unit_limit(256) == fp4.OK
    yield
    assert fp4.lib().fp4_set_launch_unit_limit(0) == fp4.OK


def test_row_longer_than_a_launch_is_refused(small_launches):
    # 257 blocks in one row cannot be split between launches of 256 units
    with pytest.raises(fp4.FP4Error) as e:
        fp4.nvfp4_quantize_padded(torch.randn(2, 4101, device=DEV))
    assert e.value.status == fp4.ERR_SHAPE


def test_limit_arguments():
    L = fp4.lib()
    assert L.fp4_set_launch_unit_limit(100) == fp4.ERR_INVALID_ARG
    assert L.fp4_set_launch_unit_limit(32) == fp4.ERR_INVALID_ARG
    assert L.fp4_set_launch_unit_limit((1 << 30) + 64) == fp4.ERR_INVALID_ARG
    assert L.fp4_set_launch_unit_limit(0) == fp4.OK


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_plain_calls_split_into_launches(small_launches, dtype):
    x = rand(64, 1056, dtype, seed=41)  # 4224 NV blocks, 2112 MX blocks, 4224 dequant units
    xo = odata(x)
    xd = x.to(DEV)
    nv, mx, ss = fp4.nvfp4_quantize(xd), fp4.mxfp4_quantize(xd), fp4.scale_search(xd)
    ynv, ymx = fp4.dequantize(nv, torch.float32), fp4.dequantize(mx, torch.bfloat16)
    torch.cuda.synchronize()
    for q in (nv, mx, ss):
        q.check()
    p, s, g = oracle.nvfp4_quantize(xo)
    assert nv.global_scale.item() == g
    assert_same(nv.packed, p, "NV packed")
    assert_same(nv.scales, s, "NV scales")
    assert_same_bits(ynv, oracle.nvfp4_dequantize(p, s, g, *x.shape), "NV dequant")
    p, s = oracle.mxfp4_quantize(xo)
    assert_same(mx.packed, p, "MX packed")
    assert_same_bits(ymx, oracle.mxfp4_dequantize(p, s, *x.shape), "MX dequant")
    p, s, g, _ = oracle.nvfp4_scale_search(xo)
    assert_same(ss.packed, p, "search packed")
    assert_same(ss.scales, s, "search scales")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(37, 999), (9, 4001), (300, 17)])
def test_ragged_rows_split_into_row_chunks(small_launches, dtype, shape):
    # K = 999 bf16: chunk r0 starts at byte 1998 * r0, not 32-byte aligned
    check_padded(rand(*shape, dtype, seed=shape[1]))


def test_columns_unaffected_by_the_limit(small_launches):
    check_columns(rand(200, 264, torch.bfloat16, seed=3))


def test_grouped_matrices_split_between_launches(small_launches):
    g = torch.Generator().manual_seed(8)
    xs = [(torch.randn(r, c, generator=g) * (i + 1)).to(torch.bfloat16)
          for i, (r, c) in enumerate([(64, 320), (3, 64), (128, 96), (0, 32), (33, 1024)])]
    xd = [x.to(DEV) for x in xs]
    nv = fp4.nvfp4_quantize_grouped(xd)
    mx = fp4.mxfp4_quantize_grouped(xd)
    ynv = fp4.dequantize_grouped(nv, torch.float32)
    ymx = fp4.dequantize_grouped(mx, torch.float32)
    torch.cuda.synchronize()
    assert nv[0].status.item() == 0 and mx[0].status.item() == 0
    for i, x in enumerate(xs):
        if not x.numel():
            assert nv[i].global_scale.item() == 1.0
            continue
        xo = odata(x)
        R, C = x.shape
        p, s, gg = oracle.nvfp4_quantize(xo)
        assert nv[i].global_scale.item() == gg
        assert_same(nv[i].packed, p, f"item {i} NV packed")
        assert_same(nv[i].scales, s, f"item {i} NV scales")
        assert_same_bits(ynv[i], oracle.nvfp4_dequantize(p, s, gg, R, C), f"item {i} NV dequant")
        p, s = oracle.mxfp4_quantize(xo)
        assert_same(mx[i].packed, p, f"item {i} MX packed")
        assert_same_bits(ymx[i], oracle.mxfp4_dequantize(p, s, R, C), f"item {i} MX dequant")
