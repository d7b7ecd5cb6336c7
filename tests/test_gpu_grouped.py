"""GPU parity of the grouped calls: many matrices per call, each with its own
scales ("NVFP4 与 MXFP4 格式" section 3: g belongs to one tensor).  The
grouped outputs must equal, bit for bit, one single-matrix call per item --
itself parity-tested against the oracle -- and the oracle directly on
small items and sampled rows."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
import workloads
from test_gpu_parity import assert_same, assert_same_bits, odata

pytestmark = pytest.mark.gpu
DEV = "cuda"


def mixed_items(dtype, seed, n=12):
    """Matrices of assorted shapes (empty, one block, ragged row counts,
    several tiles) and value ranges, so that every item has its own g."""
    g = torch.Generator().manual_seed(seed)
    shapes = [(0, 64), (1, 32), (3, 96), (17, 160), (64, 512), (129, 2080), (0, 0), (5, 32),
              (256, 1024), (33, 4128), (2, 64), (400, 800)][:n]
    xs = []
    for i, (r, c) in enumerate(shapes):
        scale = float(2.0 ** (i - 6))
        x = torch.randn(r, c, generator=g) * scale
        if r * c:
            x.view(-1)[torch.randint(0, r * c, (max(1, r * c // 500),), generator=g)] *= 40
        xs.append(x.to(dtype))
    return xs


def check_group(xs):
    xd = [x.to(DEV) for x in xs]
    nv = fp4.nvfp4_quantize_grouped(xd)
    mx = fp4.mxfp4_quantize_grouped(xd)
    mxc = fp4.mxfp4_quantize_grouped(xd, ceil=True)
    ynv = fp4.dequantize_grouped(nv, torch.float32)
    ymx = fp4.dequantize_grouped(mx, torch.bfloat16)
    amax, ast = fp4.tensor_amax_grouped(xd)
    torch.cuda.synchronize()
    assert ast.item() == 0
    for i, x in enumerate(xd):
        want = x.abs().amax().float().item() if x.numel() else 0.0
        assert amax[i].item() == want, f"item {i} amax"
        one_nv = fp4.nvfp4_quantize(x)
        one_mx = fp4.mxfp4_quantize(x)
        one_mxc = fp4.mxfp4_quantize_ceil(x)
        torch.cuda.synchronize()
        assert nv[i].global_scale.item() == one_nv.global_scale.item(), f"item {i} g"
        assert torch.equal(nv[i].packed, one_nv.packed), f"item {i} NV packed"
        assert torch.equal(nv[i].scales, one_nv.scales), f"item {i} NV scales"
        assert torch.equal(mx[i].packed, one_mx.packed) and torch.equal(mx[i].scales, one_mx.scales)
        assert torch.equal(mxc[i].packed, one_mxc.packed) and torch.equal(mxc[i].scales, one_mxc.scales)
        assert torch.equal(ynv[i].view(torch.int32), fp4.dequantize(one_nv, torch.float32).view(torch.int32))
        assert torch.equal(ymx[i].view(torch.int16), fp4.dequantize(one_mx, torch.bfloat16).view(torch.int16))
        # and the oracle on the whole (small) item
        if x.numel() and x.numel() <= 1 << 16:
            xo = odata(x.cpu())
            R, C = x.shape
            p, s, g = oracle.nvfp4_quantize(xo)
            assert nv[i].global_scale.item() == g
            assert_same(nv[i].packed, p, f"item {i} NV packed vs oracle")
            assert_same(nv[i].scales, s, f"item {i} NV scales vs oracle")
            assert_same_bits(ynv[i], oracle.nvfp4_dequantize(p, s, g, R, C), f"item {i} NV dequant")
            p, s = oracle.mxfp4_quantize(xo)
            assert_same(mx[i].packed, p, f"item {i} MX packed vs oracle")
            assert_same_bits(ymx[i], oracle.mxfp4_dequantize(p, s, R, C), f"item {i} MX dequant")
    assert nv[0].status.item() == 0 and mx[0].status.item() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_grouped_mixed_shapes(dtype):
    check_group(mixed_items(dtype, seed=5))


def test_grouped_more_items_than_one_launch_holds():
    # 300 items > 256 entries per launch: two launches of each kernel
    g = torch.Generator().manual_seed(9)
    xs = [(torch.randn(1 + i % 7, 32 * (1 + i % 5), generator=g) * (1 + i)).to(torch.bfloat16)
          for i in range(300)]
    check_group(xs)


def test_grouped_empty_list_and_all_empty_items():
    assert fp4.nvfp4_quantize_grouped([]) == []
    xs = [torch.zeros(0, 64, device=DEV), torch.zeros(0, 32, device=DEV)]
    nv = fp4.nvfp4_quantize_grouped(xs)
    torch.cuda.synchronize()
    assert [q.global_scale.item() for q in nv] == [1.0, 1.0] and nv[0].status.item() == 0


def test_grouped_data_errors_leave_other_items_correct():
    g = torch.Generator().manual_seed(3)
    xs = [torch.randn(8, 64, generator=g) for _ in range(4)]
    xs[1][3, 7] = float("nan")
    xs[2] = torch.full((1, 32), 2.0 ** -149)  # g underflows
    xd = [x.to(DEV) for x in xs]
    nv = fp4.nvfp4_quantize_grouped(xd)
    torch.cuda.synchronize()
    assert nv[0].status.item() in (fp4.ERR_NONFINITE, fp4.ERR_RANGE)
    for i in (0, 3):
        one = fp4.nvfp4_quantize(xd[i])
        torch.cuda.synchronize()
        assert torch.equal(nv[i].packed, one.packed) and torch.equal(nv[i].scales, one.scales)
        assert nv[i].global_scale.item() == one.global_scale.item()
    mx = fp4.mxfp4_quantize_grouped(xd)
    torch.cuda.synchronize()
    assert mx[0].status.item() == fp4.ERR_NONFINITE


def test_grouped_argument_errors():
    x = torch.randn(4, 48, device=DEV)  # 48 % 32 != 0
    with pytest.raises(fp4.FP4Error) as e:
        fp4.mxfp4_quantize_grouped([torch.randn(4, 64, device=DEV), x])
    assert e.value.status == fp4.ERR_SHAPE
    with pytest.raises(TypeError):
        fp4.nvfp4_quantize_grouped([torch.randn(4, 64, device=DEV), torch.randn(4, 64, device=DEV).bfloat16()])


def test_grouped_model_7b_layer_against_single_calls_and_oracle_rows():
    """One layer of the 7B-class weight set (4 x 4096^2 + 3 x 4096x14336
    bf16) in one grouped call per pass."""
    layer = 5
    ws = [workloads.model_matrix(layer, i) for i in range(len(workloads.MODEL_MATRICES))]
    xd = [workloads.generate(w, device=DEV) for w in ws]
    nv = fp4.nvfp4_quantize_grouped(xd)
    mx = fp4.mxfp4_quantize_grouped(xd)
    ynv = fp4.dequantize_grouped(nv)
    ymx = fp4.dequantize_grouped(mx)
    torch.cuda.synchronize()
    assert nv[0].status.item() == 0 and mx[0].status.item() == 0
    for i, (w, x) in enumerate(zip(ws, xd)):
        one = fp4.nvfp4_quantize(x)
        onem = fp4.mxfp4_quantize(x)
        torch.cuda.synchronize()
        assert nv[i].global_scale.item() == one.global_scale.item()
        assert torch.equal(nv[i].packed, one.packed) and torch.equal(nv[i].scales, one.scales)
        assert torch.equal(mx[i].packed, onem.packed) and torch.equal(mx[i].scales, onem.scales)
        assert torch.equal(ynv[i].view(torch.int16), fp4.dequantize(one).view(torch.int16))
        assert torch.equal(ymx[i].view(torch.int16), fp4.dequantize(onem).view(torch.int16))
        g = oracle.nv_global_scale(x.abs().amax().float().item())
        assert nv[i].global_scale.item() == g
        rows = workloads.sample_rows(w.rows, 3, seed=17 + i)
        sub = odata(x[rows].cpu())
        p, s = oracle.nvfp4_quantize_with_g(sub, g)
        assert_same(nv[i].packed[rows], p, f"{w.name} NV packed")
        assert_same(nv[i].scales[rows], s, f"{w.name} NV scales")
        assert_same_bits(ynv[i][rows], oracle.nvfp4_dequantize(p, s, g, len(rows), w.cols), f"{w.name} NV dq")
        p, s = oracle.mxfp4_quantize(sub)
        assert_same(mx[i].packed[rows], p, f"{w.name} MX packed")
        assert_same_bits(ymx[i][rows], oracle.mxfp4_dequantize(p, s, len(rows), w.cols), f"{w.name} MX dq")
