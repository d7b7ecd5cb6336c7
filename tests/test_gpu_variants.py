"""GPU parity of the scale-rule variants against the oracle, bit for bit:
the MXFP4 ceil rule ("NVFP4 与 MXFP4 格式" §5-§6, the `mx_scale` helper) and
NVFP4 four over six ("FP4、FP8 与 INT8/INT4" §4)."""
import dataclasses

import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
import workloads
from conftest import golden
from test_gpu_parity import assert_same, assert_same_bits, odata, oracle_call

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check_variants(x: torch.Tensor):
    xo = odata(x)
    R, C = x.shape
    xd = x.to(DEV)
    mx = fp4.mxfp4_quantize_ceil(xd) if C % 32 == 0 else None
    f6 = fp4.nvfp4_quantize_four_over_six(xd)
    y6 = fp4.dequantize(f6, torch.float32)
    ymx = fp4.dequantize(mx, torch.float32) if mx is not None else None
    torch.cuda.synchronize()
    if mx is not None:
        want, st = oracle_call(oracle.mxfp4_quantize_rule, xo, oracle.MX_CEIL)
        assert mx.status.item() == st, "MXFP4 ceil status"
        if want is not None:
            p, s = want
            assert_same(mx.packed, p, "MXFP4 ceil packed")
            assert_same(mx.scales, s, "MXFP4 ceil scales")
            assert_same_bits(ymx, oracle.mxfp4_dequantize(p, s, R, C), "MXFP4 ceil dequant")
    want, st = oracle_call(oracle.nvfp4_quantize_four_over_six, xo)
    assert f6.status.item() == st, "four-over-six status"
    if want is not None:
        p, s, g, loss = want
        assert f6.global_scale.item() == g
        assert_same(f6.scales, s, "four-over-six scales")
        assert_same(f6.packed, p, "four-over-six packed")
        assert_same(f6.block_loss, loss.astype(np.float32), "four-over-six loss")
        assert_same_bits(y6, oracle.nvfp4_dequantize(p, s, g, R, C), "four-over-six dequant")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 32), (7, 96), (129, 2080), (517, 4128)])
def test_variant_parity_shapes(dtype, shape):
    w = workloads.with_shape(workloads.SEARCH_4K, *shape, seed_offset=shape[0] + 3 * shape[1])
    check_variants(workloads.generate(dataclasses.replace(w, dtype=dtype)))


def test_variant_pages_examples():
    gd = golden("mx_ceil_rule.json")
    x = torch.tensor([[7.0] + [0.0] * 31 + [0.0] * 32], dtype=torch.float32)
    check_variants(x)
    q = fp4.mxfp4_quantize_ceil(x.to(DEV))
    torch.cuda.synchronize()
    assert [oracle.e8m0_value(int(b)) for b in q.scales.cpu().view(-1)] == [gd["amax_7_scale"],
                                                                               gd["zero_block_scale"]]
    n = gd["transpose_matrix"]["size"]
    w = torch.full((n, n), gd["transpose_matrix"]["rest"])
    w[0, 0] = gd["transpose_matrix"]["corner"]
    for m, want in ((w, gd["quantize_then_transpose_0_1"]), (w.T.contiguous(), gd["transpose_then_quantize_0_1"])):
        check_variants(m)
        y = fp4.dequantize(fp4.mxfp4_quantize_ceil(m.to(DEV)), torch.float32)
        torch.cuda.synchronize()
        got = y.T[0, 1].item() if m is w else y[0, 1].item()
        assert got == want
    g6 = golden("four_over_six.json")
    for key, want_map in (("max_to_4_exact", 4.0), ("max_to_6_exact", 6.0)):
        vals = g6[key]
        blk = vals + [0.0] * (16 - len(vals))
        x = torch.tensor([[2688.0] * 16 + blk], dtype=torch.float32)
        check_variants(x)
        q = fp4.nvfp4_quantize_four_over_six(x.to(DEV))
        torch.cuda.synchronize()
        assert oracle.e4m3_value(int(q.scales[0, 1].item())) == max(vals) / want_map
        assert q.block_loss[0, 1].item() == 0.0


def test_variant_edge_values():
    fmax = float(np.finfo(np.float32).max)
    rows = [[0.0] * 32, [-0.0] * 32, [fmax, -fmax] + [1.0] * 30,
            [1e-45, -1e-45, 2.0 ** -126, -(2.0 ** -127)] * 8, list(np.linspace(-3, 3, 32))]
    for r in rows:
        check_variants(torch.tensor([r], dtype=torch.float32))
    check_variants(torch.tensor(rows[2:], dtype=torch.float32))
    x = torch.randn(4, 64)
    x[1, 5] = float("nan")
    for q in (fp4.mxfp4_quantize_ceil(x.to(DEV)), fp4.nvfp4_quantize_four_over_six(x.to(DEV))):
        torch.cuda.synchronize()
        assert q.status.item() == fp4.ERR_NONFINITE


def test_variant_full_size_sampled_rows():
    for wl in (workloads.ACT_8K, workloads.SEARCH_4K):
        x = workloads.generate(wl)
        xd = x.to(DEV)
        mx = fp4.mxfp4_quantize_ceil(xd)
        f6 = fp4.nvfp4_quantize_four_over_six(xd)
        torch.cuda.synchronize()
        mx.check()
        f6.check()
        xo = odata(x)
        g = oracle.nv_global_scale(oracle.tensor_amax(xo))
        assert f6.global_scale.item() == g
        rows = workloads.sample_rows(wl.rows, 16, seed=wl.seed)
        sub = np.ascontiguousarray(xo[rows])
        p, s = oracle.mxfp4_quantize_rule(sub, oracle.MX_CEIL)
        assert_same(mx.packed[rows], p, f"{wl.name} MX ceil packed")
        assert_same(mx.scales[rows], s, f"{wl.name} MX ceil scales")
        p, s, loss = oracle.nvfp4_quantize_four_over_six_with_g(sub, g)
        assert_same(f6.scales[rows], s, f"{wl.name} 4/6 scales")
        assert_same(f6.packed[rows], p, f"{wl.name} 4/6 packed")
        assert_same(f6.block_loss[rows], loss.astype(np.float32), f"{wl.name} 4/6 loss")
