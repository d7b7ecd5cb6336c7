"""GPU parity of the ragged-row (padded) and column-wise layouts against the
oracle, bit for bit ("NVFP4 与 MXFP4 格式" section 6: grouping along the
other axis; section 7: decode padded, then cut each row back; section 8:
R * ceil(K/G) blocks)."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
import workloads
from conftest import golden
from test_gpu_parity import assert_same, assert_same_bits, odata

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rand(R, K, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, K, generator=g) * 0.05
    if R * K:
        x.view(-1)[torch.randint(0, R * K, (max(1, R * K // 300),), generator=g)] *= 30
    return x.to(dtype)


def check_padded(x):
    R, K = x.shape
    xo = odata(x)
    xd = x.to(DEV)
    nv = fp4.nvfp4_quantize_padded(xd)
    mxf = fp4.mxfp4_quantize_padded(xd, fp4.MX_FLOOR)
    mxc = fp4.mxfp4_quantize_padded(xd, fp4.MX_CEIL)
    ynv = fp4.dequantize_padded(nv, torch.float32)
    ynvb = fp4.dequantize_padded(nv, torch.bfloat16)
    ymx = fp4.dequantize_padded(mxf, torch.bfloat16)
    torch.cuda.synchronize()
    for q in (nv, mxf, mxc):
        q.check()
    p, s, g = oracle.nvfp4_quantize_padded(xo)
    assert nv.global_scale.item() == g
    assert_same(nv.packed, p, f"NV padded packed {R}x{K}")
    assert_same(nv.scales, s, f"NV padded scales {R}x{K}")
    want = oracle.nvfp4_dequantize_padded(p, s, g, R, K)
    assert ynv.shape == (R, K)
    assert_same_bits(ynv, want, f"NV padded dequant fp32 {R}x{K}")
    assert_same_bits(ynvb, want, f"NV padded dequant bf16 {R}x{K}")
    for q, rule in ((mxf, oracle.MX_FLOOR), (mxc, oracle.MX_CEIL)):
        p, s = oracle.mxfp4_quantize_padded(xo, rule)
        assert_same(q.packed, p, f"MX padded packed rule {rule} {R}x{K}")
        assert_same(q.scales, s, f"MX padded scales rule {rule} {R}x{K}")
    p, s = oracle.mxfp4_quantize_padded(xo, oracle.MX_FLOOR)
    assert_same_bits(ymx, oracle.mxfp4_dequantize_padded(p, s, R, K), f"MX padded dequant {R}x{K}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 1), (2, 17), (3, 15), (5, 33), (7, 100), (64, 1000), (129, 4099), (4, 64)])
def test_padded_rows_parity(dtype, shape):
    check_padded(rand(*shape, dtype, seed=shape[0] * 7 + shape[1]))


def test_padded_layout_bytes_of_the_page():
    gd = golden("padded_layout.json")
    x = torch.linspace(-1, 1, gd["rows"] * gd["cols"]).reshape(gd["rows"], gd["cols"]).to(DEV)
    q = fp4.nvfp4_quantize_padded(x)
    torch.cuda.synchronize()
    q.check()
    assert q.packed.numel() + q.scales.numel() + 4 == gd["nv_bytes"]
    assert q.scales.numel() == gd["blocks_padded"]
    check_padded(x.cpu())


def test_padded_equals_plain_for_complete_rows():
    x = rand(33, 256, torch.bfloat16, seed=2).to(DEV)
    a, b = fp4.nvfp4_quantize(x), fp4.nvfp4_quantize_padded(x)
    c, d = fp4.mxfp4_quantize(x), fp4.mxfp4_quantize_padded(x)
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed) and torch.equal(a.scales, b.scales)
    assert a.global_scale.item() == b.global_scale.item()
    assert torch.equal(c.packed, d.packed) and torch.equal(c.scales, d.scales)


def check_columns(x):
    R, C = x.shape
    xo = odata(x)
    xd = x.to(DEV)
    nv = fp4.nvfp4_quantize_columns(xd)
    mxf = fp4.mxfp4_quantize_columns(xd, fp4.MX_FLOOR)
    mxc = fp4.mxfp4_quantize_columns(xd, fp4.MX_CEIL)
    torch.cuda.synchronize()
    for q in (nv, mxf, mxc):
        q.check()
    p, s, g = oracle.nvfp4_quantize_columns(xo)
    assert nv.global_scale.item() == g
    assert_same(nv.packed, p, f"NV columns packed {R}x{C}")
    assert_same(nv.scales, s, f"NV columns scales {R}x{C}")
    y = fp4.dequantize_padded(nv, torch.float32)
    torch.cuda.synchronize()
    assert y.shape == (C, R)
    assert_same_bits(y, oracle.nvfp4_dequantize_padded(p, s, g, C, R), f"NV columns dequant {R}x{C}")
    for q, rule in ((mxf, oracle.MX_FLOOR), (mxc, oracle.MX_CEIL)):
        p, s = oracle.mxfp4_quantize_columns(xo, rule)
        assert_same(q.packed, p, f"MX columns packed rule {rule} {R}x{C}")
        assert_same(q.scales, s, f"MX columns scales rule {rule} {R}x{C}")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(16, 8), (20, 8), (64, 256), (100, 264), (129, 520), (300, 1032), (65, 4),
                                   (256, 520), (192, 264), (33, 6), (70, 98), (257, 130), (31, 1), (40, 3)])
def test_columns_parity(dtype, shape):
    R, C = shape
    if dtype == torch.bfloat16 and C % 2:
        # an odd bf16 row is not a whole number of the 4-byte words the
        # kernels read: the documented answer is FP4_ERR_ALIGN, returned
        # before anything is queued
        xd = rand(R, C, dtype, seed=R * 5 + C).to(DEV)
        for call in (fp4.nvfp4_quantize_columns, fp4.mxfp4_quantize_columns):
            with pytest.raises(fp4.FP4Error) as e:
                call(xd)
            assert e.value.status == fp4.ERR_ALIGN
        return
    check_columns(rand(R, C, dtype, seed=R * 5 + C))


def test_columns_transpose_counterexample_of_the_page():
    gd = golden("transpose_floor_rule.json")
    n = gd["size"]
    w = torch.full((n, n), gd["rest"])
    w[0, 0] = gd["corner"]
    wd = w.to(DEV)
    col = fp4.mxfp4_quantize_columns(wd)
    row = fp4.mxfp4_quantize(wd)
    yc = fp4.dequantize_padded(col, torch.float32)
    yr = fp4.dequantize(row, torch.float32)
    torch.cuda.synchronize()
    assert yc[0, 1].item() == gd["column_wise_0_1"]
    assert yr.T[0, 1].item() == gd["row_wise_then_transpose_0_1"]
    check_columns(w)


def test_columns_argument_errors():
    x = torch.randn(16, 13, device=DEV).bfloat16()  # 26-byte pitch: not whole 4-byte words
    with pytest.raises(fp4.FP4Error) as e:
        fp4.nvfp4_quantize_columns(x)
    assert e.value.status == fp4.ERR_ALIGN
    for R, C in ((0, 64), (64, 0)):
        q = fp4.nvfp4_quantize_columns(torch.zeros(R, C, device=DEV))
        torch.cuda.synchronize()
        assert q.status.item() == 0 and q.global_scale.item() == 1.0


def test_nonfinite_in_layouts():
    x = torch.randn(40, 72)
    x[13, 5] = float("inf")
    xd = x.to(DEV)
    for q in (fp4.nvfp4_quantize_padded(xd[:, :70].contiguous()), fp4.mxfp4_quantize_padded(xd[:, :70].contiguous()),
              fp4.nvfp4_quantize_columns(xd), fp4.mxfp4_quantize_columns(xd)):
        torch.cuda.synchronize()
        assert q.status.item() == fp4.ERR_NONFINITE


def test_columns_full_size_weight_sampled_columns():
    """4096 x 4096 bf16 weight: column-wise blocks checked against the
    oracle on sampled columns (each is one output row)."""
    w = workloads.WEIGHT_4K
    x = workloads.generate(w)
    xd = x.to(DEV)
    nv = fp4.nvfp4_quantize_columns(xd)
    mx = fp4.mxfp4_quantize_columns(xd)
    torch.cuda.synchronize()
    nv.check()
    mx.check()
    g = oracle.nv_global_scale(x.abs().amax().float().item())
    assert nv.global_scale.item() == g
    cols = workloads.sample_rows(w.cols, 12, seed=3)
    sub = odata(x[:, cols].T.contiguous())  # [k, R]: the sampled columns as rows
    p, s = oracle.nvfp4_quantize_with_g(sub, g)
    assert_same(nv.packed[cols], p, "NV columns packed (sampled)")
    assert_same(nv.scales[cols], s, "NV columns scales (sampled)")
    p, s = oracle.mxfp4_quantize(sub)
    assert_same(mx.packed[cols], p, "MX columns packed (sampled)")
    assert_same(mx.scales[cols], s, "MX columns scales (sampled)")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_with_amax_entry_points(dtype):
    """The _with_amax calls are the plain ones minus their amax pass: byte
    for byte the same outputs for the tensor's own amax, and, for a larger
    amax handed in (a max over shards), the oracle's quantisation at
    g = fl32(A / 2688) of that amax."""
    for R, K in ((5, 33), (129, 4099), (4, 64)):
        x = rand(R, K, dtype, seed=R + 11 * K)
        xd = x.to(DEV)
        a, _ = fp4.tensor_amax(xd)
        q0 = fp4.nvfp4_quantize_padded(xd)
        q1 = fp4.nvfp4_quantize_padded(xd, amax=a)
        big = torch.full((1,), 4.0 * a.item(), dtype=torch.float32, device=DEV)
        q2 = fp4.nvfp4_quantize_padded(xd, amax=big)
        torch.cuda.synchronize()
        for q in (q0, q1, q2):
            q.check()
        assert torch.equal(q0.packed, q1.packed) and torch.equal(q0.scales, q1.scales)
        assert q0.global_scale.item() == q1.global_scale.item()
        g = oracle.nv_global_scale(big.item())
        assert q2.global_scale.item() == g
        p, s = oracle.nvfp4_quantize_with_g(oracle.pad_rows(odata(x), 16), g)
        assert_same(q2.packed, p, f"NV padded with amax {R}x{K}")
        assert_same(q2.scales, s, f"NV padded scales with amax {R}x{K}")
    for R, C in ((100, 264), (300, 1032), (20, 8)):
        x = rand(R, C, dtype, seed=R + 13 * C)
        xd = x.to(DEV)
        a, _ = fp4.tensor_amax(xd)
        q0 = fp4.nvfp4_quantize_columns(xd)
        q1 = fp4.nvfp4_quantize_columns(xd, amax=a)
        big = torch.full((1,), 3.0 * a.item(), dtype=torch.float32, device=DEV)
        q2 = fp4.nvfp4_quantize_columns(xd, amax=big)
        torch.cuda.synchronize()
        for q in (q0, q1, q2):
            q.check()
        assert torch.equal(q0.packed, q1.packed) and torch.equal(q0.scales, q1.scales)
        assert q0.global_scale.item() == q1.global_scale.item()
        g = oracle.nv_global_scale(big.item())
        assert q2.global_scale.item() == g
        p, s = oracle.nvfp4_quantize_with_g(oracle.pad_rows(oracle.transpose(odata(x)), 16), g)
        assert_same(q2.packed, p, f"NV columns with amax {R}x{C}")
        assert_same(q2.scales, s, f"NV columns scales with amax {R}x{C}")


def test_with_amax_argument_errors():
    L = fp4.lib()
    x = torch.randn(8, 40, device=DEV)
    pk = torch.empty(8 * 24, dtype=torch.uint8, device=DEV)
    sc = torch.empty(8 * 3, dtype=torch.uint8, device=DEV)
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    st = fp4.new_status(DEV)
    a = torch.zeros(2, dtype=torch.float32, device=DEV)
    ab = a.view(torch.uint8)
    P = lambda t: t.data_ptr()  # noqa: E731
    for fn in (L.fp4_nvfp4_quantize_padded_with_amax, L.fp4_nvfp4_quantize_columns_with_amax):
        assert fn(P(x), fp4.F32, 8, 40, None, P(pk), P(sc), P(g), P(st), None) == fp4.ERR_INVALID_ARG
        assert fn(P(x), fp4.F32, 8, 40, P(ab[1:]), P(pk), P(sc), P(g), P(st), None) == fp4.ERR_ALIGN
        assert fn(P(x), fp4.F32, 8, 40, P(a), P(pk), P(sc), None, P(st), None) == fp4.ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_with_amax_nonfinite_amax_sets_status():
    """A non-finite amax handed in is a data error (NONFINITE in the status
    word), as for the plain calls' own amax."""
    x = rand(8, 40, torch.float32, seed=3).to(DEV)
    for bad in (float("inf"), float("nan")):
        a = torch.full((1,), bad, dtype=torch.float32, device=DEV)
        for call in (fp4.nvfp4_quantize_padded, fp4.nvfp4_quantize_columns):
            q = call(x, amax=a)
            torch.cuda.synchronize()
            assert q.status.item() == fp4.ERR_NONFINITE, (call.__name__, bad)


def test_padded_full_size_ragged_sampled_rows():
    """The 8192 x 14335 bf16 ragged-row workload as the benchmark runs it
    (the step's amax handed to the NVFP4 call): padded NVFP4 / MXFP4 codes
    and scales, and both bf16 dequantisations cut back to 14335 columns,
    checked against the oracle on sampled rows (first and last included)."""
    w = workloads.RAGGED_8K
    x = workloads.generate(w)
    xd = x.to(DEV)
    amax, _ = fp4.tensor_amax(xd)
    nv = fp4.nvfp4_quantize_padded(xd, amax=amax)
    mx = fp4.mxfp4_quantize_padded(xd)
    ynv = fp4.dequantize_padded(nv, torch.bfloat16)
    ymx = fp4.dequantize_padded(mx, torch.bfloat16)
    torch.cuda.synchronize()
    nv.check()
    mx.check()
    g = oracle.nv_global_scale(x.abs().amax().float().item())
    assert nv.global_scale.item() == g
    R, K = x.shape
    rows = workloads.sample_rows(R, 16, seed=5)
    sub = odata(x[rows].contiguous())
    p, s = oracle.nvfp4_quantize_with_g(oracle.pad_rows(sub, 16), g)
    assert_same(nv.packed[rows], p, "NV padded packed (sampled rows)")
    assert_same(nv.scales[rows], s, "NV padded scales (sampled rows)")
    assert_same_bits(ynv[rows], oracle.nvfp4_dequantize_padded(p, s, g, len(rows), K), "NV padded dequant (sampled)")
    p, s = oracle.mxfp4_quantize_padded(sub)
    assert_same(mx.packed[rows], p, "MX padded packed (sampled rows)")
    assert_same(mx.scales[rows], s, "MX padded scales (sampled rows)")
    assert_same_bits(ymx[rows], oracle.mxfp4_dequantize_padded(p, s, len(rows), K), "MX padded dequant (sampled)")
