"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Integer / byte outputs (codes, packed bytes, scale bytes) and the fp32 /
bf16 dequantised values are compared bit for bit; so are the global scale
and the scale search's per-block loss (the search compares candidates in
the definition's double arithmetic whenever fp32 cannot settle them).
Sizes: small shapes spanning several CTAs with ragged tails, the full
tiny-f32 and weight-4096 workloads, and sampled rows of the full
8192x14336 activation, the 4096x14336 search input and the 7B-class weight
set, at the sizes and launch configuration the benchmark uses.
"""
import dataclasses

import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda"


def odata(x: torch.Tensor) -> np.ndarray:
    return workloads.as_oracle_array(x)


def f32bits(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu()
        if a.dtype == torch.bfloat16:
            return a.view(torch.int16).numpy().view(np.uint16)
        return a.numpy().view(np.uint32)
    return np.asarray(a).view(np.uint32)


def assert_same(got: torch.Tensor, want: np.ndarray, what: str):
    g = got.detach().cpu().numpy()
    if not np.array_equal(g, want):
        bad = np.argwhere(g != want)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: got {g[i]!r} want {want[i]!r}")


def assert_same_bits(got: torch.Tensor, want_f32: np.ndarray, what: str):
    """fp32 output vs the oracle's fp32 (or bf16 output vs the oracle's fp32
    rounded to bf16 by the oracle's own rounding), bit for bit; NaNs match
    any NaN."""
    if got.dtype == torch.bfloat16:
        want = oracle.f32_to_bf16_fast(want_f32)
        g = f32bits(got)
        nan_w = np.isnan(want_f32)
        nan_g = (g & 0x7FFF) > 0x7F80
    else:
        want = want_f32.view(np.uint32)
        g = f32bits(got)
        nan_w = np.isnan(want_f32)
        nan_g = np.isnan(got.detach().cpu().numpy())
    assert np.array_equal(nan_w, nan_g), f"{what}: NaN positions differ"
    ok = (g == want) | nan_w
    if not ok.all():
        bad = np.argwhere(~ok)
        i = tuple(bad[0])
        raise AssertionError(f"{what}: {len(bad)} mismatches, first at {i}: got {g[i]:#x} want {want[i]:#x}")


def run_all(xd: torch.Tensor, search: bool = True):
    nv = fp4.nvfp4_quantize(xd)
    mx = fp4.mxfp4_quantize(xd) if xd.shape[-1] % 32 == 0 else None
    out = {"nv": nv, "mx": mx,
           "ynv32": fp4.dequantize(nv, torch.float32), "ynv16": fp4.dequantize(nv, torch.bfloat16)}
    if mx is not None:
        out["ymx32"] = fp4.dequantize(mx, torch.float32)
        out["ymx16"] = fp4.dequantize(mx, torch.bfloat16)
    if search:
        out["ss"] = fp4.scale_search(xd)
    torch.cuda.synchronize()
    return out


def oracle_call(fn, *args):
    """(result, 0) or (None, the oracle's data-error status)."""
    try:
        return fn(*args), 0
    except oracle.OracleError as e:
        return None, e.status


def check_full(x: torch.Tensor, search: bool = True):
    """Every output of every entry point against the oracle on all of x.
    Where the oracle rejects the input, the device status must carry the
    same error (the oracle's and the library's data-error values agree)."""
    xo = odata(x)
    R, C = x.shape
    res = run_all(x.to(DEV), search)
    want, st = oracle_call(oracle.nvfp4_quantize, xo)
    assert res["nv"].status.item() == st, "NVFP4 status"
    if want is not None:
        p, s, g = want
        assert_same(res["nv"].packed, p, "NVFP4 packed")
        assert_same(res["nv"].scales, s, "NVFP4 scales")
        assert res["nv"].global_scale.item() == g
        y = oracle.nvfp4_dequantize(p, s, g, R, C)
        assert_same_bits(res["ynv32"], y, "NVFP4 dequant fp32")
        assert_same_bits(res["ynv16"], y, "NVFP4 dequant bf16")
    if res["mx"] is not None:
        want, st = oracle_call(oracle.mxfp4_quantize, xo)
        assert res["mx"].status.item() == st, "MXFP4 status"
        if want is not None:
            p, s = want
            assert_same(res["mx"].packed, p, "MXFP4 packed")
            assert_same(res["mx"].scales, s, "MXFP4 scales")
            y = oracle.mxfp4_dequantize(p, s, R, C)
            assert_same_bits(res["ymx32"], y, "MXFP4 dequant fp32")
            assert_same_bits(res["ymx16"], y, "MXFP4 dequant bf16")
    if search:
        want, st = oracle_call(oracle.nvfp4_scale_search, xo)
        assert res["ss"].status.item() == st, "search status"
        if want is not None:
            p, s, g, loss = want
            assert res["ss"].global_scale.item() == g
            assert_same(res["ss"].scales, s, "search scales")
            assert_same(res["ss"].packed, p, "search packed")
            # the fp32 rounding of the double loss: a block near +-FLT_MAX has a
            # loss above FLT_MAX, which both sides round to +inf
            with np.errstate(over="ignore"):
                loss32 = loss.astype(np.float32)
            assert np.array_equal(np.isinf(loss32), np.isinf(res["ss"].block_loss.cpu().numpy()))
            assert_same(res["ss"].block_loss, loss32, "search block loss")
    return res


# ------------------------------------------------------------ element level

def test_e2m1_round_all_bf16_and_decisive_fp32():
    # every bf16 pattern (as fp32), then every fp32 with |v| in [2^-3, 8)
    b = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    b = b[torch.isfinite(b)]
    got = fp4.e2m1_round(b.to(DEV)).cpu().numpy()
    assert np.array_equal(got, oracle.e2m1_encode_f32(b.numpy()))
    lo, hi = 0x3E000000, 0x41000000  # 0.125 .. 8.0
    for sign in (0, 0x80000000):
        for start in range(lo, hi, 1 << 25):
            bits = torch.arange(start, min(start + (1 << 25), hi), dtype=torch.int64) | sign
            v = bits.to(torch.int32).view(torch.float32) if sign == 0 else \
                (bits - (1 << 32)).to(torch.int32).view(torch.float32)
            got = fp4.e2m1_round(v.to(DEV)).cpu().numpy()
            want = oracle.e2m1_encode_f32(v.numpy())
            assert np.array_equal(got, want), hex(start | sign)


def test_e2m1_round_every_finite_fp32_outside_the_decisive_range():
    """All 2^32 patterns: below 0.125 the code is 0 / 8 by sign, from 8 up
    (finite) it is 7 / 15 (saturation); checked on the device in chunks."""
    chunk = 1 << 28
    for start in range(0, 1 << 32, chunk):
        bits = torch.arange(start, start + chunk, dtype=torch.int64, device=DEV)
        v = (bits - ((bits >> 31) << 32)).to(torch.int32).view(torch.float32)
        c = fp4.e2m1_round(v).to(torch.int32)
        mag = v.abs()
        neg = (bits >> 31).bool()
        small = mag < 0.125
        big = (mag >= 8.0) & torch.isfinite(v)
        assert torch.equal(c[small], torch.where(neg[small], 8, 0).to(torch.int32))
        assert torch.equal(c[big], torch.where(neg[big], 15, 7).to(torch.int32))
        del bits, v, c, mag, neg, small, big


def test_e2m1_register_roundtrip():
    """Codes handed from the encoder to the decoder in registers (the
    kernels' own chain), and the fused quantise-dequantise of the search,
    both give the oracle's decode(encode(v)) for every bf16 pattern and a
    dense fp32 sweep."""
    b = torch.arange(1 << 16, dtype=torch.int32).to(torch.int16).view(torch.bfloat16).float()
    v = torch.cat([b[torch.isfinite(b)], torch.linspace(-8, 8, 1 << 20)]).contiguous()
    out = fp4.e2m1_roundtrip(v.to(DEV)).cpu().numpy()
    codes = oracle.e2m1_encode_f32(v.numpy())
    mag = np.array([oracle.e2m1_decode(c) for c in range(16)], np.float32)
    want = mag[codes]
    ok_chain = np.array_equal(out[:, 0].view(np.uint32), want.view(np.uint32))
    ok_fused = np.array_equal(out[:, 1].view(np.uint32), want.view(np.uint32))
    assert ok_chain and ok_fused, f"decode(encode) in registers: {ok_chain}, fused quantise-dequantise: {ok_fused}"


def test_nv_quotient_bracket_matches_ieee_division():
    """codes of fl32(x / d) for random pairs and for pairs placed exactly
    on, and a few ulps either side of, every E2M1 midpoint."""
    gen = torch.Generator().manual_seed(17)
    n = 1 << 22
    d = torch.exp2(torch.rand(n, generator=gen) * 200 - 100)
    x = (torch.rand(n, generator=gen) * 14 - 7) * d
    mids = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 6.0])
    dm = torch.exp2(torch.randint(-60, 60, (4096,), generator=gen).float()) * \
        (1 + torch.randint(0, 8, (4096,), generator=gen).float() / 8)
    xs, ds = [x], [d]
    for m in mids:
        base = (m * dm).view(torch.int32)
        for k in range(-3, 4):
            xs.append((base + k).view(torch.float32) * torch.where(torch.rand(4096, generator=gen) < 0.5, -1.0, 1.0))
            ds.append(dm)
    # subnormal x, subnormal-range d
    xs.append(torch.tensor([1e-45, -3e-40, 2.0 ** -126, -(2.0 ** -127) * 5]))
    ds.append(torch.tensor([1e-45, 2.0 ** -128, 2.0 ** -126, 2.0 ** -126]))
    X, D = torch.cat(xs), torch.cat(ds)
    keep = torch.isfinite(X / D) & (D > 0)
    X, D = X[keep].contiguous(), D[keep].contiguous()
    got = fp4.nv_encode_quotient(X.to(DEV), D.to(DEV)).cpu().numpy()
    v = X.numpy() / D.numpy()      # IEEE single division, as the oracle does
    assert np.array_equal(got, oracle.e2m1_encode_f32(v))


# --------------------------------------------------------------- whole path

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("shape", [(1, 32), (3, 64), (7, 96), (33, 1024), (129, 2080), (517, 4128)])
def test_parity_shapes(dtype, shape):
    w = workloads.with_shape(workloads.WEIGHT_4K, *shape, seed_offset=shape[0] * 7 + shape[1])
    check_full(workloads.generate(dataclasses.replace(w, dtype=dtype)))


def test_parity_nv_only_shape_cols_16():
    w = workloads.with_shape(workloads.WEIGHT_4K, 5, 48, seed_offset=3)
    check_full(workloads.generate(w), search=True)


def test_parity_tiny_f32_workload():
    check_full(workloads.generate(workloads.TINY_F32))


def test_parity_weight_4096_workload_full():
    check_full(workloads.generate(workloads.WEIGHT_4K), search=False)


def test_parity_weight_4096_search_sampled_rows():
    x = workloads.generate(workloads.WEIGHT_4K)
    ss = fp4.scale_search(x.to(DEV))
    torch.cuda.synchronize()
    ss.check()
    xo = odata(x)
    g = oracle.nv_global_scale(oracle.tensor_amax(xo))
    assert ss.global_scale.item() == g
    rows = workloads.sample_rows(x.shape[0], 24)
    p, s, loss = oracle.nvfp4_scale_search_with_g(np.ascontiguousarray(xo[rows]), g)
    assert_same(ss.packed[rows], p, "search packed")
    assert_same(ss.scales[rows], s, "search scales")
    assert_same(ss.block_loss[rows], loss.astype(np.float32), "search loss")


def test_parity_activation_8192x14336_sampled_rows():
    x = workloads.generate(workloads.ACT_8K)
    xd = x.to(DEV)
    res = run_all(xd, search=False)
    xo = odata(x)
    A = oracle.tensor_amax(xo)
    g = oracle.nv_global_scale(A)
    assert res["nv"].global_scale.item() == g
    rows = workloads.sample_rows(x.shape[0], 48)
    sub = np.ascontiguousarray(xo[rows])
    p, s = oracle.nvfp4_quantize_with_g(sub, g)
    assert_same(res["nv"].packed[rows], p, "NVFP4 packed")
    assert_same(res["nv"].scales[rows], s, "NVFP4 scales")
    assert_same_bits(res["ynv16"][rows], oracle.nvfp4_dequantize(p, s, g, len(rows), x.shape[1]), "NV dequant")
    p, s = oracle.mxfp4_quantize(sub)
    assert_same(res["mx"].packed[rows], p, "MXFP4 packed")
    assert_same(res["mx"].scales[rows], s, "MXFP4 scales")
    assert_same_bits(res["ymx16"][rows], oracle.mxfp4_dequantize(p, s, len(rows), x.shape[1]), "MX dequant")


def test_parity_search_4096x14336_sampled_rows_and_mse():
    x = workloads.generate(workloads.SEARCH_4K)
    ss = fp4.scale_search(x.to(DEV))
    nv = fp4.nvfp4_quantize(x.to(DEV))
    torch.cuda.synchronize()
    ss.check()
    xo = odata(x)
    g = oracle.nv_global_scale(oracle.tensor_amax(xo))
    assert ss.global_scale.item() == g
    rows = workloads.sample_rows(x.shape[0], 12)
    sub = np.ascontiguousarray(xo[rows])
    p, s, loss = oracle.nvfp4_scale_search_with_g(sub, g)
    assert_same(ss.scales[rows], s, "search scales")
    assert_same(ss.packed[rows], p, "search packed")
    assert_same(ss.block_loss[rows], loss.astype(np.float32), "search loss")
    # properties at full size: never worse than max-based, MSE within 1e-6
    l_search = ss.block_loss.double()
    yb = fp4.dequantize(nv, torch.float32).double()
    l_max = ((x.to(DEV).double() - yb) ** 2).reshape(-1, 16).sum(1).reshape(l_search.shape)
    assert bool((l_search <= l_max * (1 + 1e-6) + 1e-30).all())
    ys = fp4.dequantize(ss, torch.float32).double()
    mse = ((x.to(DEV).double() - ys) ** 2).mean().item()
    assert abs(mse - l_search.sum().item() / x.numel()) <= 1e-6 * mse


def test_parity_model_7b_layer0_full_and_all_matrices_sampled():
    for layer in range(workloads.MODEL_LAYERS):
        for idx in range(len(workloads.MODEL_MATRICES)):
            w = workloads.model_matrix(layer, idx)
            xd = workloads.generate(w, device=DEV)
            if layer == 0:
                check_full(xd.cpu(), search=False)
                continue
            res = run_all(xd, search=False)
            res["nv"].check()
            res["mx"].check()
            A = xd.abs().amax().float().item()
            g = oracle.nv_global_scale(A)
            assert res["nv"].global_scale.item() == g
            rows = workloads.sample_rows(w.rows, 2, seed=layer * 7 + idx)
            sub = odata(xd[rows].cpu())
            p, s = oracle.nvfp4_quantize_with_g(sub, g)
            assert_same(res["nv"].packed[rows], p, f"{w.name} NV packed")
            assert_same(res["nv"].scales[rows], s, f"{w.name} NV scales")
            p, s = oracle.mxfp4_quantize(sub)
            assert_same(res["mx"].packed[rows], p, f"{w.name} MX packed")
            assert_same(res["mx"].scales[rows], s, f"{w.name} MX scales")
            del xd, res


# ------------------------------------------------------------- edge cases

def test_pages_worked_examples_on_gpu():
    pattern = [0.0, 0.3, 0.6, 0.9, 1.2, 1.8, 2.4, 3.6]
    for blk in (pattern * 2, [0.4] * 15 + [3.6], [0.0] * 16, [1e-10] * 16, [-0.0] * 8 + [0.0] * 8):
        x = torch.tensor([[2688.0] * 16 + blk], dtype=torch.float32)
        check_full(x)
    res = run_all(torch.tensor([[2688.0] * 16 + pattern * 2], device=DEV))
    assert res["nv"].scales.cpu().tolist() == [[0x7E, 0x32]]
    assert res["ynv32"][0, 16:].cpu().tolist() == [0.0, 0.3125, 0.625, 0.9375, 1.25, 1.875, 2.5, 3.75] * 2


def test_edge_values():
    fmax = float(np.finfo(np.float32).max)
    rows = [
        [0.0] * 32,                                        # zero tensor rows
        [-0.0] * 32,
        [fmax, -fmax] + [1.0] * 30,                         # saturating magnitudes
        [1e-45, -1e-45, 2.0 ** -126, -(2.0 ** -127)] * 8,   # subnormals
        [7.0] + [0.0] * 31,                                 # MX clipping 7 -> 6
        [6.0] + [0.3] * 31,
        list(np.linspace(-3, 3, 32)),
    ]
    for r in rows:
        check_full(torch.tensor([r], dtype=torch.float32))
    check_full(torch.tensor(rows[2:], dtype=torch.float32))
    # bf16 extremes
    bmax = float(torch.finfo(torch.bfloat16).max)
    check_full(torch.tensor([[bmax, -bmax] + [1.0] * 30, [2.0 ** -133] * 32], dtype=torch.bfloat16))


def test_zero_tensor_and_empty():
    check_full(torch.zeros(4, 64))
    x = torch.zeros(0, 64, device=DEV)
    q = fp4.nvfp4_quantize(x)
    torch.cuda.synchronize()
    assert q.global_scale.item() == 1.0 and q.status.item() == 0


@pytest.mark.parametrize("bad", [float("nan"), float("inf"), -float("inf")])
def test_nonfinite_sets_status(bad):
    x = torch.randn(64, 256)
    x[37, 101] = bad
    for dt in (torch.float32, torch.bfloat16):
        xd = x.to(dt).to(DEV)
        for q in (fp4.nvfp4_quantize(xd), fp4.mxfp4_quantize(xd), fp4.scale_search(xd)):
            torch.cuda.synchronize()
            assert q.status.item() == fp4.ERR_NONFINITE
        a, st = fp4.tensor_amax(xd)
        torch.cuda.synchronize()
        assert st.item() == fp4.ERR_NONFINITE and not np.isfinite(a.item())


def test_global_scale_underflow_sets_range():
    x = torch.full((1, 16), 2.0 ** -149, dtype=torch.float32, device=DEV)
    for q in (fp4.nvfp4_quantize(x), fp4.scale_search(x)):
        torch.cuda.synchronize()
        assert q.status.item() == fp4.ERR_RANGE


def test_status_is_sticky_first_error_wins():
    st = fp4.new_status(DEV)
    bad = torch.full((1, 16), 2.0 ** -149, device=DEV)
    fp4.nvfp4_quantize(bad, status=st)
    nanx = torch.full((1, 32), float("nan"), device=DEV)
    fp4.mxfp4_quantize(nanx, status=st)
    fp4.nvfp4_quantize(torch.ones(1, 16, device=DEV), status=st)
    torch.cuda.synchronize()
    assert st.item() == fp4.ERR_RANGE


def test_tensor_amax_and_with_amax_variant():
    x = workloads.generate(workloads.with_shape(workloads.ACT_8K, 300, 4096)).to(DEV)
    a, st = fp4.tensor_amax(x)
    torch.cuda.synchronize()
    assert st.item() == 0 and a.item() == x.abs().amax().float().item()
    # subnormal and normal magnitudes mixed, both signs: the packed
    # sign-agnostic max must order subnormals like their magnitudes
    g = torch.Generator().manual_seed(11)
    for dt, lo, hi in ((torch.bfloat16, -133, -120), (torch.float32, -149, -120)):
        e = torch.randint(lo, hi, (4096,), generator=g).double()
        s = torch.where(torch.rand(4096, generator=g) < 0.5, -1.0, 1.0).double()
        y = (s * torch.exp2(e) * (1 + torch.rand(4096, generator=g).double() * 0.9)).to(dt)
        y[torch.randperm(4096, generator=g)[:9]] = 0.0
        a, st = fp4.tensor_amax(y.to(DEV))
        torch.cuda.synchronize()
        assert st.item() == 0 and a.item() == y.abs().amax().float().item()
        m = fp4.mxfp4_quantize(y.reshape(128, 32).to(DEV))
        torch.cuda.synchronize()
        p, sc = oracle.mxfp4_quantize(odata(y.reshape(128, 32)))
        assert_same(m.scales, sc, "MX scales on subnormals")
        assert_same(m.packed, p, "MX codes on subnormals")
    # odd element counts take the scalar tail
    for n in (1, 7, 8, 9, 1001):
        y = torch.randn(n, device=DEV).to(torch.bfloat16)
        a, st = fp4.tensor_amax(y)
        torch.cuda.synchronize()
        assert a.item() == y.abs().amax().float().item()
    q = fp4.nvfp4_quantize(x)
    amax = x.abs().amax().float().reshape(1)
    packed = torch.empty_like(q.packed)
    scales = torch.empty_like(q.scales)
    g = torch.empty(1, device=DEV)
    st = fp4.new_status(DEV)
    assert fp4.fp4_nvfp4_quantize_with_amax(x, amax, packed, scales, g, st) == 0
    torch.cuda.synchronize()
    assert torch.equal(packed, q.packed) and torch.equal(scales, q.scales) and g.item() == q.global_scale.item()
    assert fp4.fp4_nvfp4_quantize_with_amax(x, torch.tensor([float("inf")], device=DEV), packed, scales, g, st) == 0
    torch.cuda.synchronize()
    assert st.item() == fp4.ERR_NONFINITE


def test_dequant_foreign_scale_bytes():
    R, C = 2, 64
    packed = torch.randint(0, 256, (R, C // 2), dtype=torch.uint8)
    s_nv = torch.randint(0, 256, (R, C // 16), dtype=torch.uint8)
    s_nv[0, 0], s_nv[1, 1] = 0x7F, 0xFF
    s_mx = torch.randint(0, 256, (R, C // 32), dtype=torch.uint8)
    s_mx[0, 0], s_mx[1, 1] = 255, 0
    g = torch.tensor([0.0123], dtype=torch.float32)
    qn = fp4.Quantized(fp4.NVFP4, packed.to(DEV), s_nv.to(DEV), g.to(DEV), fp4.new_status(DEV), R, C)
    qm = fp4.Quantized(fp4.MXFP4, packed.to(DEV), s_mx.to(DEV), None, fp4.new_status(DEV), R, C)
    yn, ym = fp4.dequantize(qn, torch.float32), fp4.dequantize(qm, torch.float32)
    torch.cuda.synchronize()
    assert_same_bits(yn, oracle.nvfp4_dequantize(packed.numpy(), s_nv.numpy(), g.item(), R, C), "NV foreign")
    assert_same_bits(ym, oracle.mxfp4_dequantize(packed.numpy(), s_mx.numpy(), R, C), "MX foreign")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("grid", [(32, 16, 48), (8, 100, 100), (20, 40, 50), (5, 200, 160), (64, 147, 210),
                                  (1, 16, 16), (128, 16, 100), (3, 1000, 4096)])
def test_scale_search_grid_parity(dtype, grid):
    """The search over a caller's candidate grid (p + k) / q, k < n: codes,
    scales, g and the per-block loss bit for bit against the oracle's brute
    force over the same grid, including grids reaching above the max-based
    scale (saturating at 448) and the single max-based candidate."""
    w = workloads.with_shape(workloads.SEARCH_4K, 48, 512, 50 + grid[0])
    x = workloads.generate(w).to(dtype)
    q = fp4.scale_search(x.to(DEV), grid=grid)
    torch.cuda.synchronize()
    q.check()
    p, s, g, loss = oracle.nvfp4_scale_search_grid(odata(x), *grid)
    assert q.global_scale.item() == g
    assert_same(q.scales, s, f"grid {grid} scales")
    assert_same(q.packed, p, f"grid {grid} packed")
    with np.errstate(over="ignore"):
        loss32 = loss.astype(np.float32)
    assert_same(q.block_loss, loss32, f"grid {grid} block loss")


def test_scale_search_grid_arguments():
    L = fp4.lib()
    x = torch.randn(4, 64, device=DEV)
    pk = torch.empty(4 * 32, dtype=torch.uint8, device=DEV)
    sc = torch.empty(4 * 4, dtype=torch.uint8, device=DEV)
    g = torch.empty(1, dtype=torch.float32, device=DEV)
    ws = fp4.workspace_for(x)
    st = fp4.new_status(DEV)
    P = lambda t: t.data_ptr()  # noqa: E731
    for n, p, q in ((0, 147, 210), (64, 15, 210), (64, 147, 0), (2, 1 << 20, 4), (4, 16, (1 << 20) + 1)):
        assert L.fp4_scale_search_grid(P(x), fp4.F32, 4, 64, n, p, q, P(pk), P(sc), P(g), None, P(ws),
                                       ws.numel() * ws.element_size(), P(st), None) == fp4.ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert st.item() == 0
