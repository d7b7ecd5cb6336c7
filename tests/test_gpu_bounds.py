"""Out-of-bounds writes: every entry point writes its outputs and nothing
next to them.

Each output (and each workspace) lives inside one larger buffer with 256
sentinel bytes before and after it, filled with a byte pattern; after the
call (and a device synchronise) the sentinels must be untouched and the
output must equal the output of the same call on plain tensors, which the
parity tests check against the oracle.  Shapes are small and ragged (row
counts that fill no grid evenly, rows one block long, the padded layouts'
tail blocks), and every case also runs with the launch size limited to 128
units, so that every kernel is split into several launches whose edges
fall inside the tensor.
"""
import ctypes
import math

import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4

pytestmark = pytest.mark.gpu
DEV = "cuda"
PAD = 256


class Guarded:
    """A device tensor of `shape` and `dtype` at byte `offset` past PAD
    sentinel bytes, with PAD sentinel bytes after it."""

    def __init__(self, shape, dtype, fill: int, offset: int = 0):
        esz = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape) * esz
        self.fill = fill
        self.off = PAD + offset
        self.buf = torch.full((self.off + self.n + PAD,), fill, dtype=torch.uint8, device=DEV)
        self.t = self.buf[self.off:self.off + self.n].view(dtype).reshape(shape)

    @property
    def ptr(self):
        return ctypes.c_void_p(self.t.data_ptr())

    def check(self, what: str):
        pre, post = self.buf[:self.off], self.buf[self.off + self.n:]
        bad_pre = torch.nonzero(pre != self.fill).flatten()
        bad_post = torch.nonzero(post != self.fill).flatten()
        assert bad_pre.numel() == 0, f"{what}: bytes written before the buffer at {bad_pre[:8].tolist()}"
        assert bad_post.numel() == 0, f"{what}: bytes written after the buffer at {bad_post[:8].tolist()}"


def rand(R, C, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(R, C, generator=g) * 0.05
    if R * C:
        x.view(-1)[torch.randint(0, R * C, (max(1, R * C // 200),), generator=g)] *= 40
    return x.to(dtype).to(DEV)


def stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


@pytest.fixture(params=[0, 128], ids=["one-launch", "launch-limit-128"])
def launch_limit(request):
    L = fp4.lib()
    assert L.fp4_set_launch_unit_limit(request.param) == fp4.OK
    yield request.param
    assert L.fp4_set_launch_unit_limit(0) == fp4.OK


FILLS = (0xA5, 0x5A)
ROW_SHAPES = [(1, 32), (3, 64), (37, 1056), (130, 544), (257, 96)]
DTYPES = [torch.bfloat16, torch.float32]


def new_status():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def ws_bytes():
    return fp4.lib().fp4_workspace_bytes(fp4.NVFP4, 1, 1)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", ROW_SHAPES)
def test_row_quantisers_and_dequantisers(shape, dtype, launch_limit):
    L = fp4.lib()
    R, C = shape
    x = rand(R, C, dtype, seed=R * 7 + C)
    dt = fp4._dtype_code(x)
    ref_nv = fp4.nvfp4_quantize(x)
    ref_mx = fp4.mxfp4_quantize(x)
    ref_mxc = fp4.mxfp4_quantize_ceil(x)
    ref_ss = fp4.scale_search(x)
    ref_46 = fp4.nvfp4_quantize_four_over_six(x)
    for fill in FILLS:
        # NVFP4 quantise (its workspace guarded too)
        p, s, g = Guarded((R, C // 2), torch.uint8, fill), Guarded((R, C // 16), torch.uint8, fill), \
            Guarded((1,), torch.float32, fill)
        ws = Guarded((ws_bytes(),), torch.uint8, fill)
        ws.t.zero_()
        st = new_status()
        assert L.fp4_nvfp4_quantize(x.data_ptr(), dt, R, C, p.ptr, s.ptr, g.ptr, ws.ptr, ws.n, st.data_ptr(),
                                    stream()) == fp4.OK
        torch.cuda.synchronize()
        for b, what in ((p, "nv packed"), (s, "nv scales"), (g, "nv g"), (ws, "nv workspace")):
            b.check(what)
        assert torch.equal(p.t, ref_nv.packed) and torch.equal(s.t, ref_nv.scales) and torch.equal(g.t, ref_nv.global_scale)
        # NVFP4 without a workspace
        p2, s2, g2 = Guarded((R, C // 2), torch.uint8, fill), Guarded((R, C // 16), torch.uint8, fill), \
            Guarded((1,), torch.float32, fill)
        assert L.fp4_nvfp4_quantize_noalloc(x.data_ptr(), dt, R, C, p2.ptr, s2.ptr, g2.ptr, st.data_ptr(),
                                            stream()) == fp4.OK
        torch.cuda.synchronize()
        for b, what in ((p2, "noalloc packed"), (s2, "noalloc scales"), (g2, "noalloc g")):
            b.check(what)
        assert torch.equal(p2.t, ref_nv.packed) and torch.equal(s2.t, ref_nv.scales)
        # tensor amax alone
        a = Guarded((1,), torch.float32, fill)
        assert L.fp4_tensor_amax(x.data_ptr(), dt, R * C, a.ptr, ws.ptr, ws.n, st.data_ptr(), stream()) == fp4.OK
        torch.cuda.synchronize()
        a.check("amax")
        ws.check("amax workspace")
        assert a.t.item() == x.float().abs().max().item()
        # MXFP4, both scale rules
        for fn, ref, what in ((L.fp4_mxfp4_quantize, ref_mx, "mx"), (L.fp4_mxfp4_quantize_ceil, ref_mxc, "mx ceil")):
            p, s = Guarded((R, C // 2), torch.uint8, fill), Guarded((R, C // 32), torch.uint8, fill)
            assert fn(x.data_ptr(), dt, R, C, p.ptr, s.ptr, st.data_ptr(), stream()) == fp4.OK
            torch.cuda.synchronize()
            p.check(what + " packed")
            s.check(what + " scales")
            assert torch.equal(p.t, ref.packed) and torch.equal(s.t, ref.scales)
        # scale search and four over six, with the per-block loss
        for fn, ref, what in ((L.fp4_scale_search, ref_ss, "search"),
                              (L.fp4_nvfp4_quantize_four_over_six, ref_46, "four over six")):
            p, s, g = Guarded((R, C // 2), torch.uint8, fill), Guarded((R, C // 16), torch.uint8, fill), \
                Guarded((1,), torch.float32, fill)
            lo = Guarded((R, C // 16), torch.float32, fill)
            assert fn(x.data_ptr(), dt, R, C, p.ptr, s.ptr, g.ptr, lo.ptr, ws.ptr, ws.n, st.data_ptr(),
                      stream()) == fp4.OK
            torch.cuda.synchronize()
            for b, w in ((p, "packed"), (s, "scales"), (g, "g"), (lo, "block loss"), (ws, "workspace")):
                b.check(f"{what} {w}")
            assert torch.equal(p.t, ref.packed) and torch.equal(s.t, ref.scales)
            assert torch.equal(lo.t, ref.block_loss)
        assert st.item() == fp4.OK
        # dequantisation, both formats, both output types
        for q in (ref_nv, ref_mx):
            for out_dt in DTYPES:
                y = Guarded((R, C), out_dt, fill)
                assert L.fp4_dequantize(q.fmt, q.packed.data_ptr(), q.scales.data_ptr(),
                                        q.global_scale.data_ptr() if q.global_scale is not None else None,
                                        R, C, y.ptr, fp4._dtype_code(y.t), stream()) == fp4.OK
                torch.cuda.synchronize()
                y.check(f"dequant fmt {q.fmt} {out_dt}")
                assert torch.equal(y.t.view(torch.uint8), fp4.dequantize(q, out_dt).view(torch.uint8))


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("shape", [(1, 1), (3, 17), (37, 1041), (130, 529), (65, 40)])
def test_padded_and_column_layouts(shape, dtype, launch_limit):
    L = fp4.lib()
    R, K = shape
    x = rand(R, K, dtype, seed=R * 11 + K)
    dt = fp4._dtype_code(x)
    pad = lambda n, gsz: -(-n // gsz) * gsz  # noqa: E731
    refs = {"nv": fp4.nvfp4_quantize_padded(x), "mx": fp4.mxfp4_quantize_padded(x, fp4.MX_FLOOR)}
    columns = (K * (2 if dtype == torch.bfloat16 else 4)) % 4 == 0  # rows of whole 4-byte words
    refs["nva"] = refs["nv"]  # the same outputs from the _with_amax call
    if columns:
        refs["nvc"] = fp4.nvfp4_quantize_columns(x)
        refs["mxc"] = fp4.mxfp4_quantize_columns(x, fp4.MX_CEIL)
        refs["nvca"] = refs["nvc"]
    amax, _ = fp4.tensor_amax(x)
    st = new_status()
    for fill in FILLS:
        ws = Guarded((ws_bytes(),), torch.uint8, fill)
        ws.t.zero_()
        for key, ref in refs.items():
            OR, OC = (K, R) if key in ("nvc", "mxc", "nvca") else (R, K)
            G = 16 if key.startswith("nv") else 32
            p = Guarded((OR, pad(OC, G) // 2), torch.uint8, fill)
            s = Guarded((OR, pad(OC, G) // G), torch.uint8, fill)
            g = Guarded((1,), torch.float32, fill)
            if key == "nv":
                rc = L.fp4_nvfp4_quantize_padded(x.data_ptr(), dt, R, K, p.ptr, s.ptr, g.ptr, ws.ptr, ws.n,
                                                 st.data_ptr(), stream())
            elif key == "mx":
                rc = L.fp4_mxfp4_quantize_padded(x.data_ptr(), dt, R, K, fp4.MX_FLOOR, p.ptr, s.ptr,
                                                 st.data_ptr(), stream())
            elif key == "nva":
                rc = L.fp4_nvfp4_quantize_padded_with_amax(x.data_ptr(), dt, R, K, amax.data_ptr(), p.ptr, s.ptr,
                                                           g.ptr, st.data_ptr(), stream())
            elif key == "nvca":
                rc = L.fp4_nvfp4_quantize_columns_with_amax(x.data_ptr(), dt, R, K, amax.data_ptr(), p.ptr, s.ptr,
                                                            g.ptr, st.data_ptr(), stream())
            elif key == "nvc":
                rc = L.fp4_nvfp4_quantize_columns(x.data_ptr(), dt, R, K, p.ptr, s.ptr, g.ptr, ws.ptr, ws.n,
                                                  st.data_ptr(), stream())
            else:
                rc = L.fp4_mxfp4_quantize_columns(x.data_ptr(), dt, R, K, fp4.MX_CEIL, p.ptr, s.ptr,
                                                  st.data_ptr(), stream())
            assert rc == fp4.OK
            torch.cuda.synchronize()
            for b, w in ((p, "packed"), (s, "scales"), (g, "g"), (ws, "workspace")):
                b.check(f"{key} {w}")
            assert torch.equal(p.t, ref.packed) and torch.equal(s.t, ref.scales)
            # dequantise the padded layout into a y at an odd element offset
            for out_dt in DTYPES:
                esz = 2 if out_dt == torch.bfloat16 else 4
                y = Guarded((OR, OC), out_dt, fill, offset=esz)
                rc = L.fp4_dequantize_padded(ref.fmt, ref.packed.data_ptr(), ref.scales.data_ptr(),
                                             ref.global_scale.data_ptr() if ref.global_scale is not None else None,
                                             OR, OC, y.ptr, fp4._dtype_code(y.t), stream())
                assert rc == fp4.OK
                torch.cuda.synchronize()
                y.check(f"{key} padded dequant {out_dt}")
                assert torch.equal(y.t.view(torch.uint8), fp4.dequantize_padded(ref, out_dt).view(torch.uint8))
        assert st.item() == fp4.OK


@pytest.mark.parametrize("dtype", DTYPES)
def test_grouped_calls(dtype, launch_limit):
    L = fp4.lib()
    shapes = [(3, 64), (1, 32), (130, 544), (0, 64), (37, 1056)]
    xs = [rand(r, c, dtype, seed=r + c) for r, c in shapes]
    dt = fp4._dtype_code(xs[0])
    refs_nv = [fp4.nvfp4_quantize(x) if x.numel() else None for x in xs]
    refs_mx = [fp4.mxfp4_quantize(x) if x.numel() else None for x in xs]
    st = new_status()
    for fill in FILLS:
        k = len(xs)
        ws = Guarded((L.fp4_grouped_workspace_bytes(k),), torch.uint8, fill)
        outs = {}
        items_nv, items_mx = (fp4.QuantItem * k)(), (fp4.QuantItem * k)()
        for i, ((r, c), x) in enumerate(zip(shapes, xs)):
            o = outs[i] = {"nvp": Guarded((r, c // 2), torch.uint8, fill), "nvs": Guarded((r, c // 16), torch.uint8, fill),
                           "g": Guarded((1,), torch.float32, fill), "mxp": Guarded((r, c // 2), torch.uint8, fill),
                           "mxs": Guarded((r, c // 32), torch.uint8, fill)}
            items_nv[i] = fp4.QuantItem(x.data_ptr(), r, c, o["nvp"].t.data_ptr(), o["nvs"].t.data_ptr(),
                                        o["g"].t.data_ptr())
            items_mx[i] = fp4.QuantItem(x.data_ptr(), r, c, o["mxp"].t.data_ptr(), o["mxs"].t.data_ptr(), None)
        cp = lambda a: ctypes.cast(a, ctypes.c_void_p)  # noqa: E731
        assert L.fp4_nvfp4_quantize_grouped(cp(items_nv), k, dt, ws.ptr, ws.n, st.data_ptr(), stream()) == fp4.OK
        assert L.fp4_mxfp4_quantize_grouped(cp(items_mx), k, dt, st.data_ptr(), stream()) == fp4.OK
        torch.cuda.synchronize()
        ws.check("grouped workspace")
        for i, o in outs.items():
            for key, b in o.items():
                b.check(f"grouped item {i} {key}")
            if refs_nv[i] is not None:
                assert torch.equal(o["nvp"].t, refs_nv[i].packed) and torch.equal(o["nvs"].t, refs_nv[i].scales)
                assert torch.equal(o["g"].t, refs_nv[i].global_scale)
                assert torch.equal(o["mxp"].t, refs_mx[i].packed) and torch.equal(o["mxs"].t, refs_mx[i].scales)
        for fmt, refs in ((fp4.NVFP4, refs_nv), (fp4.MXFP4, refs_mx)):
            for out_dt in DTYPES:
                items = (fp4.DequantItem * k)()
                ys = []
                for i, ((r, c), q) in enumerate(zip(shapes, refs)):
                    y = Guarded((r, c), out_dt, fill)
                    ys.append(y)
                    if q is None:
                        items[i] = fp4.DequantItem(None, None, None, y.t.data_ptr(), r, c)
                    else:
                        items[i] = fp4.DequantItem(q.packed.data_ptr(), q.scales.data_ptr(),
                                                   q.global_scale.data_ptr() if q.global_scale is not None else None,
                                                   y.t.data_ptr(), r, c)
                assert L.fp4_dequantize_grouped(fmt, cp(items), k, fp4._dtype_code(ys[0].t), stream()) == fp4.OK
                torch.cuda.synchronize()
                for i, (y, q) in enumerate(zip(ys, refs)):
                    y.check(f"grouped dequant fmt {fmt} item {i} {out_dt}")
                    if q is not None:
                        assert torch.equal(y.t.view(torch.uint8), fp4.dequantize(q, out_dt).view(torch.uint8))
        assert st.item() == fp4.OK


@pytest.mark.parametrize("rows,blocks", [(1, 1), (37, 5), (130, 33), (256, 64)])
def test_scales_to_mma_layout(rows, blocks):
    L = fp4.lib()
    g = torch.Generator().manual_seed(rows * 3 + blocks)
    s = torch.randint(1, 255, (rows, blocks), generator=g, dtype=torch.uint8).to(DEV)
    ref = fp4.scales_to_mma(s)
    for fill in FILLS:
        out = Guarded((L.fp4_mma_scales_bytes(rows, blocks),), torch.uint8, fill)
        assert L.fp4_scales_to_mma_layout(s.data_ptr(), rows, blocks, out.ptr, stream()) == fp4.OK
        torch.cuda.synchronize()
        out.check("mma scale layout")
        assert torch.equal(out.t, ref)


@pytest.mark.parametrize("kernel", [fp4.GEMM_CTA, fp4.GEMM_CTA_PAIR])
def test_gemm_output(kernel):
    L = fp4.lib()
    M, N, K = 256, 256, 512
    qa = fp4.nvfp4_quantize(rand(M, K, torch.bfloat16, 1))
    qb = fp4.nvfp4_quantize(rand(N, K, torch.bfloat16, 2))
    sa, sb = fp4.scales_to_mma(qa.scales), fp4.scales_to_mma(qb.scales)
    ref = fp4.nvfp4_gemm(qa, qb, kernel=kernel)
    st = new_status()
    for fill in FILLS:
        d = Guarded((M, N), torch.float32, fill)
        rc = L.fp4_nvfp4_gemm_ex(qa.packed.data_ptr(), sa.data_ptr(), qa.global_scale.data_ptr(),
                                 qb.packed.data_ptr(), sb.data_ptr(), qb.global_scale.data_ptr(), M, N, K,
                                 d.ptr, kernel, st.data_ptr(), stream())
        assert rc == fp4.OK
        torch.cuda.synchronize()
        d.check("gemm D")
        assert st.item() == fp4.OK
        assert torch.equal(d.t, ref)
