"""The consumer on the tensor cores: the tiled MMA scale layout (bit for
bit against the oracle) and the block-scaled NVFP4 product (against the
oracle's exact product, to fp32 accumulation accuracy), with the grouped
dot of "NVFP4 与 MXFP4 格式" section 6 as the pinned case."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
from conftest import golden

pytestmark = pytest.mark.gpu
DEV = "cuda"


def tolerance(mag: np.ndarray, K: int) -> np.ndarray:
    """fp32 accumulation of K/16 scaled block sums, the two global scales
    and the final product: at most (K/16 + 8) units of 2^-23 of the sum of
    the magnitudes of the terms."""
    return (K / 16 + 8) * 2.0 ** -23 * mag + 1e-30


@pytest.mark.parametrize("shape", [(1, 1), (128, 4), (130, 5), (256, 16), (333, 100)])
def test_scales_mma_layout_parity(shape):
    g = torch.Generator().manual_seed(shape[0] * 7 + shape[1])
    s = torch.randint(0, 255, shape, generator=g, dtype=torch.uint8)
    got = fp4.scales_to_mma(s.to(DEV))
    torch.cuda.synchronize()
    assert np.array_equal(got.cpu().numpy(), oracle.scales_mma_layout(s.numpy()))


def operand(rows, K, codes_rows, scale_rows):
    """Packed [rows, K/2] and scales [rows, K/16] with the given first rows."""
    p = np.zeros((rows, K // 2), np.uint8)
    s = np.zeros((rows, K // 16), np.uint8)
    for r, codes in enumerate(codes_rows):
        b = np.frombuffer(oracle.pack4(codes), np.uint8)
        p[r, :b.size] = b
    for r, sc in enumerate(scale_rows):
        s[r, :len(sc)] = sc
    return p, s


def run_gemm(pa, sa, ga, pb, sb, gb, M, N, K, kernel=fp4.GEMM_AUTO):
    qa = fp4.Quantized(fp4.NVFP4, torch.from_numpy(pa).to(DEV), torch.from_numpy(sa).to(DEV),
                       torch.tensor([ga], dtype=torch.float32, device=DEV), fp4.new_status(DEV), M, K)
    qb = fp4.Quantized(fp4.NVFP4, torch.from_numpy(pb).to(DEV), torch.from_numpy(sb).to(DEV),
                       torch.tensor([gb], dtype=torch.float32, device=DEV), fp4.new_status(DEV), N, K)
    st = fp4.new_status(DEV)
    d = fp4.nvfp4_gemm(qa, qb, status=st, kernel=kernel)
    torch.cuda.synchronize()
    assert st.item() == 0
    return d.cpu().numpy()


@pytest.mark.parametrize("kernel,size", [(fp4.GEMM_CTA, 128), (fp4.GEMM_CTA_PAIR, 256)])
@pytest.mark.parametrize("where", ["first", "last"])
def test_grouped_dot_of_the_page_on_the_tensor_cores(kernel, size, where):
    """The page's worked group (two 16-element blocks) as one row of A and
    one row of B; every other element is zero, so D holds the group's value
    at one place and zeros elsewhere.  "last" puts it in the last row of A
    and of B (the second CTA of a pair, the second half of its columns)."""
    gd = golden("grouped_dot.json")
    def codes(spec):
        out = []
        for value, count in spec:
            out += [oracle.e2m1_encode(value)] * count
        return out
    e4 = oracle.e4m3_encode
    M = N = size
    K = 256
    pa, sa = operand(M, K, [codes(gd["px"])], [[e4(v) for v in gd["bx"]]])
    pb, sb = operand(N, K, [codes(gd["pw"])], [[e4(v) for v in gd["bw"]]])
    r = 0 if where == "first" else size - 1
    if r:
        pa, sa, pb, sb = (np.roll(a, r, axis=0) for a in (pa, sa, pb, sb))
    d = run_gemm(pa, sa, gd["ax"], pb, sb, gd["aw"], M, N, K, kernel)
    assert d[r, r] == gd["group_result"]
    d[r, r] = 0.0
    assert not d.any()


CTA_SHAPES = [(128, 128, 256), (256, 384, 512), (384, 128, 1280)]
PAIR_SHAPES = [(256, 256, 256), (512, 768, 1024), (256, 512, 2560), (768, 256, 512)]


@pytest.mark.parametrize("M,N,K,kernel", [s + (fp4.GEMM_CTA,) for s in CTA_SHAPES] +
                         [s + (fp4.GEMM_CTA_PAIR,) for s in PAIR_SHAPES] +
                         [(512, 768, 1024, fp4.GEMM_CTA)])
def test_gemm_matches_the_exact_product(M, N, K, kernel):
    g = torch.Generator().manual_seed(M + N + K)
    xa = torch.randn(M, K, generator=g) * torch.rand(M, 1, generator=g) * 3
    xb = torch.randn(N, K, generator=g) * 0.02
    xb.view(-1)[torch.randint(0, N * K, (N * K // 500,), generator=g)] *= 40
    qa = fp4.nvfp4_quantize(xa.to(torch.bfloat16).to(DEV))
    qb = fp4.nvfp4_quantize(xb.to(torch.bfloat16).to(DEV))
    st = fp4.new_status(DEV)
    d = fp4.nvfp4_gemm(qa, qb, status=st, kernel=kernel)
    torch.cuda.synchronize()
    qa.check()
    qb.check()
    assert st.item() == 0
    want, mag = oracle.nvfp4_gemm(qa.packed.cpu().numpy(), qa.scales.cpu().numpy(), qa.global_scale.item(),
                                  qb.packed.cpu().numpy(), qb.scales.cpu().numpy(), qb.global_scale.item(),
                                  M, N, K)
    err = np.abs(d.cpu().numpy().astype(np.float64) - want)
    assert (err <= tolerance(mag, K)).all(), f"max err {err.max()} vs tol {tolerance(mag, K).max()}"


@pytest.mark.parametrize("M,N,K,kernel", [(1024, 1024, 4096, fp4.GEMM_CTA),
                                           (1024, 1024, 4096, fp4.GEMM_CTA_PAIR),
                                           (4096, 4096, 512, fp4.GEMM_CTA_PAIR)])
def test_gemm_large_sampled_rows(M, N, K, kernel):
    """Sampled rows against the exact product; 4096 x 4096 gives the pair
    kernel 256 tiles, more than there are SM pairs, so clusters take several
    tiles each (the persistent loop and the accumulator hand-over)."""
    g = torch.Generator().manual_seed(5)
    xa = (torch.randn(M, K, generator=g) * 0.5).to(torch.bfloat16).to(DEV)
    xb = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    qa, qb = fp4.nvfp4_quantize(xa), fp4.nvfp4_quantize(xb)
    st = fp4.new_status(DEV)
    d = fp4.nvfp4_gemm(qa, qb, status=st, kernel=kernel)
    torch.cuda.synchronize()
    assert st.item() == 0
    rows = sorted({0, 1, 127, 128, 255, 256, 500, M // 2 + 129, M - 1})
    pa = qa.packed.cpu().numpy()[rows]
    sa = qa.scales.cpu().numpy()[rows]
    want, mag = oracle.nvfp4_gemm(pa, sa, qa.global_scale.item(), qb.packed.cpu().numpy(),
                                  qb.scales.cpu().numpy(), qb.global_scale.item(), len(rows), N, K)
    err = np.abs(d.cpu().numpy()[rows].astype(np.float64) - want)
    assert (err <= tolerance(mag, K)).all()


def test_gemm_argument_errors():
    q = fp4.nvfp4_quantize(torch.randn(128, 320, device=DEV))  # K = 320 is not a multiple of 256
    with pytest.raises(fp4.FP4Error) as e:
        fp4.nvfp4_gemm(q, q)
    assert e.value.status == fp4.ERR_SHAPE


def test_pair_kernel_shape_and_argument_errors():
    q = fp4.nvfp4_quantize(torch.randn(384, 256, device=DEV))  # 384 is not a multiple of 256
    with pytest.raises(fp4.FP4Error) as e:
        fp4.nvfp4_gemm(q, q, kernel=fp4.GEMM_CTA_PAIR)
    assert e.value.status == fp4.ERR_SHAPE
    d = fp4.nvfp4_gemm(q, q, kernel=fp4.GEMM_AUTO)  # falls back to one CTA per tile
    torch.cuda.synchronize()
    assert d.shape == (384, 384)
    with pytest.raises(fp4.FP4Error) as e:
        fp4.nvfp4_gemm(q, q, kernel=7)
    assert e.value.status == fp4.ERR_INVALID_ARG
