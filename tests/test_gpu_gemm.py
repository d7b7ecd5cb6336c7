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


def run_gemm(pa, sa, ga, pb, sb, gb, M, N, K):
    qa = fp4.Quantized(fp4.NVFP4, torch.from_numpy(pa).to(DEV), torch.from_numpy(sa).to(DEV),
                       torch.tensor([ga], dtype=torch.float32, device=DEV), fp4.new_status(DEV), M, K)
    qb = fp4.Quantized(fp4.NVFP4, torch.from_numpy(pb).to(DEV), torch.from_numpy(sb).to(DEV),
                       torch.tensor([gb], dtype=torch.float32, device=DEV), fp4.new_status(DEV), N, K)
    st = fp4.new_status(DEV)
    d = fp4.nvfp4_gemm(qa, qb, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return d.cpu().numpy()


def test_grouped_dot_of_the_page_on_the_tensor_cores():
    gd = golden("grouped_dot.json")
    def codes(spec):
        out = []
        for value, count in spec:
            out += [oracle.e2m1_encode(value)] * count
        return out
    e4 = oracle.e4m3_encode
    M = N = 128
    K = 256
    pa, sa = operand(M, K, [codes(gd["px"])], [[e4(v) for v in gd["bx"]]])
    pb, sb = operand(N, K, [codes(gd["pw"])], [[e4(v) for v in gd["bw"]]])
    d = run_gemm(pa, sa, gd["ax"], pb, sb, gd["aw"], M, N, K)
    assert d[0, 0] == gd["group_result"]
    d[0, 0] = 0.0
    assert not d.any()


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (256, 384, 512), (384, 128, 1280)])
def test_gemm_matches_the_exact_product(M, N, K):
    g = torch.Generator().manual_seed(M + N + K)
    xa = torch.randn(M, K, generator=g) * torch.rand(M, 1, generator=g) * 3
    xb = torch.randn(N, K, generator=g) * 0.02
    xb.view(-1)[torch.randint(0, N * K, (N * K // 500,), generator=g)] *= 40
    qa = fp4.nvfp4_quantize(xa.to(torch.bfloat16).to(DEV))
    qb = fp4.nvfp4_quantize(xb.to(torch.bfloat16).to(DEV))
    st = fp4.new_status(DEV)
    d = fp4.nvfp4_gemm(qa, qb, status=st)
    torch.cuda.synchronize()
    qa.check()
    qb.check()
    assert st.item() == 0
    want, mag = oracle.nvfp4_gemm(qa.packed.cpu().numpy(), qa.scales.cpu().numpy(), qa.global_scale.item(),
                                  qb.packed.cpu().numpy(), qb.scales.cpu().numpy(), qb.global_scale.item(),
                                  M, N, K)
    err = np.abs(d.cpu().numpy().astype(np.float64) - want)
    assert (err <= tolerance(mag, K)).all(), f"max err {err.max()} vs tol {tolerance(mag, K).max()}"


def test_gemm_large_sampled_rows():
    M, N, K = 1024, 1024, 4096
    g = torch.Generator().manual_seed(5)
    xa = (torch.randn(M, K, generator=g) * 0.5).to(torch.bfloat16).to(DEV)
    xb = (torch.randn(N, K, generator=g) * 0.02).to(torch.bfloat16).to(DEV)
    qa, qb = fp4.nvfp4_quantize(xa), fp4.nvfp4_quantize(xb)
    d = fp4.nvfp4_gemm(qa, qb)
    torch.cuda.synchronize()
    rows = [0, 1, 127, 128, 500, 1023]
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
