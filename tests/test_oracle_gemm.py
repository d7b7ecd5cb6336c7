"""Oracle pins for the consumer of the quantised operands: the block-scaled
matrix product ("NVFP4 与 MXFP4 格式" section 6) and the tiled scale layout
the tensor-core MMA reads."""
import numpy as np
import pytest

from conftest import golden


def page_operands(o):
    gd = golden("grouped_dot.json")
    def codes(spec):
        out = []
        for value, count in spec:
            out += [o.e2m1_encode(value)] * count
        return out
    pa = np.frombuffer(o.pack4(codes(gd["px"])), np.uint8).reshape(1, 16)
    pb = np.frombuffer(o.pack4(codes(gd["pw"])), np.uint8).reshape(1, 16)
    sa = np.array([[o.e4m3_encode(v) for v in gd["bx"]]], np.uint8)
    sb = np.array([[o.e4m3_encode(v) for v in gd["bw"]]], np.uint8)
    return gd, pa, sa, pb, sb


def test_grouped_dot_of_the_page(oracle_mod):
    o = oracle_mod
    gd, pa, sa, pb, sb = page_operands(o)
    d, mag = o.nvfp4_gemm(pa, sa, gd["ax"], pb, sb, gd["aw"], 1, 1, 32)
    assert d[0, 0] == gd["group_result"]
    # taking the first block's scales for the whole K is the page's wrong result
    sa1 = np.array([[sa[0, 0], sa[0, 0]]], np.uint8)
    sb1 = np.array([[sb[0, 0], sb[0, 0]]], np.uint8)
    d1, _ = o.nvfp4_gemm(pa, sa1, gd["ax"], pb, sb1, gd["aw"], 1, 1, 32)
    assert d1[0, 0] == gd["wrong_result"]


def test_gemm_is_the_product_of_the_dequantised_operands(oracle_mod):
    """D equals x_hat_A x_hat_B^T with x_hat = p s_b g formed in double."""
    o = oracle_mod
    rng = np.random.default_rng(3)
    M, N, K = 5, 7, 96
    xa = rng.standard_normal((M, K)).astype(np.float32)
    xb = (rng.standard_normal((N, K)) * 0.01).astype(np.float32)
    pa, sa, ga = o.nvfp4_quantize(xa)
    pb, sb, gb = o.nvfp4_quantize(xb)

    def deq(p, s, g, R, C):
        codes = np.array(o.unpack4(p.tobytes()), np.int64).reshape(R, C)
        vals = np.array([o.e2m1_decode(int(c)) for c in range(16)])[codes]
        sc = np.array([o.e4m3_decode_byte(int(b)) for b in range(256)])[s.astype(np.int64)]
        return vals * np.repeat(sc, 16, axis=1) * g

    want = deq(pa, sa, ga, M, K) @ deq(pb, sb, gb, N, K).T
    d, mag = o.nvfp4_gemm(pa, sa, ga, pb, sb, gb, M, N, K)
    assert np.allclose(d, want, rtol=1e-12, atol=1e-12 * np.abs(want).max())
    assert (mag >= np.abs(d) * (1 - 1e-12)).all()


def test_scales_mma_layout_positions(oracle_mod):
    """The pages do not give this layout (it is the sm100 block-scaled MMA's
    operand layout), so nothing here can pin it to them: this test only
    restates the oracle's index formula and checks the padding.  The layout's
    real anchor is the tensor-core product in the GPU GEMM tests, which reads
    these bytes: a wrong byte order there gives a wrong D."""
    o = oracle_mod
    rows, nb = 130, 5
    s = (np.arange(rows * nb) % 251 + 1).astype(np.uint8).reshape(rows, nb)
    out = o.scales_mma_layout(s)
    kt, rt = 2, 2
    assert out.size == rt * kt * 512
    for r in range(rows):
        for j in range(nb):
            tile = (r // 128) * kt + j // 4
            rr = r % 128
            assert out[tile * 512 + (rr % 32) * 16 + (rr // 32) * 4 + j % 4] == s[r, j]
    # every written byte is one of the inputs; the padding is zero
    assert np.count_nonzero(out) == rows * nb
