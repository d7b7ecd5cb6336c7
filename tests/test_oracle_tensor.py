"""Pins of the oracle's tensor-level NVFP4 / MXFP4 / dequant / scale-search
paths against the worked examples and printed numbers of the pages, closed
forms and invariants that a dropped term, a wrong sign or index or a
transposed operand would break.

Pages: "NVFP4 与 MXFP4 格式" (charlestar.github.io) §3-§8; "FP4 / NVFP4
数学总结" (devpress.csdn.net) §5, §7-§10; FP4 glossary (ultralytics.com,
"Come funziona FP4").
"""
import math
import struct
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads
from conftest import golden


def f32(v):
    return struct.unpack("f", struct.pack("f", v))[0]


def expand(spec):
    out = []
    for v, n in spec:
        out += [v] * n
    return out


def nv_codes(packed: np.ndarray) -> np.ndarray:
    p = packed.reshape(-1)
    return np.stack([p & 15, p >> 4], axis=1).reshape(-1)


# ------------------------------------------------------------ worked ------

def test_worked_block_alpha_0155(oracle_mod):
    gd = golden("worked_block_alpha_0155.json")
    alpha = f32(gd["alpha"])
    assert f32(gd["amax"] / 6) == alpha or abs(gd["amax"] / 6 - alpha) < 1e-7
    codes = [oracle_mod.e2m1_encode(f32(f32(x) / alpha)) for x in gd["x"]]
    q = [oracle_mod.e2m1_decode(c) for c in codes]
    assert q == [float(v) for v in gd["q"]]
    xhat = [round(v * gd["alpha"], gd["x_hat_printed_decimals"]) for v in q]
    assert xhat == gd["x_hat"]


def test_worked_scale_0p2(oracle_mod):
    gd = golden("worked_scale_0p2.json")
    v = f32(f32(gd["x"]) / f32(gd["scale"]))
    assert abs(v - gd["normalised"]) < 1e-6
    q = oracle_mod.e2m1_decode(oracle_mod.e2m1_encode(v))
    assert q == gd["q"]
    assert abs(q * gd["scale"] - gd["x_hat"]) < 1e-12
    assert abs((q * gd["scale"] - gd["x"]) - gd["error"]) < 1e-12


# -------------------------------------------------------------- NVFP4 -----

def _reconstruct_real_scale(oracle_mod, values, scale):
    return [scale * oracle_mod.e2m1_decode(oracle_mod.e2m1_encode(v / scale)) for v in values]


def test_nv_pipeline_pattern(oracle_mod):
    gd = golden("nv_pipeline_pattern.json")
    forcing = [gd["forcing_block"][0]] * gd["forcing_block"][1]
    x = np.array(forcing + gd["pattern"] * 2, np.float32)
    packed, scales, g = oracle_mod.nvfp4_quantize(x)
    assert g == gd["global_scale"]
    assert oracle_mod.e4m3_value(int(scales[0, 0])) == 448.0
    assert oracle_mod.e4m3_value(int(scales[0, 1])) == gd["e4m3_scale"]
    assert scales.tolist() == [[0x7E, 0x32]]
    y = oracle_mod.nvfp4_dequantize(packed, scales, g, 1, 32)[0]
    assert y[:16].tolist() == forcing
    assert y[16:].tolist() == gd["reconstruction_at_0625"] * 2
    mse = float(np.mean((y[16:].astype(np.float64) - x[16:].astype(np.float64)) ** 2))
    # inputs are fp32 roundings of the page's decimals: ~1e-7 relative
    assert mse == pytest.approx(gd["mse"]["0.625"], rel=1e-6)
    # the page's real-valued comparison scales (double arithmetic)
    pat = gd["pattern"]
    for s, want in gd["mse"].items():
        r = _reconstruct_real_scale(oracle_mod, pat, float(s))
        m = sum((a - b) ** 2 for a, b in zip(pat, r)) / len(pat)
        assert m == pytest.approx(want, rel=1e-12, abs=1e-28)
    assert _reconstruct_real_scale(oracle_mod, pat, 1.0) == gd["reconstruction_at_1"]


def test_nv_counterexample(oracle_mod):
    gd = golden("nv_counterexample.json")
    forcing = [gd["forcing_block"][0]] * gd["forcing_block"][1]
    blk = expand(gd["block"])
    x = np.array(forcing + blk, np.float32)
    packed, scales, g = oracle_mod.nvfp4_quantize(x)
    assert g == 1.0 and oracle_mod.e4m3_value(int(scales[0, 1])) == gd["max_based_scale"]
    y = oracle_mod.nvfp4_dequantize(packed, scales, g, 1, 32)[0, 16:]
    assert sorted(set(y.tolist())) == gd["reconstruction_max_based"]
    num, den = gd["mse_max_based"]
    xb = np.array(blk, np.float32)
    assert oracle_mod.nv_block_loss(xb, int(scales[0, 1]), g) / 16 == pytest.approx(num / den, rel=1e-6)
    alt = oracle_mod.e4m3_encode(gd["alternative_scale"])
    assert oracle_mod.e4m3_value(alt) == gd["alternative_scale"]
    num, den = gd["mse_alternative"]
    assert oracle_mod.nv_block_loss(xb, alt, g) / 16 == pytest.approx(num / den, rel=1e-6)


def test_nv_zero_tensor_and_zero_block(oracle_mod):
    packed, scales, g = oracle_mod.nvfp4_quantize(np.zeros(16, np.float32))
    assert g == 1.0 and scales.tolist() == [[0]] and not packed.any()
    assert not oracle_mod.nvfp4_dequantize(packed, scales, g, 1, 16).any()
    x = np.array([2688.0] * 16 + [0.0] * 8 + [-0.0] * 8, np.float32)
    packed, scales, g = oracle_mod.nvfp4_quantize(x)
    y = oracle_mod.nvfp4_dequantize(packed, scales, g, 1, 32)[0]
    assert y[16:].tolist() == [0.0] * 16
    assert scales[0, 1] == 0 and not packed[0, 8:].any()   # zero scale -> all-zero codes


def test_nv_rejections_and_zero_scale_convention(oracle_mod):
    with pytest.raises(ValueError) as e:
        oracle_mod.nvfp4_quantize(np.ones(17, np.float32))
    assert e.value.status == oracle_mod.ERR_SHAPE
    with pytest.raises(ValueError) as e:
        oracle_mod.nvfp4_quantize(np.full(16, np.nan, np.float32))
    assert e.value.status == oracle_mod.ERR_NONFINITE
    with pytest.raises(ValueError) as e:
        oracle_mod.nvfp4_quantize(np.array([np.inf] + [0.0] * 15, np.float32))
    assert e.value.status == oracle_mod.ERR_NONFINITE
    # fp32 analogue of the page's [1e-50]*16 (global scale underflow)
    tiny = np.full(16, 2.0 ** -149, np.float32)
    with pytest.raises(ValueError) as e:
        oracle_mod.nvfp4_quantize(tiny)
    assert e.value.status == oracle_mod.ERR_RANGE
    # the page rejects [2688]*16 + [1e-10]*16 (block scale rounds to zero);
    # the fixed convention maps it to a zero scale with all-zero codes
    x = np.array([2688.0] * 16 + [1e-10] * 16, np.float32)
    packed, scales, g = oracle_mod.nvfp4_quantize(x)
    assert scales[0, 1] == 0 and not packed[0, 8:].any()
    assert not oracle_mod.nvfp4_dequantize(packed, scales, g, 1, 32)[0, 16:].any()


def test_global_scale_is_fp32_quotient(oracle_mod):
    rng = np.random.default_rng(5)
    A = np.float32(2.0) ** rng.uniform(-100, 127, 20000).astype(np.float32)
    A = A[np.isfinite(A)]
    want = A / np.float32(2688.0)
    for a, w in zip(A.tolist(), want.tolist()):
        if w >= np.finfo(np.float32).tiny:
            assert oracle_mod.nv_global_scale(a) == w
    assert oracle_mod.nv_global_scale(0.0) == 1.0
    with pytest.raises(ValueError):
        oracle_mod.nv_global_scale(2688.0 * 2.0 ** -127)


def _random_tensor(rows, cols, seed, dtype=torch.bfloat16):
    w = workloads.with_shape(workloads.WEIGHT_4K, rows, cols, seed_offset=seed)
    return workloads.as_oracle_array(workloads.generate(w).to(dtype))


def test_nv_scale_bytes_are_exact_rationals_and_codes_requantize(oracle_mod):
    """On random bf16 data: every scale byte is the exact-rational E4M3
    rounding of A_b/(6g); every element's reconstruction error is at most
    half the local grid gap (unless saturated); re-quantising the
    dequantised tensor with the same scales and g returns the same codes."""
    x = _random_tensor(64, 256, 3)
    xf = oracle_mod.bf16_to_f32(x).reshape(64, 256)
    packed, scales, g = oracle_mod.nvfp4_quantize(x)
    assert g == np.float32(np.abs(xf).max()) / np.float32(2688.0)
    tab = [Fraction(v) for v in torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().tolist()]
    blocks = xf.reshape(-1, 16)
    ab = np.abs(blocks).max(axis=1)
    for b in range(0, blocks.shape[0], 7):
        t = min(Fraction(float(ab[b])) / (6 * Fraction(g)), tab[126])
        want = min(range(127), key=lambda c: (abs(tab[c] - t), c & 1))
        assert scales.reshape(-1)[b] == want
    y = oracle_mod.nvfp4_dequantize(packed, scales, g, 64, 256)
    codes = nv_codes(packed).reshape(-1, 16)
    sb = np.array([oracle_mod.e4m3_value(int(c)) for c in scales.reshape(-1)])
    d = (sb.astype(np.float32) * np.float32(g))[:, None]
    gap = np.array([0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0, 2.0])  # gap below/around each magnitude
    err = np.abs(y.reshape(-1, 16).astype(np.float64) - blocks)
    unsat = np.abs(blocks / d) <= 6.0
    bound = gap[codes & 7] / 2 * d * (1 + 1e-6) + 1e-30
    assert np.all(err[unsat & (sb[:, None] > 0)] <= bound[unsat & (sb[:, None] > 0)])
    # signs survive: negative inputs give codes with bit 3 (or +0 under a zero scale)
    neg = blocks < 0
    assert np.all((codes[neg] & 8) | (codes[neg] == 0))
    # requantise the reconstruction with the same scales and g
    ybf = y.reshape(-1)
    p2, s2 = oracle_mod.nvfp4_quantize_with_g(ybf.reshape(64, 256), g)
    nz = sb > 0
    c2 = nv_codes(p2).reshape(-1, 16)
    # same scale bytes where the block maximum reconstructs onto the same scale
    same = s2.reshape(-1) == scales.reshape(-1)
    assert same.mean() > 0.9
    assert np.array_equal(c2[same & nz], codes[same & nz])


def test_nv_dequant_grouped_dot(oracle_mod):
    """The grouped block-scaled dot product of the page's example equals the
    dot of the two dequantised vectors: -120 (the wrong one-scale form: -8)."""
    gd = golden("grouped_dot.json")
    px, pw = expand(gd["px"]), expand(gd["pw"])
    enc = lambda v: [oracle_mod.e2m1_encode(t) for t in v]
    pk = lambda c: np.frombuffer(oracle_mod.pack4(c), np.uint8)
    sx = np.array([oracle_mod.e4m3_encode(b) for b in gd["bx"]], np.uint8)
    sw = np.array([oracle_mod.e4m3_encode(b) for b in gd["bw"]], np.uint8)
    yx = oracle_mod.nvfp4_dequantize(pk(enc(px)), sx, gd["ax"], 1, 32)[0].astype(np.float64)
    yw = oracle_mod.nvfp4_dequantize(pk(enc(pw)), sw, gd["aw"], 1, 32)[0].astype(np.float64)
    assert float(yx @ yw) == gd["group_result"]
    wrong = gd["ax"] * gd["aw"] * gd["bx"][0] * gd["bw"][0] * float(np.dot(px, pw))
    assert wrong == gd["wrong_result"]


# -------------------------------------------------------------- MXFP4 -----

def test_mx_amax_7(oracle_mod):
    gd = golden("mx_examples.json")
    x = np.array([7.0] + [0.0] * 31, np.float32)
    packed, scales = oracle_mod.mxfp4_quantize(x)
    assert oracle_mod.e8m0_value(int(scales[0, 0])) == gd["amax_7_scale"]
    y = oracle_mod.mxfp4_dequantize(packed, scales, 1, 32)[0]
    assert y[0] == gd["amax_7_reconstruction_of_7"]


def test_mx_transpose_counterexample(oracle_mod):
    gd = golden("mx_examples.json")
    n = gd["transpose_matrix"]["size"]
    w = np.full((n, n), gd["transpose_matrix"]["rest"], np.float32)
    w[0, 0] = gd["transpose_matrix"]["corner"]

    def qdq(m):
        p, s = oracle_mod.mxfp4_quantize(np.ascontiguousarray(m))
        return oracle_mod.mxfp4_dequantize(p, s, *m.shape)

    assert qdq(w).T[0, 1] == gd["quantize_then_transpose_0_1"]
    assert qdq(w.T)[0, 1] == gd["transpose_then_quantize_0_1"]
    p, s = oracle_mod.mxfp4_quantize(np.ascontiguousarray(w[1]))
    assert oracle_mod.e8m0_value(int(s[0, 0])) == gd["row_of_0p3_scale"]
    assert f32(w[1, 0] / gd["row_of_0p3_scale"]) == pytest.approx(gd["row_of_0p3_normalised"], rel=1e-6)


def test_mx_invariants_random(oracle_mod):
    x = _random_tensor(32, 512, 9)
    xf = oracle_mod.bf16_to_f32(x).reshape(-1, 32).astype(np.float64)
    packed, scales = oracle_mod.mxfp4_quantize(x)
    e = scales.reshape(-1).astype(np.int64) - 127
    ab = np.abs(xf).max(axis=1)
    nz = ab > 0
    # floor rule: A_b / 2^e in [4, 8)
    r = ab[nz] / np.exp2(e[nz].astype(np.float64))
    assert np.all((r >= 4) & (r < 8))
    y = oracle_mod.mxfp4_dequantize(packed, scales, 32, 512).reshape(-1, 32).astype(np.float64)
    codes = nv_codes(packed).reshape(-1, 32)
    mag = np.array([0, .5, 1, 1.5, 2, 3, 4, 6])
    sign = np.where(codes & 8, -1.0, 1.0)
    assert np.array_equal(y, sign * mag[codes & 7] * np.exp2(e.astype(np.float64))[:, None])
    v = xf / np.exp2(e.astype(np.float64))[:, None]
    gap = np.array([0.5, 0.5, 0.5, 0.5, 1.0, 1.0, 2.0, 2.0])
    unsat = np.abs(v) <= 6
    assert np.all(np.abs(v - y / np.exp2(e)[:, None])[unsat] <= gap[codes & 7][unsat] / 2)


def test_mx_zero_block_and_sign(oracle_mod):
    x = np.array([0.0] * 16 + [-0.0] * 16, np.float32)
    packed, scales = oracle_mod.mxfp4_quantize(x)
    assert scales.tolist() == [[0]]
    assert nv_codes(packed).tolist() == [0] * 16 + [8] * 16
    with pytest.raises(ValueError):
        oracle_mod.mxfp4_quantize(np.ones(48, np.float32))
    with pytest.raises(ValueError):
        oracle_mod.mxfp4_quantize(np.array([np.nan] + [1.0] * 31, np.float32))


# ------------------------------------------------------- scale search -----

def test_search_on_counterexample_block(oracle_mod):
    """Candidates 0.7..1.0 x 0.6 collapse to E4M3 0.40625..0.625; by hand the
    block MSEs are 0.5: 0.031875, 0.5625: 0.016384..., 0.625: 879/102400,
    0.4375: 0.060731...; the search keeps the max-based 0.625."""
    gd = golden("nv_counterexample.json")
    blk = expand(gd["block"])
    x = np.array([2688.0] * 16 + blk, np.float32)
    packed, scales, g, loss = oracle_mod.nvfp4_scale_search(x)
    assert g == 1.0 and scales[0, 1] == 0x32
    num, den = gd["mse_max_based"]
    assert loss[0, 1] / 16 == pytest.approx(num / den, rel=1e-6)
    cand = sorted({oracle_mod.search_candidate_code(3.6, 1.0, k) for k in range(64)})
    assert [oracle_mod.e4m3_value(c) for c in cand] == [0.40625, 0.4375, 0.46875, 0.5, 0.5625, 0.625]
    xb = np.array(blk, np.float32)
    hand = {0.5: (15 * 0.1 ** 2 + 0.6 ** 2) / 16,
            0.5625: (15 * 0.11875 ** 2 + 0.225 ** 2) / 16,
            0.4375: (15 * 0.0375 ** 2 + 0.975 ** 2) / 16}
    for s, want in hand.items():
        assert oracle_mod.nv_block_loss(xb, oracle_mod.e4m3_encode(s), 1.0) / 16 == pytest.approx(want, rel=1e-5)


def test_search_candidates_are_exact_and_never_worse_than_max_based(oracle_mod):
    x = _random_tensor(16, 256, 21)
    xf = oracle_mod.bf16_to_f32(x).reshape(-1, 16)
    packed, scales, g, loss = oracle_mod.nvfp4_scale_search(x)
    p0, s0, g0 = oracle_mod.nvfp4_quantize(x)
    assert g == g0
    base = oracle_mod.nvfp4_artefact_loss(x, p0, s0, g0).reshape(-1)
    assert np.all(loss.reshape(-1) <= base)
    # the chosen artefact's loss, recomputed from the emitted bytes
    assert np.array_equal(oracle_mod.nvfp4_artefact_loss(x, packed, scales, g), loss)
    tab = [Fraction(v) for v in torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().tolist()]
    ab = np.abs(xf).max(axis=1)
    for b in range(0, xf.shape[0], 5):
        cset = set()
        for k in range(64):
            t = min(Fraction(147 + k, 210) * Fraction(float(ab[b])) / (6 * Fraction(g)), tab[126])
            cset.add(min(range(127), key=lambda c: (abs(tab[c] - t), c & 1)))
        assert {oracle_mod.search_candidate_code(float(ab[b]), g, k) for k in range(64)} == cset
        assert scales.reshape(-1)[b] in cset
        # the emitted loss is the loss of quantising at the chosen scale
        assert oracle_mod.nv_block_loss(xf[b].copy(), int(scales.reshape(-1)[b]), g) == loss.reshape(-1)[b]
    # the k = 63 candidate is the max-based scale
    for b in range(xf.shape[0]):
        assert oracle_mod.search_candidate_code(float(ab[b]), g, 63) == s0.reshape(-1)[b]


def test_search_zero_tensor(oracle_mod):
    packed, scales, g, loss = oracle_mod.nvfp4_scale_search(np.zeros((2, 32), np.float32))
    assert g == 1.0 and not packed.any() and not scales.any() and not loss.any()


# -------------------------------------------------------------- storage ---

def test_storage_bytes(oracle_mod):
    gd = golden("storage_bytes.json")
    assert oracle_mod.storage_bytes(1024, 32, 0) == gd["mx_1024"]
    assert oracle_mod.storage_bytes(1024, 16, 4) == gd["nv_1024"]
    assert oracle_mod.storage_bytes(16, 16, 4) == gd["nv_16"]
    assert oracle_mod.storage_bytes(16, 16, 4) * 8 / 16 == gd["nv_16_bits_per_value"]
    assert oracle_mod.storage_bytes(1 << 20, 32, 0) * 8 / (1 << 20) == gd["mx_bits_per_element"]
    assert oracle_mod.storage_bytes(1 << 20, 16, 0) * 8 / (1 << 20) == gd["nv_bits_per_element"]
    with pytest.raises(ValueError):
        oracle_mod.storage_bytes(17, 16, 4)


# --------------------------------------------------- block-size MAE -------

def test_block_size_mae_experiment(oracle_mod):
    """The ultralytics page's experiment, redone with the oracle's E2M1
    encoder (nearest value; exact ties have probability zero here): one real
    scale amax/6 per block, MAE printed to four decimals."""
    gd = golden("block_size_mae.json")
    x = workloads.page_mae_input()
    mag = np.array([oracle_mod.e2m1_decode(c) for c in range(8)], np.float32)
    for block, want in gd["mae"].items():
        b = x.reshape(-1, int(block))
        scale = b.abs().amax(dim=1, keepdim=True) / 6.0
        codes = oracle_mod.e2m1_encode_f32((b.abs() / scale).numpy())
        dq = torch.from_numpy(mag[codes & 7]) * b.sign() * scale
        mae = (dq.flatten() - x).abs().mean().item()
        assert round(mae, gd["printed_decimals"]) == want
