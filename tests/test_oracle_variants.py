"""Pins of the oracle's scale-rule variants: the MXFP4 ceil rule of the page's
`mx_scale` helper ("NVFP4 与 MXFP4 格式", §5-§6) and NVFP4 "four over six"
("FP4、FP8 与 INT8/INT4", §4)."""
import numpy as np
import pytest

import workloads
from conftest import golden


def codes_of(packed):
    p = packed.reshape(-1)
    return np.stack([p & 15, p >> 4], axis=1).reshape(-1)


def test_mx_ceil_amax_7_and_zero_block(oracle_mod):
    gd = golden("mx_ceil_rule.json")
    e = oracle_mod.mx_block_exponent_ceil(7.0)
    assert 2.0 ** e == gd["amax_7_scale"] and 6 * 2.0 ** e == gd["amax_7_range"]
    x = np.array([7.0] + [0.0] * 31 + [0.0] * 32, np.float32)
    p, s = oracle_mod.mxfp4_quantize_rule(x, oracle_mod.MX_CEIL)
    assert oracle_mod.e8m0_value(int(s[0, 0])) == gd["amax_7_scale"]
    assert oracle_mod.e8m0_value(int(s[0, 1])) == gd["zero_block_scale"]
    y = oracle_mod.mxfp4_dequantize(p, s, 1, 64)[0]
    assert y[0] == 8.0          # 7 / 2 = 3.5 rounds to the even code, 4
    # the floor rule keeps its own reading for the same input
    p0, s0 = oracle_mod.mxfp4_quantize_rule(x, oracle_mod.MX_FLOOR)
    assert np.array_equal(s0, oracle_mod.mxfp4_quantize(x)[1])


def test_mx_ceil_transpose_counterexample(oracle_mod):
    gd = golden("mx_ceil_rule.json")
    n = gd["transpose_matrix"]["size"]
    w = np.full((n, n), gd["transpose_matrix"]["rest"], np.float32)
    w[0, 0] = gd["transpose_matrix"]["corner"]

    def qdq(m):
        p, s = oracle_mod.mxfp4_quantize_rule(np.ascontiguousarray(m), oracle_mod.MX_CEIL)
        return oracle_mod.mxfp4_dequantize(p, s, *m.shape)

    assert qdq(w).T[0, 1] == gd["quantize_then_transpose_0_1"]
    assert qdq(w.T)[0, 1] == gd["transpose_then_quantize_0_1"]


def test_mx_ceil_never_clips_and_is_minimal(oracle_mod):
    rng = np.random.default_rng(4)
    a = (2.0 ** rng.uniform(-120, 120, 20000)).astype(np.float32)
    a = np.concatenate([a, np.float32([6.0, 6.0000005, 5.9999995, 12.0, 3.0, 1e-40])])
    for v in a.tolist():
        e = oracle_mod.mx_block_exponent_ceil(v)
        assert v <= 6 * 2.0 ** e
        if e > -127:
            assert v > 6 * 2.0 ** (e - 1)


def test_four_over_six_page_examples(oracle_mod):
    gd = golden("four_over_six.json")
    for key, want_map in (("max_to_4_exact", 4.0), ("max_to_6_exact", 6.0)):
        vals = gd[key]
        blk = vals + [0.0] * (16 - len(vals))
        x = np.array([2688.0] * 16 + blk, np.float32)       # forces g = 1
        p, s, g, loss = oracle_mod.nvfp4_quantize_four_over_six(x)
        assert g == 1.0
        scale = oracle_mod.e4m3_value(int(s[0, 1]))
        assert scale == max(vals) / want_map
        assert loss[0, 1] == 0.0
        y = oracle_mod.nvfp4_dequantize(p, s, g, 1, 32)[0, 16:]
        assert y.tolist() == blk


def test_four_over_six_never_worse_than_max_based(oracle_mod):
    x = workloads.as_oracle_array(workloads.generate(workloads.with_shape(workloads.SEARCH_4K, 16, 512)))
    p, s, g, loss = oracle_mod.nvfp4_quantize_four_over_six(x)
    p0, s0, g0 = oracle_mod.nvfp4_quantize(x)
    assert g == g0
    base = oracle_mod.nvfp4_artefact_loss(x, p0, s0, g0).reshape(-1)
    assert np.all(loss.reshape(-1) <= base)
    assert np.array_equal(oracle_mod.nvfp4_artefact_loss(x, p, s, g), loss)
    xf = oracle_mod.bf16_to_f32(x).reshape(-1, 16)
    ab = np.abs(xf).max(axis=1)
    c4 = np.array([oracle_mod.e4m3_encode(float(a) / (4 * g)) for a in ab])
    chosen = s.reshape(-1)
    assert np.all((chosen == s0.reshape(-1)) | (chosen == c4))
    assert (chosen == c4).any() and (chosen != c4).any()
