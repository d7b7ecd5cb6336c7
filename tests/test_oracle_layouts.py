"""Oracle pins for ragged rows and column-wise grouping ("NVFP4 与 MXFP4 格式"
sections 6-8): the page's padded byte count, its transposition
counterexample, closed forms for single-element rows, and the invariants
that tie the padded and column-wise forms to the plain quantisers."""
import numpy as np
import pytest

from conftest import golden


def bf16_bits(v):
    import oracle
    return oracle.f32_to_bf16(np.asarray(v, np.float32))


def test_padded_block_count_and_bytes_of_the_page(oracle_mod):
    o = oracle_mod
    gd = golden("padded_layout.json")
    R, K, G = gd["rows"], gd["cols"], gd["group"]
    assert o.padded_blocks(R, K, G) == gd["blocks_padded"]
    assert -(-R * K // G) == gd["blocks_if_flattened"] != gd["blocks_padded"]
    assert o.padded_storage_bytes(R, K, G, 4) == gd["nv_bytes"]
    # the quantiser's outputs have exactly that size
    x = np.linspace(-1, 1, R * K, dtype=np.float32).reshape(R, K)
    p, s, g = o.nvfp4_quantize_padded(x)
    assert p.nbytes + s.nbytes + np.float32(g).nbytes == gd["nv_bytes"]
    assert s.shape == (R, gd["blocks_padded"] // R)
    # complete blocks: the padded count equals the plain one
    assert o.padded_storage_bytes(1, 1024, 32, 0) == o.storage_bytes(1024, 32, 0) == 544
    assert o.padded_storage_bytes(1, 1024, 16, 4) == o.storage_bytes(1024, 16, 4) == 580


def test_transpose_counterexample_floor_rule(oracle_mod):
    o = oracle_mod
    gd = golden("transpose_floor_rule.json")
    n = gd["size"]
    w = np.full((n, n), gd["rest"], np.float32)
    w[0, 0] = gd["corner"]
    p, s = o.mxfp4_quantize(w)
    y_rows = o.mxfp4_dequantize(p, s, n, n)
    pc, sc = o.mxfp4_quantize_columns(w)
    y_cols = o.mxfp4_dequantize(pc, sc, n, n)  # [C, R]: row c = column c of w
    assert y_rows.T[0, 1] == gd["row_wise_then_transpose_0_1"]
    assert y_cols[0, 1] == gd["column_wise_0_1"]
    assert int(s[1, 0]) - 127 == gd["row_scale_exponent"]
    assert int(sc[0, 0]) - 127 == gd["column_scale_exponent"]


def test_single_element_rows_closed_forms(oracle_mod):
    """A row of one value v is the block [v, +0 x (G-1)].  NVFP4 with A = |v|:
    t = A / (6 g) rounds to 448 (code 0x7E), v / fl32(448 g) = +-6 (code 7
    with v's sign), pads code 0.  MXFP4 with v = 3: e = floor(log2 3) - 2 =
    -1, 3 * 2 = 6 (code 7), scale byte 126."""
    o = oracle_mod
    for v in (3.0, -3.0, 0.75):
        p, s, g = o.nvfp4_quantize_padded(np.array([[v]], np.float32))
        assert p.shape == (1, 8) and s.shape == (1, 1)
        assert s[0, 0] == 0x7E
        assert p[0, 0] == (0x7 | (0x8 if v < 0 else 0)) and not p[0, 1:].any()
        y = o.nvfp4_dequantize_padded(p, s, g, 1, 1)
        assert y.shape == (1, 1) and abs(y[0, 0] - v) <= 1e-6 * abs(v)
    p, s = o.mxfp4_quantize_padded(np.array([[3.0]], np.float32))
    assert p.shape == (1, 16) and s[0, 0] == 126 and p[0, 0] == 0x07 and not p[0, 1:].any()
    assert o.mxfp4_dequantize_padded(p, s, 1, 1)[0, 0] == 3.0


@pytest.mark.parametrize("dtype", [np.float32, np.uint16])
def test_padding_changes_nothing_for_complete_rows(oracle_mod, dtype):
    o = oracle_mod
    rng = np.random.default_rng(4)
    x = rng.standard_normal((5, 64)).astype(np.float32)
    if dtype == np.uint16:
        x = bf16_bits(x)
    p, s, g = o.nvfp4_quantize(x)
    pp, sp, gp = o.nvfp4_quantize_padded(x)
    assert g == gp and np.array_equal(p, pp) and np.array_equal(s, sp)
    for rule in (0, 1):
        a = o.mxfp4_quantize_rule(x, rule)
        b = o.mxfp4_quantize_padded(x, rule)
        assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_ragged_rows_keep_their_own_blocks(oracle_mod):
    """With K = 17 the second block of every row holds one real element:
    it is quantised on its own (its scale comes from that element alone),
    unlike a flattened grouping where it would share a block with the next
    row's first 15 elements."""
    o = oracle_mod
    R, K = 3, 17
    x = np.arange(1, R * K + 1, dtype=np.float32).reshape(R, K) / 8.0
    p, s, g = o.nvfp4_quantize_padded(x)
    assert s.shape == (R, 2) and p.shape == (R, 16)
    for r in range(R):
        # the lone element is the block maximum: t = A_b / (6g) gives a scale
        # with the element at +6 or just below, i.e. code 6 or 7
        assert s[r, 1] == o.nv_block_scale_code(float(x[r, 16]), g)
        assert (p[r, 8] & 0xF) in (6, 7) and not p[r, 8] >> 4 and not p[r, 9:].any()
    y = o.nvfp4_dequantize_padded(p, s, g, R, K)
    assert y.shape == (R, K)
    yfull = o.nvfp4_dequantize(p, s, g, R, 32)
    assert np.array_equal(y, yfull[:, :K]) and not yfull[:, K:].any()


def test_column_wise_is_row_wise_of_the_transpose_by_hand(oracle_mod):
    """x [16, 2]: column-wise NVFP4 puts each column in one block; the
    block of column c is the row-wise block of the 16 values x[:, c]."""
    o = oracle_mod
    rng = np.random.default_rng(1)
    x = rng.standard_normal((16, 2)).astype(np.float32)
    pc, sc, g = o.nvfp4_quantize_columns(x)
    assert pc.shape == (2, 8) and sc.shape == (2, 1)
    for c in range(2):
        col = np.ascontiguousarray(x[:, c]).reshape(1, 16)
        p1, s1 = o.nvfp4_quantize_with_g(col, g)
        assert np.array_equal(pc[c], p1[0]) and sc[c, 0] == s1[0, 0]
    # a ragged row count pads the columns: R = 20 -> two blocks per column
    x = rng.standard_normal((20, 3)).astype(np.float32)
    pc, sc, g = o.nvfp4_quantize_columns(x)
    assert pc.shape == (3, 16) and sc.shape == (3, 2)
