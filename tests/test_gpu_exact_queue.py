"""The NVFP4 quantisers' warp-shared exact path ("NVFP4 与 MXFP4 格式"
section 3: v = x / (s_b g) in IEEE single, then E2M1 with ties to even).
A half-block whose bracketed quotient may straddle an E2M1 midpoint is
queued with the rest of its warp's and divided by the whole warp, one
element per lane.  That path runs on whole warp steps only (every lane of
the warp with all its blocks in range), i.e. on tensors of millions of
elements, so the inputs here are large (2^23 - 2^24 elements, which the C
oracle quantises in a second or two) and built to put many quotients on or
next to midpoints:

* tie-rich: with g = fl32(A / 2688), a block whose maximum is A 2^-j gets
  the scale 1.75 2^(8-j) (448 2^-j exactly), and one whose maximum is
  fl_bf16(6/7 A) 2^-j the scale 1.5 2^(8-j); an element A 2^-k then has
  x / d within an fp32 step or two of 3 2^(1+j-k) or 7 2^(j-k), i.e. of the
  midpoints 0.75, 1.75 and 3.5.  About a third of the elements are placed
  so, the rest drawn around them;
* all-flagged: A = 2^-108 and every other block near 2^-125, so that
  d = fl32(s_b g) is subnormal and every half-block takes the exact path
  (the queue holds every half-block of every warp step).

Codes and scale bytes must equal the oracle's bit for bit, for the
single-tensor, grouped, padded (ragged rows) and column-wise calls."""
import numpy as np
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
from test_gpu_parity import assert_same, odata

pytestmark = pytest.mark.gpu
DEV = "cuda"


def tie_rich(rows: int, cols: int, seed: int) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    A = 0.75
    n_blocks = rows * cols // 16
    j = rng.integers(0, 6, n_blocks)
    f = np.where(rng.random(n_blocks) < 0.5, 1.0, float(torch.tensor(6 / 7 * A).bfloat16().float()) / A)
    bmax = A * f * np.exp2(-j)
    x = rng.uniform(-1.0, 1.0, (n_blocks, 16)) * bmax[:, None]
    k = rng.integers(1, 5, (n_blocks, 16))
    on_tie = rng.random((n_blocks, 16)) < 0.35
    sign = np.where(rng.random((n_blocks, 16)) < 0.5, -1.0, 1.0)
    x = np.where(on_tie, sign * A * np.exp2(-(j[:, None] + k)), x)
    x[np.arange(n_blocks), rng.integers(0, 16, n_blocks)] = bmax * np.where(rng.random(n_blocks) < 0.5, -1, 1)
    x[0, 0] = A
    return torch.from_numpy(x.reshape(rows, cols).astype(np.float32)).bfloat16()


def all_flagged(rows: int, cols: int, seed: int) -> torch.Tensor:
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((rows, cols)) * 2.0 ** -126.5
    x[0, 0] = 2.0 ** -108
    return torch.from_numpy(x.astype(np.float32)).bfloat16()


def quotients(x: torch.Tensor):
    """|x| / d in double per element ([blocks, 16]) and d per block, with the
    oracle's g and scale codes."""
    _, s, g = oracle.nvfp4_quantize(odata(x))
    d = np.array([oracle.e4m3_value(c) for c in range(256)])[s.reshape(-1)] * np.float64(np.float32(g))
    v = np.abs(x.float().numpy().reshape(-1, 16).astype(np.float64)) / np.where(d > 0, d, 1.0)[:, None]
    return v, d


def midpoint_fraction(x: torch.Tensor) -> float:
    """Fraction of elements whose x / d lies within 2^-20 (relative) of an
    E2M1 midpoint."""
    v, _ = quotients(x)
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])
    near = np.min(np.abs(v[..., None] - mids) / mids, axis=-1) < 2.0 ** -20
    return float(near.mean())


def check_q(q, p, s, g):
    torch.cuda.synchronize()
    assert q.status.item() == 0
    assert q.global_scale.item() == g
    assert_same(q.scales, s, "scales")
    assert_same(q.packed, p, "packed")


def check_single(x: torch.Tensor):
    xo = odata(x)
    p, s, g = oracle.nvfp4_quantize(xo)
    q = fp4.nvfp4_quantize(x.to(DEV))
    torch.cuda.synchronize()
    assert q.status.item() == 0
    assert q.global_scale.item() == g
    assert_same(q.scales, s, "scales")
    assert_same(q.packed, p, "packed")


def test_tie_rich_single():
    x = tie_rich(4096, 4096, seed=21)
    assert midpoint_fraction(x[:256]) > 0.05  # the input does what it is for
    check_single(x)


def test_all_flagged_single():
    x = all_flagged(2048, 4096, seed=22)
    _, d = quotients(x[:64])
    nonzero = d[d > 0]
    assert (nonzero < 2.0 ** -126).mean() > 0.99  # d subnormal: the exact path for all of them
    check_single(x)


def test_tie_rich_grouped():
    xs = [tie_rich(2048, 4096, seed=30 + i) for i in range(2)] + [all_flagged(1024, 4096, seed=33)]
    nv = fp4.nvfp4_quantize_grouped([x.to(DEV) for x in xs])
    torch.cuda.synchronize()
    assert nv[0].status.item() == 0
    for i, x in enumerate(xs):
        p, s, g = oracle.nvfp4_quantize(odata(x))
        assert nv[i].global_scale.item() == g, f"item {i} g"
        assert_same(nv[i].scales, s, f"item {i} scales")
        assert_same(nv[i].packed, p, f"item {i} packed")


def test_tie_rich_padded():
    x = tie_rich(2048, 4096, seed=40)[:, :4095].contiguous()
    check_q(fp4.nvfp4_quantize_padded(x.to(DEV)), *oracle.nvfp4_quantize_padded(odata(x)))


def test_tie_rich_columns():
    x = tie_rich(4096, 2048, seed=41)
    xt = x.t().contiguous()
    assert midpoint_fraction(xt[:256]) > 0.02  # ties along the columns too
    check_q(fp4.nvfp4_quantize_columns(x.to(DEV)), *oracle.nvfp4_quantize_columns(odata(x)))
