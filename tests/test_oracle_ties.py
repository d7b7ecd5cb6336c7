"""Pins of the oracle's tie rules and of its argmin, against an independent
exact-arithmetic model written in this file.

- Scale search ("FP4 / NVFP4 数学总结" §9, Loss(s) = sum (x - s Round(x/s))^2;
  the fixed search convention: 64 candidates (147+k)/210 x A_b/(6g), the
  smallest loss wins, ties go to the larger scale).
- Four over six ("FP4、FP8 与 INT8/INT4" §4: the block maximum mapped to 4
  instead of 6 only where that is better; the reading taken here is
  "strictly better", so an exact tie keeps the max-based scale).

The model shares nothing with the oracle: E4M3 values come from torch's
float8_e4m3fn table, E2M1 rounding is a nearest-value search with ties to
the even code in exact rationals, the fp32 steps of the contract (the
element quotient x / fl32(s_b g) and the dequantised value
fl32(fl32(p s_b) g)) are numpy float32 operations, and every loss is summed
as an exact Fraction.  A loss tie found by the model is therefore an exact
tie of real numbers, which the oracle's double sum reproduces exactly for
the short dyadic blocks used below.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import workloads

MAG = [Fraction(v) for v in (0, 0.5, 1, 1.5, 2, 3, 4, 6)]
E4 = [Fraction(v) for v in torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().tolist()]
F32 = np.float32


def e2m1_code(v: float) -> tuple[int, bool]:
    """Nearest E2M1 magnitude to |v| (saturating at 6), ties to the even code."""
    m = abs(Fraction(v))
    return min(range(8), key=lambda c: (abs(MAG[c] - m), c & 1)), bool(np.signbit(v))


def e4m3_code(t: Fraction) -> int:
    """Nearest E4M3 code to t >= 0 after saturation at 448, ties to the even code."""
    t = min(t, E4[126])
    return min(range(127), key=lambda c: (abs(E4[c] - t), c & 1))


def model_loss(xs, code: int, g) -> Fraction:
    """Exact loss of the artefact emitted at scale code `code`: sum of
    (x - x_hat)^2 with x_hat = fl32(fl32(p s_b) g); a zero scale emits zero
    codes, so x_hat = 0."""
    s = F32(float(E4[code]))
    g = F32(g)
    d = F32(s * g)
    total = Fraction(0)
    for x in xs:
        x = F32(x)
        if code == 0:
            xh = F32(0.0)
        else:
            c, neg = e2m1_code(float(F32(x / d)))
            p = F32(-float(MAG[c]) if neg else float(MAG[c]))
            xh = F32(F32(p * s) * g)
        total += (Fraction(float(x)) - Fraction(float(xh))) ** 2
    return total


def model_candidates(amax_b: float, g) -> list[int]:
    return sorted({e4m3_code(Fraction(147 + k, 210) * Fraction(float(amax_b)) / (6 * Fraction(float(F32(g)))))
                   for k in range(64)})


def model_search(xs, g) -> tuple[int, Fraction, Fraction]:
    """(chosen code, its loss, the runner-up's loss) of the definition:
    smallest exact loss over the candidate set, an exact tie to the larger
    scale (E4M3 codes order like their values)."""
    amax_b = max(abs(float(F32(x))) for x in xs)
    losses = {c: model_loss(xs, c, g) for c in model_candidates(amax_b, g)}
    best = min(losses, key=lambda c: (losses[c], -c))
    rest = [v for c, v in losses.items() if c != best]
    return best, losses[best], (min(rest) if rest else None)


def forced_g1(block):
    """A 16-element block behind a block of 2688s, so that the tensor amax is
    2688 and g = fl32(2688 / 2688) = 1."""
    blk = list(block) + [0.0] * (16 - len(block))
    return np.array([2688.0] * 16 + blk, np.float32)


# Blocks (first element the block maximum, the rest zero-padded to 16) whose
# two best candidate scales tie exactly; each tie is re-derived below.
SEARCH_TIES = [
    ([6.0, 0.03125, 2.53125], (0.9375, 1.0)),   # the max-based scale in the tie
    ([6.0, 0.03125, 3.59375], (0.9375, 1.0)),
    ([6.0, 0.03125, 4.875], (0.875, 0.9375)),   # two scales below the max-based one
]


@pytest.mark.parametrize("block,tied", SEARCH_TIES)
def test_search_exact_tie_keeps_the_larger_scale(oracle_mod, block, tied):
    # the tie itself, in exact arithmetic
    cands = model_candidates(6.0, 1.0)
    losses = {float(E4[c]): model_loss(block, c, 1.0) for c in cands}
    lo, hi = tied
    assert losses[lo] == losses[hi] == min(losses.values())
    assert sum(v == losses[hi] for v in losses.values()) == 2
    best, best_loss, _ = model_search(block, 1.0)
    assert float(E4[best]) == hi
    # the oracle keeps the larger of the two tied scales
    packed, scales, g, loss = oracle_mod.nvfp4_scale_search(forced_g1(block))
    assert g == 1.0
    assert oracle_mod.e4m3_value(int(scales[0, 1])) == hi
    assert Fraction(float(loss[0, 1])) == best_loss
    # and the oracle's own loss function sees the same exact tie
    xb = np.array(list(block) + [0.0] * (16 - len(block)), np.float32)
    assert oracle_mod.nv_block_loss(xb, e4m3_code(Fraction(lo)), 1.0) == \
        oracle_mod.nv_block_loss(xb, e4m3_code(Fraction(hi)), 1.0)


def test_search_strictly_better_smaller_scale_wins(oracle_mod):
    """Without a tie the smaller scale must win when it is better: the
    counter-check that the tie rule is not simply "prefer the larger"."""
    block = [6.0, 0.03125, 2.5]
    best, best_loss, runner = model_search(block, 1.0)
    assert runner > best_loss and float(E4[best]) < 1.0
    _, scales, _, loss = oracle_mod.nvfp4_scale_search(forced_g1(block))
    assert int(scales[0, 1]) == best
    assert Fraction(float(loss[0, 1])) == best_loss


def test_search_argmin_matches_independent_model(oracle_mod):
    """On random blocks of the search workload's distribution (Laplace, bf16)
    and of the activation's (Student-t), the oracle's choice is the exact
    argmin over the candidate set, and its reported loss is the exact loss
    of that choice up to double rounding."""
    checked = 0
    for wl, seed in ((workloads.SEARCH_4K, 31), (workloads.ACT_8K, 32)):
        x = workloads.as_oracle_array(workloads.generate(workloads.with_shape(wl, 4, 512, seed)))
        xf = oracle_mod.bf16_to_f32(x).reshape(-1, 16)
        packed, scales, g, loss = oracle_mod.nvfp4_scale_search(x)
        s, lo = scales.reshape(-1), loss.reshape(-1)
        for b in range(0, xf.shape[0], 2):
            xs = [float(v) for v in xf[b]]
            best, best_loss, runner = model_search(xs, g)
            assert abs(Fraction(float(lo[b])) - best_loss) <= best_loss * Fraction(1, 10 ** 12)
            if runner is not None and runner != best_loss and \
                    abs(runner - best_loss) <= best_loss * Fraction(1, 10 ** 12):
                continue  # a near-tie double rounding may decide; none expected here
            assert int(s[b]) == best, f"block {b}: oracle chose {s[b]}, the exact argmin is {best}"
            checked += 1
    assert checked >= 120


FOUR_OVER_SIX_TIES = [
    [6.0, 0.03125, 0.625],    # 0.625 -> 0.5 at scale 1, -> 0.75 at scale 1.5: same error
    [6.0, 0.03125, 0.875],
    [4.5, 0.03125, 0.0625],
]


@pytest.mark.parametrize("block", FOUR_OVER_SIX_TIES)
def test_four_over_six_tie_keeps_the_max_based_scale(oracle_mod, block):
    amax_b = block[0]
    c6 = e4m3_code(Fraction(amax_b) / 6)
    c4 = e4m3_code(Fraction(amax_b) / 4)
    assert c4 != c6
    assert model_loss(block, c6, 1.0) == model_loss(block, c4, 1.0)
    _, scales, g, loss = oracle_mod.nvfp4_quantize_four_over_six(forced_g1(block))
    assert g == 1.0 and int(scales[0, 1]) == c6
    assert Fraction(float(loss[0, 1])) == model_loss(block, c6, 1.0)


def test_four_over_six_matches_independent_model(oracle_mod):
    """Random Student-t blocks: the oracle takes the max-to-4 scale exactly
    where the model's exact loss is strictly smaller."""
    x = workloads.as_oracle_array(workloads.generate(workloads.with_shape(workloads.ACT_8K, 4, 512, 33)))
    xf = oracle_mod.bf16_to_f32(x).reshape(-1, 16)
    _, scales, g, _ = oracle_mod.nvfp4_quantize_four_over_six(x)
    s = scales.reshape(-1)
    n4 = 0
    for b in range(xf.shape[0]):
        xs = [float(v) for v in xf[b]]
        amax_b = Fraction(float(np.abs(xf[b]).max()))
        c6 = e4m3_code(amax_b / (6 * Fraction(float(g))))
        c4 = e4m3_code(amax_b / (4 * Fraction(float(g))))
        want = c4 if model_loss(xs, c4, g) < model_loss(xs, c6, g) else c6
        assert int(s[b]) == want
        n4 += want == c4 and c4 != c6
    assert 0 < n4 < xf.shape[0]


# The search over a general grid m_k = (p + k) / q, k < n (the candidate grid
# as a parameter of the call; the fixed search is n = 64, p = 147, q = 210).
def model_grid_candidates(amax_b: float, g, n: int, p: int, q: int) -> list[int]:
    return sorted({e4m3_code(Fraction(p + k, q) * Fraction(float(amax_b)) / (6 * Fraction(float(F32(g)))))
                   for k in range(n)})


def model_grid_search(xs, g, n, p, q):
    amax_b = max(abs(float(F32(x))) for x in xs)
    losses = {c: model_loss(xs, c, g) for c in model_grid_candidates(amax_b, g, n, p, q)}
    best = min(losses, key=lambda c: (losses[c], -c))
    rest = [v for c, v in losses.items() if c != best]
    return best, losses[best], (min(rest) if rest else None)


@pytest.mark.parametrize("grid", [(32, 16, 48), (8, 100, 100), (20, 40, 50), (5, 200, 160), (64, 147, 210)])
def test_grid_search_argmin_matches_independent_model(oracle_mod, grid):
    """Random blocks: the oracle's choice over the grid is the exact argmin
    of the independent model over the same candidate set."""
    n, p, q = grid
    x = workloads.as_oracle_array(workloads.generate(workloads.with_shape(workloads.SEARCH_4K, 2, 512, 40 + n)))
    xf = oracle_mod.bf16_to_f32(x).reshape(-1, 16)
    packed, scales, g, loss = oracle_mod.nvfp4_scale_search_grid(x, n, p, q)
    s, lo = scales.reshape(-1), loss.reshape(-1)
    checked = 0
    for b in range(xf.shape[0]):
        xs = [float(v) for v in xf[b]]
        best, best_loss, runner = model_grid_search(xs, g, n, p, q)
        assert abs(Fraction(float(lo[b])) - best_loss) <= best_loss * Fraction(1, 10 ** 12)
        if runner is not None and runner != best_loss and abs(runner - best_loss) <= best_loss * Fraction(1, 10 ** 12):
            continue
        assert int(s[b]) == best, f"grid {grid} block {b}: oracle chose {s[b]}, the exact argmin is {best}"
        checked += 1
    assert checked >= 48


def test_grid_search_of_one_max_based_candidate_is_the_quantiser(oracle_mod):
    """n = 1 with p = q leaves only the max-based scale A_b / (6g): the
    search emits exactly the NVFP4 quantiser's codes and scales."""
    x = workloads.as_oracle_array(workloads.generate(workloads.with_shape(workloads.ACT_8K, 3, 256, 41)))
    for p in (1, 7, 210):
        packed, scales, g, _ = oracle_mod.nvfp4_scale_search_grid(x, 1, p, p)
        p0, s0, g0 = oracle_mod.nvfp4_quantize(x)
        assert g == g0
        assert np.array_equal(packed, p0) and np.array_equal(scales, s0)


def test_grid_search_rejects_empty_and_oversized_grids(oracle_mod):
    x = np.zeros((1, 16), np.float32)
    for n, p, q in ((0, 147, 210), (64, 0, 210), (64, 147, 0), (2, 1 << 20, 4), (4, 16, (1 << 20) + 1)):
        with pytest.raises(Exception):
            oracle_mod.nvfp4_scale_search_grid(x, n, p, q)
