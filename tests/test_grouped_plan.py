"""The grouped calls' launch planner (host logic, no GPU): every item is
covered once, in order, by pieces that respect the launch limits."""
import random

import pytest

import block_scaled_fp4_reduce_b200 as fp4


def check_plan(units, max_units, max_entries):
    plan = fp4.grouped_plan(units, max_units, max_entries)
    # pieces of each item are contiguous, in order, and cover it exactly
    pos = {}
    order = []
    for launch, item, first, count in plan:
        assert count >= 0
        assert first == pos.get(item, 0), (item, first, pos.get(item, 0))
        pos[item] = first + count
        order.append(item)
    assert order == sorted(order)
    for i, u in enumerate(units):
        assert pos.get(i) == u, f"item {i}: covered {pos.get(i)} of {u}"
    # every item, empty ones included, has at least one piece
    assert set(order) == set(range(len(units)))
    # launches are numbered consecutively and respect both limits
    launches = {}
    for launch, item, first, count in plan:
        launches.setdefault(launch, []).append((item, first, count))
    assert sorted(launches) == list(range(len(launches)))
    for pieces in launches.values():
        assert len(pieces) <= max_entries
        assert sum(c for _, _, c in pieces) <= max_units
    # a piece that does not finish its item ends on a multiple of 64 units
    for launch, item, first, count in plan:
        if first + count < units[item]:
            assert (first + count) % 64 == 0 and count > 0
    return plan


def test_small_cases_by_hand():
    assert check_plan([], 128, 4) == []
    assert check_plan([0], 128, 4) == [(0, 0, 0, 0)]
    assert check_plan([100, 0, 300, 5], 128, 3) == [
        (0, 0, 0, 100), (0, 1, 0, 0), (1, 2, 0, 128), (2, 2, 128, 128), (3, 2, 256, 44), (3, 3, 0, 5)]
    # the entry limit alone starts a new launch
    assert check_plan([1, 1, 1], 1 << 20, 2) == [(0, 0, 0, 1), (0, 1, 0, 1), (1, 2, 0, 1)]


@pytest.mark.parametrize("seed", range(20))
def test_random_items(seed):
    rnd = random.Random(seed)
    n = rnd.randint(0, 600)
    units = [rnd.choice([0, rnd.randint(1, 100), rnd.randint(1, 5000)]) for _ in range(n)]
    check_plan(units, rnd.choice([64, 100, 1000, 4096, 1 << 30]), rnd.choice([1, 2, 7, 256]))


def test_seven_b_weight_set_fits_one_launch_of_the_largest_limits():
    # 32 layers x (4 x 4096^2 + 3 x 4096x14336) bf16 matrices, NVFP4 16-blocks
    units = [4096 * 4096 // 16] * 4 * 32 + [4096 * 14336 // 16] * 3 * 32
    plan = check_plan(units, 1 << 30, 256)
    assert max(p[0] for p in plan) + 1 == 1  # 486M blocks, 224 entries: one launch
    assert len(plan) == 224


def test_invalid_limits_rejected():
    for mu, me in ((63, 4), (128, 0), (128, 257), ((1 << 30) + 1, 4)):
        with pytest.raises(ValueError):
            fp4.grouped_plan([1, 2], mu, me)
