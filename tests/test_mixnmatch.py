"""Layer-wise Mix'n'Match allocations ("Matryoshka Quantization | Summary", §4.3; App. B): the
budget holds, the allocation is maximal, each strategy has its shape, and the effective bits
agree with the oracle's accounting.  Host logic only (no GPU)."""

import itertools

import numpy as np
import pytest

import oracle as O
from nested_bit_weight_msb_b200 import mixnmatch as MM


def _mean(ws, sizes=None):
    sizes = np.ones(len(ws)) if sizes is None else np.asarray(sizes, dtype=np.float64)
    return float((np.asarray(ws) * sizes).sum() / sizes.sum())


def test_hand_worked_pyramid():
    # four equal layers, widths {2, 4, 8}, 4 bits: layers 1 and 2 are the middle; layer 1 takes
    # 8 (6 bits over 2 of the 8 available), layer 2 then fits 4 (the last 2), the ends stay at 2
    assert MM.allocate_widths(4, 4.0, "pyramid", (2, 4, 8)) == [2, 8, 4, 2]
    assert MM.allocate_widths(4, 4.0, "reverse_pyramid", (2, 4, 8)) == [8, 2, 2, 4]
    assert MM.allocate_widths(4, 4.0, "increasing", (2, 4, 8)) == [2, 2, 4, 8]
    assert MM.allocate_widths(4, 4.0, "decreasing", (2, 4, 8)) == [8, 4, 2, 2]


@pytest.mark.parametrize("strategy", MM.STRATEGIES)
@pytest.mark.parametrize("widths", [(2, 4, 8), (2, 3, 4), (3, 4, 8), (2, 3, 4, 6, 8), (4,)])
def test_budget_holds_and_allocation_is_maximal(strategy, widths):
    rng = np.random.default_rng(len(widths))
    for n in (1, 5, 32):
        for sizes in (None, list(rng.integers(1, 5, n))):
            for target in np.linspace(min(widths), max(widths), 9):
                ws = MM.allocate_widths(n, float(target), strategy, widths, sizes)
                assert all(r in widths for r in ws)
                m = _mean(ws, sizes)
                assert m <= target + 1e-12
                sz = [1] * n if sizes is None else sizes
                slack = target * sum(sz) - sum(r * s for r, s in zip(ws, sz))
                for l, r in enumerate(ws):
                    for r2 in widths:
                        if r2 > r:
                            assert (r2 - r) * sz[l] > slack + 1e-9, (l, r, r2)


def test_extreme_budgets():
    assert MM.allocate_widths(32, 2.0, "pyramid", (2, 4, 8)) == [2] * 32
    assert MM.allocate_widths(32, 8.0, "pyramid", (2, 4, 8)) == [8] * 32
    with pytest.raises(ValueError):
        MM.allocate_widths(8, 1.5, "pyramid", (2, 4, 8))
    with pytest.raises(ValueError):
        MM.allocate_widths(8, 3.0, "sideways")
    with pytest.raises(ValueError):
        MM.allocate_widths(8, 3.0, "pyramid", (2, 5))


@pytest.mark.parametrize("target", [2.5, 3.0, 4.0, 5.5])
def test_strategy_shapes(target):
    n = 32
    mid = (n - 1) / 2
    pyr = MM.allocate_widths(n, target, "pyramid", (2, 4, 8))
    rev = MM.allocate_widths(n, target, "reverse_pyramid", (2, 4, 8))
    inc = MM.allocate_widths(n, target, "increasing", (2, 4, 8))
    dec = MM.allocate_widths(n, target, "decreasing", (2, 4, 8))
    for a, b in itertools.combinations(range(n), 2):
        if abs(a - mid) < abs(b - mid):
            assert pyr[a] >= pyr[b] and rev[a] <= rev[b]
    assert all(x <= y for x, y in zip(inc, inc[1:]))
    assert all(x >= y for x, y in zip(dec, dec[1:]))
    assert pyr != inc and len(set(pyr)) > 1


def test_effective_bits_agree_with_the_oracle():
    rng = np.random.default_rng(0)
    ws = list(rng.choice([2, 3, 4, 6, 8], 32))
    sizes = list(rng.integers(1, 1000, 32))
    assert MM.effective_bits(ws) == pytest.approx(O.mixnmatch_effective_bits(ws), rel=1e-15)
    assert MM.effective_bits(ws, sizes) == pytest.approx(O.mixnmatch_effective_bits(ws, sizes), rel=1e-15)
    # the seeded {2 x 11, 3 x 10, 4 x 11} stack averages exactly 3 bits per weight
    from nested_bit_weight_msb_b200 import synth
    assert MM.effective_bits(synth.mixnmatch_widths(seed=0)) == 3.0
    # with metadata: 16-bit scale + 8-bit zero per group of 128 add 0.1875 bits a weight
    assert MM.effective_bits([4] * 8, group=128) == 4.1875
    assert MM.effective_bits([2, 8], group=64) == 5.375
