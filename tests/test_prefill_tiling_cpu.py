"""The windowed prefill kernel's tile classification, checked by brute force on the
host.

prefill_tc.cu visits a warp's KV tiles from the diagonal towards key 0.  A warp
quarter's elements on a tile have distances lo .. lo + BN + 30 (lo = centre +
32 q - 127).  Pairs with W_i < lo + BN - 1 + kZeroOffset are zeroed in its rows
of Q~, and a run of "clean" tiles is skipped through with no per-pair work.  Its
length follows from the first window not below lo and the span
kCleanSpan = 2 BN - 1 + kZeroOffset.  This file restates that rule and
simulates the zeroed set along a warp's tiles.  For every zeroing offset in the
range the kernel accepts (-96 .. 1), and for the pages' window tables and random
ones, it checks these invariants:
  - on a clean tile every pair is dead for all of the warp's elements or live for
    all of them, exactly the live ones are still in Q~, and no pair dies after it;
  - a correcting tile finds zeroed in Q~ exactly the pairs its zero point names;
  - the pairs added back on a correcting tile were zeroed after the previous
    correcting tile (the recently zeroed pairs the kernel keeps in shared memory).
The invariants hold at -97 too (a window equal to a tile's largest distance is
still live for all its elements), so the kernel's compile-time bound is one
tighter than needed.  The file also checks that they break at -98 and 2, and
with the span fixed at one offset's value: the form the rule had before it was
derived from the offset.
"""
import bisect
import os
import re

import numpy as np
import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "rope_frequency_sparse_b200", "csrc", "prefill_tc.cu")


def _kernel_constants():
    text = open(SRC).read()
    bn = int(re.search(r"constexpr int BN = (\d+);", text).group(1))
    off = int(re.search(r"constexpr int kZeroOffset = (-?\d+);", text).group(1))
    derived = re.search(r"constexpr int kCleanSpan = 2 \* BN - 1 \+ kZeroOffset;", text) is not None
    return bn, off, derived


BN, KERNEL_OFFSET, SPAN_DERIVED = _kernel_constants()


class Violation(AssertionError):
    pass


def walk(W, lo0, off, span, bn=BN):
    """Visit one warp quarter's tiles (smallest distance lo0, lo0 + bn, ...) until
    every window lies behind; raise Violation at the first broken invariant.
    Returns the number of clean and of correcting tiles."""
    W = list(W)
    npairs = len(W)

    def below(x):
        return bisect.bisect_left(W, x)

    def zero_point(lo):
        return below(lo + bn - 1 + off)

    n_tiles = (max(W) - lo0) // bn + 3
    zeroed = zero_point(lo0)  # the Q tile's first KV tile
    z_prev = None
    t = clean = corr = 0
    while t < n_tiles:
        lo = lo0 + bn * t
        a_run = below(lo)
        if a_run >= npairs:
            run = 0
        else:
            excess = W[a_run] - lo - (span - 1)
            run = 0 if excess <= 0 else min(-(-excess // bn), n_tiles - t)
        if run:
            # the conditions are monotone in lo: the run's first and last tiles decide
            last = lo + bn * (run - 1)
            if zeroed != a_run:
                raise Violation(f"clean run at lo={lo}: {zeroed} pairs zeroed, {a_run} dead")
            if below(last + bn + 30) != a_run:
                raise Violation(f"clean tile at lo={last}: a window crosses the elements")
            if zero_point(last + bn) != zeroed:
                raise Violation(f"clean tile at lo={last}: pairs die at the next tile")
            clean += run
            t += run
        if t >= n_tiles:
            break
        lo = lo0 + bn * t
        z = zero_point(lo)
        if zeroed != z:
            raise Violation(f"correcting tile at lo={lo}: {zeroed} pairs zeroed, zero point {z}")
        if z_prev is not None and below(lo) < z_prev:
            raise Violation(f"correcting tile at lo={lo}: adds back a pair zeroed before the previous one")
        z_prev = z
        zeroed = max(zeroed, zero_point(lo + bn))
        corr += 1
        t += 1
    return clean, corr


def _tables():
    out = []
    for d, theta in ((128, 1e7), (128, 1e4), (64, 1e4), (128, 5e5)):
        for alpha in (0.25, 1.0, 2.0):
            out.append([int(x) for x in oracle.windows(d, theta, alpha)[0]])
    rng = np.random.default_rng(7)
    for _ in range(12):  # clustered, duplicated and widely spaced windows
        steps = rng.choice([0, 1, 3, 17, 40, 90, 130, 300, 2000], size=64)
        out.append([int(x) for x in np.cumsum(steps) + int(rng.integers(1, 50))])
    return out


TABLES = _tables()
STARTS = [c + 32 * q - (BN - 1) for c in range(-(BN - 1), BN, 9) for q in range(4)]


def _holds(off, span):
    try:
        for W in TABLES:
            for lo0 in STARTS:
                walk(W, lo0, off, span)
    except Violation:
        return False
    return True


def test_kernel_uses_the_checked_rule():
    assert BN == 128
    assert SPAN_DERIVED, "the clean span is no longer 2 BN - 1 + kZeroOffset"
    assert -96 <= KERNEL_OFFSET <= 1


@pytest.mark.parametrize("off", [1, 0, -16, -47, -48, -49, -80, -95, -96, -97])
def test_invariants_hold_across_the_offset_range(off):
    assert _holds(off, 2 * BN - 1 + off)


def test_walks_take_clean_runs():
    # the rule is not vacuous: long clean runs, few correcting tiles
    clean, corr = walk([int(x) for x in oracle.windows(128, 1e7, 1.0)[0]], -127, KERNEL_OFFSET,
                       2 * BN - 1 + KERNEL_OFFSET)
    assert clean > 100 * corr > 0


@pytest.mark.parametrize("off", [2, -98])
def test_invariants_break_outside_the_range(off):
    assert not _holds(off, 2 * BN - 1 + off)


@pytest.mark.parametrize("off", [1, -16])
def test_a_span_fixed_for_another_offset_breaks(off):
    assert not _holds(off, 2 * BN - 1 - 48)
