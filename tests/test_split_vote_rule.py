"""Host model of the column-split prefill kernel's skip vote.

The every-row rule of "Accelerating Long-Context Inference with Skip Softmax
in NVIDIA TensorRT-LLM" (Key Points; Detailed Analysis) skips a tile when,
for every row, the tile's maximum lies below the running maximum minus tau.
In the column-split kernel each softmax warpgroup holds one half of a row's
key columns, so it knows only its half maximum before the per-tile exchange.
The kernel votes per half:

    row passes  <=>  row invalid, or (m != -inf and both halves pass)
    half passes <=>  m_h == -inf  or  m_h < m - tau

and skips the tile iff every warp's rows pass in both halves.  These tests
check, in the kernel's fp32 arithmetic, that this is the full-tile test

    row passes  <=>  row invalid, or (m != -inf and (mt == -inf or mt < m - tau)),
    mt = max(m_A, m_B),

on random rows and on the edge cases (-inf halves, ties at the threshold,
rows with no history, invalid rows).  No GPU is involved."""
import numpy as np
import pytest

NEG_INF = np.float32(-np.inf)


def full_tile_pass(mA, mB, m, tau, valid):
    mt = np.maximum(mA, mB)
    thr = (m - tau).astype(np.float32)
    return ~valid | ((m != NEG_INF) & ((mt == NEG_INF) | (mt < thr)))


def half_votes_pass(mA, mB, m, tau, valid):
    thr = (m - tau).astype(np.float32)
    half = lambda mh: (mh == NEG_INF) | (mh < thr)  # noqa: E731
    passA = ~valid | ((m != NEG_INF) & half(mA))
    passB = ~valid | ((m != NEG_INF) & half(mB))
    return passA & passB


def tile_skipped(row_pass, warp_rows=32):
    """Every warp's rows pass (the kernel's skip), rows grouped by warp."""
    return bool(row_pass.reshape(-1, warp_rows).all())


@pytest.mark.parametrize("seed", range(20))
def test_half_votes_equal_full_tile_test_random(seed):
    rng = np.random.default_rng(seed)
    rows = 128
    tau = np.float32(rng.choice([0.0, 0.5, 2.0, 4.0 * 1.4426950408889634, 8.0]))
    m = rng.normal(0, 4, rows).astype(np.float32)
    # halves mostly below the running max, some above, some far below
    mA = (m - rng.exponential(tau + 1.0, rows) + rng.normal(0, 1, rows)).astype(np.float32)
    mB = (m - rng.exponential(tau + 1.0, rows) + rng.normal(0, 1, rows)).astype(np.float32)
    valid = rng.random(rows) > 0.05
    for arr in (mA, mB):
        arr[rng.random(rows) < 0.1] = NEG_INF  # fully masked halves
    m[rng.random(rows) < 0.03] = NEG_INF  # rows with no history
    full = full_tile_pass(mA, mB, m, tau, valid)
    half = half_votes_pass(mA, mB, m, tau, valid)
    assert np.array_equal(full, half)
    assert tile_skipped(full) == tile_skipped(half)


def test_half_votes_edge_cases():
    tau = np.float32(2.0)
    m = np.array([5.0, 5.0, 5.0, 5.0, -np.inf, 5.0, 5.0, 5.0], np.float32)
    thr = np.float32(m[0] - tau)
    below = np.nextafter(thr, np.float32(-np.inf))
    mA = np.array([below, thr, -np.inf, -np.inf, 0.0, below, 9.0, below], np.float32)
    mB = np.array([below, below, -np.inf, thr, 0.0, 9.0, below, -np.inf], np.float32)
    valid = np.array([True, True, True, True, True, False, True, True])
    full = full_tile_pass(mA, mB, m, tau, valid)
    half = half_votes_pass(mA, mB, m, tau, valid)
    assert np.array_equal(full, half)
    # strict: a half maximum equal to m - tau keeps the row
    assert list(full) == [True, False, True, False, False, True, False, True]


def test_one_failing_half_keeps_the_tile():
    """A warp whose rows fail in its own half knows the tile is kept without
    reading the other votes: a failing half fails the row, hence the tile."""
    rng = np.random.default_rng(7)
    rows = 128
    tau = np.float32(4.0)
    m = np.full(rows, 10.0, np.float32)
    mA = np.full(rows, 0.0, np.float32)
    mB = np.full(rows, 0.0, np.float32)
    valid = np.ones(rows, bool)
    assert tile_skipped(half_votes_pass(mA, mB, m, tau, valid))
    r = int(rng.integers(rows))
    mB[r] = np.float32(7.0)  # above 10 - 4 in half B only
    assert not tile_skipped(half_votes_pass(mA, mB, m, tau, valid))
    assert not tile_skipped(full_tile_pass(mA, mB, m, tau, valid))
