"""Pins for the oracle's sparse KV selection: a full stable sort on tiny inputs,
invariants on larger ones, and the budget arithmetic."""
import numpy as np
import pytest

from oracle import s3r_oracle as O


def brute_select(sigma, L, bp, W):
    """Stable sort of the non-window positions by (-score, position); take the first M."""
    n = -(-(L * bp) // 10000)
    w = min(W, L)
    n = min(max(n, w), L)
    order = sorted(range(L - w), key=lambda j: (-sigma[j], j))
    return sorted(order[: n - w]) + list(range(L - w, L))


@pytest.mark.parametrize("seed", range(40))
def test_select_matches_stable_sort_with_ties(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 60))
    W = int(rng.integers(1, 12))
    bp = int(rng.integers(1, 10001))
    sigma = rng.integers(0, 5, size=L).astype(np.float64) / 4.0   # many exact ties
    got = O.select_positions(sigma, L, bp, W)
    assert got.tolist() == brute_select(sigma, L, bp, W)


def test_budget_count_examples():
    assert O.budget_count(256, 2500, 16) == (64, 16)
    assert O.budget_count(300, 2500, 16) == (75, 16)
    assert O.budget_count(20, 500, 64) == (20, 20)          # L < W: whole context
    assert O.budget_count(1000, 500, 64) == (64, 64)        # n = 50 < W: window only
    assert O.budget_count(4096, 500, 64) == (205, 64)       # ceil(204.8)
    assert O.budget_count(16384, 500, 64) == (820, 64)      # ceil(819.2)
    assert O.budget_count(10000, 1, 1) == (1, 1)
    assert O.budget_count(24576, 10000, 64) == (24576, 64)


@pytest.mark.parametrize("seed", range(10))
def test_select_invariants(seed):
    rng = np.random.default_rng(100 + seed)
    L = int(rng.integers(200, 3000))
    W, bp = 64, int(rng.choice([200, 500, 1000, 2500]))
    sigma = rng.exponential(size=L)
    sel = O.select_positions(sigma, L, bp, W)
    n, w = O.budget_count(L, bp, W)
    assert sel.size == n
    assert np.all(np.diff(sel) > 0) and sel[0] >= 0 and sel[-1] < L
    assert set(range(L - w, L)) <= set(sel.tolist())
    nonwin = sel[sel < L - w]
    rest = np.setdiff1d(np.arange(L - w), nonwin)
    if nonwin.size and rest.size:
        assert sigma[nonwin].min() >= sigma[rest].max()


def test_select_full_budget_and_window_only():
    sigma = np.random.default_rng(0).random(100)
    assert O.select_positions(sigma, 100, 10000, 8).tolist() == list(range(100))
    assert O.select_positions(sigma, 100, 100, 8).tolist() == list(range(92, 100))


def test_margin_cases_flag_near_threshold():
    sigma = np.array([5.0, 1.0, 1.0 + 1e-7, 3.0, 0.5, 1.0, 9.0, 9.0])
    # L = 8, W = 2 -> non-window 0..5; n = ceil(8 * 0.5) = 4 -> M = 2 -> threshold 3.0
    assert O.select_positions(sigma, 8, 5000, 2).tolist() == [0, 3, 6, 7]
    assert O.selection_margin_cases(sigma, 8, 5000, 2).tolist() == [3]
    # M = 3 -> threshold 1.0000001: positions 1, 2, 5 lie within 1e-5 of it
    assert O.selection_margin_cases(sigma, 8, 6250, 2).tolist() == [1, 2, 5]
