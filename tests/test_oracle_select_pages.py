"""Pins for the oracle's page-granular selection: page size 1 is the token selection
(pinned on its own by a full stable sort), a brute-force page sort with Python floats,
invariants, the budget arithmetic worked by hand, and float32 page sums added in order."""
import numpy as np
import pytest

from oracle import s3r_oracle as O


def brute_pages(sigma, L, bp, W, P):
    """Whole pages by a stable sort of (-page score, page); page scores added one position
    at a time in Python floats of the given precision."""
    n = -(-(L * bp) // 10000)
    w = min(W, L)
    n = min(max(n, w), L)
    fw = (L - w) // P
    nwp = -(-L // P) - fw
    m = max(-(-n // P) - nwp, 0)
    cast = type(sigma[0]) if len(sigma) else float
    score = []
    for q in range(fw):
        acc = sigma[q * P]
        for t in range(1, P):
            acc = cast(acc + sigma[q * P + t])
        score.append(acc)
    order = sorted(range(fw), key=lambda q: (-score[q], q))
    pages = sorted(order[:m])
    return [q * P + t for q in pages for t in range(P)] + list(range(fw * P, L))


@pytest.mark.parametrize("seed", range(40))
def test_page_size_one_is_token_selection(seed):
    rng = np.random.default_rng(seed)
    L = int(rng.integers(1, 80))
    W = int(rng.integers(1, 12))
    bp = int(rng.integers(1, 10001))
    sigma = rng.integers(0, 5, size=L).astype(np.float64) / 4.0
    assert O.select_pages(sigma, L, bp, W, page=1).tolist() == O.select_positions(sigma, L, bp, W).tolist()


@pytest.mark.parametrize("seed", range(60))
def test_pages_match_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    P = int(rng.choice([2, 4, 16]))
    L = int(rng.integers(1, 400))
    W = int(rng.integers(1, 40))
    bp = int(rng.integers(1, 10001))
    if seed % 2:
        sigma = (rng.integers(0, 3, size=L) / 8.0).astype(np.float64)      # page ties
        ref = brute_pages([float(x) for x in sigma], L, bp, W, P)
    else:
        sigma = rng.random(L).astype(np.float32)
        ref = brute_pages([np.float32(x) for x in sigma], L, bp, W, P)
    assert O.select_pages(sigma, L, bp, W, page=P).tolist() == ref


def test_float32_page_sums_are_in_position_order():
    # 1 + 2^-24 + 2^-24 ... : in order each tiny add is lost; pairwise it would survive
    x = np.array([1.0] + [2.0 ** -24] * 15, dtype=np.float32)
    assert O.page_scores(x, 1, 16)[0] == np.float32(1.0)
    y = np.array([2.0 ** -24] * 15 + [1.0], dtype=np.float32)
    assert O.page_scores(y, 1, 16)[0] == np.float32(1.0) + np.float32(15 * 2.0 ** -24)


def test_page_budget_worked_examples():
    sig = np.zeros(24576)
    # L = 24576, s = 0.05, W = 64: n = 1229 -> 77 pages; the window is 4 whole pages
    got = O.select_pages(sig, 24576, 500, 64)
    assert got.size == 77 * 16 and got[-64:].tolist() == list(range(24512, 24576))
    # L = 1000, W = 64: window 936..999 starts inside page 58 -> pages 58..62 (5 pages,
    # 72 positions); n = 64 -> 4 pages <= 5: window pages only
    got = O.select_pages(sig, 1000, 500, 64)
    assert got.tolist() == list(range(928, 1000))
    # L = 20 < W: everything
    assert O.select_pages(sig, 20, 500, 64).tolist() == list(range(20))


@pytest.mark.parametrize("seed", range(10))
def test_page_selection_invariants(seed):
    rng = np.random.default_rng(200 + seed)
    L = int(rng.integers(2000, 30000))
    bp = int(rng.choice([200, 500, 1000, 2000]))
    sigma = rng.random(L) ** 4
    got = O.select_pages(sigma, L, bp, 64)
    n, w = O.budget_count(L, bp, 64)
    assert np.all(np.diff(got) > 0) and got[-1] == L - 1
    pages = np.unique(got // 16)
    assert got.size == sum(min(16, L - 16 * q) for q in pages)         # whole pages
    assert set(range(L - w, L)) <= set(got.tolist())
    assert got.size <= n + 15
    fw = (L - w) // 16
    ps = O.page_scores(sigma, fw, 16)
    cand = pages[pages < fw]
    rest = np.setdiff1d(np.arange(fw), cand)
    if cand.size and rest.size:
        assert ps[cand].min() >= ps[rest].max()
    assert O.select_pages(sigma, L, 10000, 64).tolist() == list(range(L))   # s = 1
