"""Pins for the oracle's boundary margins: the values that decide which GPU/oracle
disagreements a parity test may excuse.

Every case is worked by hand from the definitions, with scores and probabilities chosen
as exact binary fractions so that the expected margins are exact:
  * selection: a non-window position (or page) is a boundary case when its score lies
    within rel * threshold of the threshold, the M-th largest score, band edges included
    ([Explainer] walkthrough: the most-attended positions / top-scoring pages are kept);
  * inverse-CDF draw of v: the distance of u to the nearer edge of v's cell,
    [C_{v-1} / Z, C_v / Z), C the inclusive cumulative sum of the weights;
  * accept test of a draft d: |u - p(d) / q(d)| ([News] Interpretation, [Explainer]
    Jargon: exact speculative sampling accepts with probability min(1, p/q)).
A margin taken against the wrong edge, a band measured in absolute units or around the
wrong order statistic, or a p/q ratio inverted fails one of these cases.
"""
import math

import numpy as np
import pytest

from oracle import s3r_oracle as O

EPS = 2.0 ** -10   # relative band used below (exact in binary)


# ------------------------------------------------------------------ token selection ----
def test_selection_margin_band_edges_are_exact():
    # L = 12, W = 2: non-window positions 0..9; bp 5800 -> n = ceil(6.96) = 7, M = 5.
    # Non-window scores sorted: 8, 4, 2 + 2^-8, 2 + 2^-9, 2 (the 5th largest: threshold
    # T = 2), 2 - 2^-9, 2 - 2^-8, 1, 0.5, 0.25.
    T = 2.0
    sigma = np.array([8.0, T + 2 * T * EPS, T, 4.0, T - T * EPS, T + T * EPS,
                      0.5, T - 2 * T * EPS, 0.25, 1.0, 7.0, 7.0])
    sel = O.select_positions(sigma, 12, 5800, 2)
    assert sel.tolist() == [0, 1, 2, 3, 5, 10, 11]
    # T + T*EPS (position 5) and T - T*EPS (position 4) sit exactly on the band's edges
    # (|s - T| = EPS * T): included; T +- 2 T EPS (positions 1, 7) lie outside.
    assert O.selection_margin_cases(sigma, 12, 5800, 2, rel=EPS).tolist() == [2, 4, 5]
    # the band is relative to the threshold: the same offsets around a threshold 8x larger
    assert O.selection_margin_cases(sigma * 8, 12, 5800, 2, rel=EPS).tolist() == [2, 4, 5]
    # a smaller band keeps only the threshold position itself
    assert O.selection_margin_cases(sigma, 12, 5800, 2, rel=EPS / 4).tolist() == [2]
    # M = 4 (bp 5000 -> n = 6): the threshold moves up to 2 + 2^-9 (position 5), and the
    # band with it: positions 1 and 2 lie on its edges, position 4 outside
    assert O.selection_margin_cases(sigma, 12, 5000, 2, rel=EPS).tolist() == [1, 2, 5]


def test_selection_margin_uses_the_mth_largest_score():
    # M = 1 (bp 2500, L = 8, W = 1 -> n = 2): threshold = the largest non-window score
    sigma = np.array([1.0, 3.0, 3.0 - 3.0 * EPS, 2.0, 3.0 - 3.0 * EPS / 2, 0.0, 0.0, 9.0])
    assert O.select_positions(sigma, 8, 2500, 1).tolist() == [1, 7]
    assert O.selection_margin_cases(sigma, 8, 2500, 1, rel=EPS).tolist() == [1, 2, 4]
    # ties at the threshold are all boundary cases (their order decides which are kept)
    sigma = np.array([5.0, 1.0, 1.0, 1.0, 0.0, 9.0])
    assert O.select_positions(sigma, 6, 5000, 1).tolist() == [0, 1, 5]
    assert O.selection_margin_cases(sigma, 6, 5000, 1, rel=EPS).tolist() == [1, 2, 3]


def test_selection_margin_empty_when_the_window_fills_the_budget():
    sigma = np.linspace(1.0, 2.0, 100)
    assert O.selection_margin_cases(sigma, 100, 100, 8).size == 0      # n = 1 < W
    assert O.selection_margin_cases(sigma, 4, 10000, 8).size == 0      # L < W


# ------------------------------------------------------------------- page selection ----
def _pages(page_scores, page=4, tail=()):
    """Per-position scores whose page sums are the given values (each position holds a
    quarter of its page's score, exact in binary), followed by `tail` positions."""
    s = np.repeat(np.asarray(page_scores, dtype=np.float64) / page, page)
    return np.concatenate([s, np.asarray(tail, dtype=np.float64)])


def test_page_margin_band_edges_are_exact():
    # page size 4, L = 32, W = 4: candidate pages 0..6 (page 7 holds the window).
    # bp 6250 -> n = 20 -> 5 pages in all, 1 of them the window page -> M = 4.
    # Page scores sorted: 8, 4, 1 + 2^-9, 1 + 2^-10 ... the 4th largest: T = 1 + 2^-10.
    T = 1.0 + EPS
    ps = [8.0, T - T * EPS, T, 4.0, 0.5, 1.0 + 2 * EPS, T - 3 * T * EPS]
    sigma = _pages(ps, tail=[1.0, 1.0, 1.0, 1.0])
    sel = O.select_pages(sigma, 32, 6250, 4, page=4)
    assert sel.tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 12, 13, 14, 15, 20, 21, 22, 23,
                            28, 29, 30, 31]
    # page 1 sits on the lower band edge (T - T*EPS), page 2 is the threshold page; page 5
    # is T + 2^-10 (1 + 2^-9 vs T = 1 + 2^-10: offset 2^-10 < T * EPS): inside; page 6
    # lies 3 T EPS below: outside
    assert O.page_selection_margin_cases(sigma, 32, 6250, 4, page=4, rel=EPS).tolist() == [1, 2, 5]


def test_page_margin_is_taken_on_page_sums_not_positions():
    # two pages with equal sums but different position scores: both at the threshold
    sigma = np.array([4.0, 0.0, 0.0, 0.0,  1.0, 1.0, 1.0, 1.0,  9.0, 9.0, 9.0, 9.0,
                      0.5, 0.5, 0.5, 0.5,  1.0, 1.0])
    # L = 18, W = 2 (first window page 4: positions 16, 17), bp 5000 -> n = 9 -> 3 pages
    # in all, 1 the window page -> M = 2: page 2 (36) and the tie 4.0 at pages 0 and 1
    assert O.select_pages(sigma, 18, 5000, 2, page=4).tolist() == [0, 1, 2, 3, 8, 9, 10, 11, 16, 17]
    assert O.page_selection_margin_cases(sigma, 18, 5000, 2, page=4, rel=EPS).tolist() == [0, 1]


def test_page_margin_with_the_library_page_size():
    # 16-position pages: L = 200, W = 64 -> window pages from (200 - 64) // 16 = 8 on;
    # candidate pages 0..7; bp 5000 -> n = 100 -> ceil(100 / 16) = 7 pages, 5 of them the
    # window's (8..12) -> M = 2
    rng = np.random.default_rng(5)
    ps = np.array([3.0, 1.0, 6.0, 2.0, 2.0 + 2.0 * EPS, 0.5, 2.0 - 2.0 * EPS / 2, 1.5])
    sigma = np.concatenate([np.repeat(ps / 16, 16), rng.random(200 - 128)])
    assert O.page_selection_margin_cases(sigma, 200, 5000, 64, rel=EPS).tolist() == [0]
    # M = 4 (bp 7000 -> n = 140 -> 9 pages): threshold 2.0 (page 3)
    assert O.page_selection_margin_cases(sigma, 200, 7000, 64, rel=EPS).tolist() == [3, 4, 6]


# ---------------------------------------------------------------- inverse-CDF draws ----
@pytest.mark.parametrize("u, v, margin", [
    (0.1, 0, 0.1),       # cell [0, 1/4): edges 0 and 0.25
    (0.3, 1, 0.05),      # cell [1/4, 3/4): nearer edge is the lower one
    (0.7, 1, 0.05),      # ... and here the upper one
    (0.25, 1, 0.0),      # on the lower edge: u*Z = C_0 is not < C_0, so v = 1, margin 0
    (0.5, 1, 0.25),      # the cell's middle
    (0.875, 2, 0.125),   # last cell [3/4, 1)
])
def test_inverse_cdf_margin_is_the_distance_to_the_nearer_cell_edge(u, v, margin):
    got_v, got_m = O.inverse_cdf(np.array([1.0, 2.0, 1.0]), u)
    assert got_v == v
    assert got_m == pytest.approx(margin, abs=1e-15)


def test_inverse_cdf_margin_skips_zero_weight_cells():
    # weights 0, 1, 0, 1 (Z = 2): token 3's cell is [1/2, 1), its lower edge the cumulative
    # sum up to token 2 (which adds nothing), not a cell of zero width
    w = np.array([0.0, 1.0, 0.0, 1.0])
    assert O.inverse_cdf(w, 0.6) == (3, pytest.approx(0.1, abs=1e-15))
    assert O.inverse_cdf(w, 0.45) == (1, pytest.approx(0.05, abs=1e-15))
    # the scale of the weights does not matter
    assert O.inverse_cdf(w * 1e-30, 0.6)[1] == pytest.approx(0.1, abs=1e-15)


def test_draft_sample_margin_from_logits():
    # logits log(1), log(2), log(1): the same cells as weights 1, 2, 1
    lg = np.log(np.array([1.0, 2.0, 1.0]))
    v, m = O.draft_sample(lg, 0.74)
    assert v == 1 and m == pytest.approx(0.01, abs=1e-12)


# ----------------------------------------------------------- speculative sampling ----
P = np.array([0.5, 0.25, 0.25])
Q = np.array([0.25, 0.5, 0.25])


def test_spec_margins_reject_then_residual_draw():
    # draft 0 = token 0: p/q = 2 -> accepted for any u; margin |0.3 - 2| = 1.7.
    # draft 1 = token 1: p/q = 1/2, u = 0.7 -> rejected (0.7 * 0.5 >= 0.25); margin 0.2.
    # residual max(0, p - q) = (1/4, 0, 0): token 0, its cell [0, 1) -> margin
    # min(0.4, 0.6) = 0.4.
    pl = np.log(np.stack([P, P, P]))
    ql = np.log(np.stack([Q, Q]))
    toks, n_out, margins = O.spec_sample_request(pl, ql, [0, 1], [0.3, 0.7], [0.9, 0.4, 0.9])
    assert toks.tolist() == [0, 0] and n_out == 2
    assert margins == pytest.approx([1.7, 0.2, 0.4], abs=1e-12)


def test_spec_margins_all_accepted_then_bonus_draw():
    # draft 1 = token 2: p/q = 1, u = 0.7 -> accepted, margin 0.3; bonus from p row 2 =
    # (1/2, 1/4, 1/4) with u = 0.6: token 1 (cell [1/2, 3/4)), margin min(0.1, 0.15) = 0.1
    pl = np.log(np.stack([P, P, P]))
    ql = np.log(np.stack([Q, Q]))
    toks, n_out, margins = O.spec_sample_request(pl, ql, [0, 2], [0.3, 0.7], [0.9, 0.9, 0.6])
    assert toks.tolist() == [0, 2, 1] and n_out == 3
    assert margins == pytest.approx([1.7, 0.3, 0.1], abs=1e-12)


def test_spec_margin_at_the_accept_boundary_is_zero():
    # u exactly p/q: u * q < p fails (strict), so the draft is rejected with margin 0;
    # the residual (1/4, 0, 0) then gives token 0
    pl = np.log(np.stack([P, P]))
    ql = np.log(Q[None])
    toks, n_out, margins = O.spec_sample_request(pl, ql, [1], [0.5], [0.3, 0.3])
    assert toks.tolist() == [0] and n_out == 1
    assert margins[0] == pytest.approx(0.0, abs=1e-12)
    # just below the boundary the draft is accepted with a margin of the offset
    toks, n_out, margins = O.spec_sample_request(pl, ql, [1], [0.5 - 2.0 ** -20], [0.3, 0.3])
    assert toks.tolist()[:1] == [1] and n_out == 2
    assert margins[0] == pytest.approx(2.0 ** -20, rel=1e-6)


def test_spec_margin_of_a_residual_draw_is_in_residual_units():
    # p = (0.5, 0.3, 0.2), q = (0.1, 0.2, 0.7); draft token 2: p/q = 2/7, u = 0.9 -> rejected.
    # residual (0.4, 0.1, 0): Z = 0.5, cells [0, 0.8), [0.8, 1); u = 0.85 -> token 1,
    # margin min(0.05, 0.15) = 0.05 (a margin taken on p's cells would be min(0.05, 0.15)
    # around 0.8 = p's edge too -- so also check u = 0.75: residual token 0 with margin
    # 0.05, where p's cells would give token 1)
    p = np.array([0.5, 0.3, 0.2])
    q = np.array([0.1, 0.2, 0.7])
    pl, ql = np.log(np.stack([p, p])), np.log(q[None])
    toks, _, margins = O.spec_sample_request(pl, ql, [2], [0.9], [0.85, 0.0])
    assert toks.tolist() == [1]
    assert margins == pytest.approx([abs(0.9 - 2 / 7), 0.05], abs=1e-12)
    toks, _, margins = O.spec_sample_request(pl, ql, [2], [0.9], [0.75, 0.0])
    assert toks.tolist() == [0]
    assert margins[-1] == pytest.approx(0.05, abs=1e-12)


def test_spec_sample_uses_the_philox_streams_of_the_round():
    # spec_sample = spec_sample_request with u_accept from stream 1 and u_draw from stream
    # 2 at positions L+1 .. L+k+1 of request r
    rng = np.random.default_rng(11)
    k, V, seed, r, L = 4, 16, 77, 3, 1000
    pl = rng.normal(size=(k + 1, V))
    ql = pl[:k] + 0.5 * rng.normal(size=(k, V))
    drafts = rng.integers(0, V, size=k)
    ua = [float(O.uniform(seed, r, L + 1 + j, O.STREAM_ACCEPT)) for j in range(k)]
    ud = [float(O.uniform(seed, r, L + 1 + j, O.STREAM_DRAW)) for j in range(k + 1)]
    a = O.spec_sample(pl, ql, drafts, seed, r, L)
    b = O.spec_sample_request(pl, ql, drafts, ua, ud)
    assert a[0].tolist() == b[0].tolist() and a[1] == b[1]
    assert np.allclose(a[2], b[2])
    p, q = O.softmax64(pl), O.softmax64(ql)
    # every decided draft's margin is |u - p/q| of that draft
    for j in range(min(a[1], k)):
        d = int(drafts[j])
        assert a[2][j] == pytest.approx(abs(ua[j] - p[j, d] / q[j, d]), rel=1e-12)
    assert not math.isinf(a[2][-1])
