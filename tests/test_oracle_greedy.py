"""Pins of the oracle's greedy (temperature 0) mode: argmax by brute force, ties to the
lowest id, NaN as -inf, and the greedy round's invariants."""
import numpy as np

from oracle import s3r_oracle as O


def test_argmax_brute_force_and_ties():
    rng = np.random.default_rng(0)
    for _ in range(200):
        V = int(rng.integers(1, 50))
        x = rng.integers(-3, 4, size=V).astype(np.float64)   # many ties
        best = max(range(V), key=lambda v: (x[v], -v))     # brute force: max value, lowest id
        assert O.argmax_token(x) == best
    assert O.argmax_token([np.nan, 1.0, 1.0]) == 1
    assert O.argmax_token([-np.inf, -np.inf]) == 0


def test_greedy_verify_round():
    rng = np.random.default_rng(1)
    V, k = 20, 6
    p = rng.normal(size=(k + 1, V))
    am = [int(np.argmax(p[j])) for j in range(k + 1)]
    # all drafts equal the target argmax: k accepted + bonus
    toks, n = O.greedy_verify(p, am[:k])
    assert n == k + 1 and toks.tolist() == am
    # first mismatch at j: the j agreeing drafts, then the target argmax of row j
    for j in range(k):
        d = list(am[:k])
        d[j] = (am[j] + 1) % V
        toks, n = O.greedy_verify(p, d)
        assert n == j + 1 and toks.tolist() == am[: j + 1]
    # with identical draft and target rows, greedy drafting is always fully accepted
    drafts = [O.argmax_token(p[j]) for j in range(k)]
    assert O.greedy_verify(p, drafts)[1] == k + 1
