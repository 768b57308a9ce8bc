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


def test_greedy_round_with_equal_logits_accepts_every_draft():
    """A whole greedy oracle round: identical draft and target logits emit k + 1 tokens,
    the argmax of each target row."""
    rng = np.random.default_rng(5)
    k, L, Hkv, G, d, V = 4, 40, 1, 2, 8, 32
    K = rng.normal(size=(Hkv, L + k + 1, d))
    Vv = rng.normal(size=(Hkv, L + k + 1, d))
    st = O.RequestState(K.copy(), Vv.copy(), L)
    O.prefill_scores(st, rng.normal(size=(Hkv * G, d)), K[:, L], Vv[:, L])
    p = rng.normal(size=(k + 1, V))
    res = O.run_round(st, 0, 1, k, 2500, 8, rng.normal(size=(k + 1, Hkv * G, d)),
                      K[:, L:L + k + 1].transpose(1, 0, 2), Vv[:, L:L + k + 1].transpose(1, 0, 2),
                      p[:k], p, greedy=True)
    assert res["n_out"] == k + 1
    assert res["tokens"].tolist() == [int(np.argmax(p[j])) for j in range(k + 1)]
    assert res["drafts"].tolist() == [int(np.argmax(p[j])) for j in range(k)]
    assert st.L == L + k + 1
