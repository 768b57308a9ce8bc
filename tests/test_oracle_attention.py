"""Pins for the oracle's dense verify attention, score capture and sparse draft attention.

The oracle is checked against things other than itself: a brute-force scalar loop,
closed forms, and the reduction of sparse attention to dense attention at s = 1.
"""
import math

import numpy as np
import pytest

from oracle import s3r_oracle as O


def brute_attention(q, K, V):
    """Scalar loops: logits, max, exponentials, normaliser, weighted sum."""
    n, d = K.shape
    logits = []
    for j in range(n):
        acc = 0.0
        for c in range(d):
            acc += q[c] * K[j][c]
        logits.append(acc / math.sqrt(d))
    m = max(logits)
    ex = [math.exp(x - m) for x in logits]
    z = sum(ex)
    out = [0.0] * d
    for j in range(n):
        for c in range(d):
            out[c] += ex[j] / z * V[j][c]
    return out, m + math.log(z), [e / z for e in ex]


@pytest.mark.parametrize("seed", range(5))
def test_attention_row_matches_brute_force(seed):
    rng = np.random.default_rng(seed)
    n, d = rng.integers(1, 9), 4
    q, K, V = rng.normal(size=d), rng.normal(size=(n, d)), rng.normal(size=(n, d))
    o, lse, p, s = O.attention_row(q, K, V)
    bo, blse, bp = brute_attention(q, K, V)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    assert abs(lse - blse) < 1e-12
    np.testing.assert_allclose(p, bp, rtol=1e-12, atol=1e-14)


def test_verify_block_matches_brute_force_with_causal_block():
    rng = np.random.default_rng(7)
    Hq, Hkv, d, L, T = 4, 2, 4, 5, 3
    q = rng.normal(size=(T, Hq, d))
    K = rng.normal(size=(Hkv, L + T, d))
    V = rng.normal(size=(Hkv, L + T, d))
    out, lse, sigma, logits = O.verify_attention(q, K, V, L)
    G = Hq // Hkv
    sig = np.zeros((Hkv, L + T))
    for h in range(Hq):
        kvh = h // G
        for t in range(T):
            vis = L + t + 1           # row t sees positions 0 .. L+t only
            bo, blse, bp = brute_attention(q[t, h], K[kvh, :vis], V[kvh, :vis])
            np.testing.assert_allclose(out[t, h], bo, rtol=1e-12, atol=1e-12)
            assert abs(lse[t, h] - blse) < 1e-12
            sig[kvh, :vis] += bp
            assert np.all(np.isneginf(logits[kvh, t * G + h % G, vis:]))
    np.testing.assert_allclose(sigma, sig, rtol=1e-12, atol=1e-14)


def test_closed_forms():
    rng = np.random.default_rng(1)
    d = 8
    V = rng.normal(size=(6, d))
    K = rng.normal(size=(6, d))
    # one visible position: the output is that value row, lse is its logit
    o, lse, p, s = O.attention_row(rng.normal(size=d), K[:1], V[:1])
    np.testing.assert_allclose(o, V[0], rtol=0, atol=1e-15)
    assert p[0] == 1.0
    # zero query: uniform weights, output = mean of V, lse = log n
    o, lse, p, _ = O.attention_row(np.zeros(d), K, V)
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=1e-13, atol=1e-15)
    assert abs(lse - math.log(6)) < 1e-13
    # identical keys: uniform weights whatever the query
    Ke = np.repeat(K[:1], 6, axis=0)
    o, _, p, _ = O.attention_row(rng.normal(size=d), Ke, V)
    np.testing.assert_allclose(p, np.full(6, 1 / 6), rtol=1e-13)
    np.testing.assert_allclose(o, V.mean(axis=0), rtol=1e-12, atol=1e-14)
    # one dominant key: output -> that value row
    Kd = np.zeros((6, d))
    Kd[3, 0] = 1e3
    qd = np.zeros(d)
    qd[0] = 1.0
    o, _, _, _ = O.attention_row(qd, Kd, V)
    np.testing.assert_allclose(o, V[3], rtol=0, atol=1e-12)


def test_scores_sum_to_rows_and_are_nonnegative():
    rng = np.random.default_rng(3)
    Hq, Hkv, d, L, T = 8, 2, 16, 40, 7
    q = rng.normal(size=(T, Hq, d))
    K = rng.normal(size=(Hkv, L + T, d)) * 3
    V = rng.normal(size=(Hkv, L + T, d))
    _, lse, sigma, logits = O.verify_attention(q, K, V, L)
    G = Hq // Hkv
    np.testing.assert_allclose(sigma.sum(axis=1), np.full(Hkv, G * T), rtol=1e-12)
    assert np.all(sigma >= 0)
    # the last block position is seen only by the last row of each head
    assert np.all(sigma[:, L + T - 1] <= G + 1e-12)
    # scores rebuilt from the captured logits and lse (row t*G+g <-> lse[t, kvh*G+g])
    for kvh in range(Hkv):
        rows_lse = np.array([lse[t, kvh * G + g] for t in range(T) for g in range(G)])
        np.testing.assert_allclose(O.scores_from_logits(logits[kvh], rows_lse), sigma[kvh],
                                   rtol=1e-12, atol=1e-15)


def test_sparse_draft_at_full_budget_equals_dense_row():
    """s = 1 selects every committed position, so draft step i equals verify row i."""
    rng = np.random.default_rng(5)
    Hq, Hkv, d, L, k = 4, 2, 16, 50, 6
    q = rng.normal(size=(k + 1, Hq, d))
    K = rng.normal(size=(Hkv, L + k + 1, d))
    V = rng.normal(size=(Hkv, L + k + 1, d))
    sigma = rng.random(L)
    sel = [O.select_positions(sigma, L, 10000, 4) for _ in range(Hkv)]
    assert all(np.array_equal(s, np.arange(L)) for s in sel)
    out, lse, _, _ = O.verify_attention(q, K, V, L)
    for i in range(k):
        o, l = O.sparse_draft_attention(q[i], K, V, sel, L, i)
        np.testing.assert_allclose(o, out[i], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(l, lse[i], rtol=1e-13)


def test_sparse_draft_single_position_is_value_row():
    rng = np.random.default_rng(9)
    Hq, Hkv, d, L = 2, 1, 8, 30
    K = rng.normal(size=(Hkv, L + 1, d))
    V = rng.normal(size=(Hkv, L + 1, d))
    o, _ = O.sparse_draft_attention(rng.normal(size=(Hq, d)), K, V, [np.zeros(0, np.int32)], L, 0)
    np.testing.assert_allclose(o, np.repeat(V[0, L][None], Hq, axis=0), rtol=0, atol=1e-15)


def test_sparse_draft_matches_brute_force_on_subset():
    rng = np.random.default_rng(11)
    Hq, Hkv, d, L, i = 4, 2, 4, 20, 2
    K = rng.normal(size=(Hkv, L + i + 1, d))
    V = rng.normal(size=(Hkv, L + i + 1, d))
    q = rng.normal(size=(Hq, d))
    sel = [np.array([1, 4, 9, 17]), np.array([0, 2, 19])]
    o, _ = O.sparse_draft_attention(q, K, V, sel, L, i)
    for h in range(Hq):
        kvh = h // 2
        rows = list(sel[kvh]) + list(range(L, L + i + 1))
        bo, _, _ = brute_attention(q[h], K[kvh, rows], V[kvh, rows])
        np.testing.assert_allclose(o[h], bo, rtol=1e-12, atol=1e-13)


def test_gather_positions_follows_page_table():
    P, H, d = 5, 2, 3
    pool = np.arange(P * H * 16 * d, dtype=np.float64).reshape(P, H, 16, d)
    pt = np.array([3, 0, 4])
    rows = O.gather_positions(pool, pt, 1, [0, 15, 16, 40])
    np.testing.assert_array_equal(rows[0], pool[3, 1, 0])
    np.testing.assert_array_equal(rows[1], pool[3, 1, 15])
    np.testing.assert_array_equal(rows[2], pool[0, 1, 0])
    np.testing.assert_array_equal(rows[3], pool[4, 1, 8])
    with pytest.raises(IndexError):
        O.gather_positions(pool, np.array([1, -1]), 0, [20])
