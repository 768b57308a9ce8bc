"""Pins for the oracle's Philox stream and its draft / speculative sampling.

Philox is pinned to the published known-answer vectors. The samplers are pinned to
closed forms (uniform and one-hot distributions, identical draft and target), to the
standard speculative-sampling results (per-position acceptance = sum_v min(p_v, q_v);
E[tau] = 1 + sum_i prod_{j<=i} alpha_j; emitted tokens follow the target distribution),
with a negative control that must fail the same distribution test.
"""
import math

import numpy as np
import pytest
from scipy import stats

from oracle import s3r_oracle as O
from tests.conftest import read_golden


def test_philox_known_answer_vectors():
    rows = read_golden("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        w = [int(x, 16) for x in r]
        got = O.philox4x32_10(np.array(w[:4], dtype=np.uint64), np.array(w[4:6], dtype=np.uint64))
        assert got.tolist() == w[6:10]


def test_philox_vectorised_matches_elementwise():
    ctr = np.random.default_rng(0).integers(0, 2**32, size=(50, 4), dtype=np.uint64)
    key = np.random.default_rng(1).integers(0, 2**32, size=(50, 2), dtype=np.uint64)
    allv = O.philox4x32_10(ctr, key)
    for i in range(50):
        assert O.philox4x32_10(ctr[i], key[i]).tolist() == allv[i].tolist()


def test_uniforms_are_24_bit_and_uniform():
    u = O.uniform(1234, np.arange(200000) % 97, np.arange(200000) // 97, O.STREAM_ACCEPT)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert np.all(u * 2**24 == np.floor(u * 2**24))
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    # different streams / requests / seeds give different numbers
    a = O.uniform(1, 0, np.arange(1000), 0)
    assert not np.array_equal(a, O.uniform(1, 0, np.arange(1000), 1))
    assert not np.array_equal(a, O.uniform(1, 1, np.arange(1000), 0))
    assert not np.array_equal(a, O.uniform(2, 0, np.arange(1000), 0))
    # the 64-bit seed uses both key words
    assert not np.array_equal(a, O.uniform(1 + (1 << 32), 0, np.arange(1000), 0))


def test_inverse_cdf_closed_forms():
    V = 64
    for u in np.linspace(0, 1, 257)[:-1]:
        v, margin = O.inverse_cdf(np.ones(V), u)
        assert v == math.floor(u * V)                     # uniform distribution
        assert margin >= -1e-15
    w = np.zeros(V)
    w[17] = 3.0
    assert O.inverse_cdf(w, 0.0)[0] == 17 and O.inverse_cdf(w, 0.999)[0] == 17
    w = np.zeros(V)
    w[[3, 40]] = 1.0
    assert O.inverse_cdf(w, 0.49)[0] == 3 and O.inverse_cdf(w, 0.5)[0] == 40
    # rounding guard: a total that u*Z exceeds falls back to the last non-zero weight
    assert O.inverse_cdf(np.array([0.0, 1.0, 0.0]), 1.0)[0] == 1


def test_identical_draft_and_target_accept_everything():
    rng = np.random.default_rng(0)
    k, V = 6, 64
    logits = rng.normal(size=(k + 1, V)) * 1.4
    for r in range(300):
        drafts = rng.integers(0, V, size=k)
        toks, n_out, _ = O.spec_sample(logits, logits[:k], drafts, 99, r, 1000)
        assert n_out == k + 1 and toks[:k].tolist() == drafts.tolist()


def test_residual_draw_support():
    p = np.log(np.array([0.5, 0.5, 1e-300, 1e-300]))
    q = np.log(np.array([0.25, 0.25, 0.25, 0.25]))
    # draft token 3 has p ~ 0: always rejected; the residual lives on tokens 0 and 1
    seen = set()
    for r in range(200):
        toks, n_out, _ = O.spec_sample(np.stack([p, p]), q[None], [3], 5, r, 10)
        assert n_out == 1
        seen.add(int(toks[0]))
    assert seen == {0, 1}


def _trials(p_logits, q_logits, n_trials, seed=777, L=5000):
    """Run the oracle sampler for many requests; drafts are drawn from q as in a round."""
    k, V = q_logits.shape
    r = np.arange(n_trials)
    ud = np.stack([O.uniform(seed, r, L + 1 + j, O.STREAM_DRAFT) for j in range(k)], 1)
    ua = np.stack([O.uniform(seed, r, L + 1 + j, O.STREAM_ACCEPT) for j in range(k)], 1)
    uw = np.stack([O.uniform(seed, r, L + 1 + j, O.STREAM_DRAW) for j in range(k + 1)], 1)
    drafts = np.array([[O.draft_sample(q_logits[j], ud[t, j])[0] for j in range(k)]
                       for t in range(n_trials)])
    outs = [O.spec_sample_request(p_logits, q_logits, drafts[t], ua[t], uw[t])
            for t in range(n_trials)]
    return drafts, outs


@pytest.fixture(scope="module")
def tiny_model():
    rng = np.random.default_rng(42)
    k, V = 6, 64
    p_logits = rng.normal(size=(k + 1, V)) * math.sqrt(2.0)
    q_logits = p_logits[:k] + rng.normal(size=(k, V)) * 0.3
    return p_logits, q_logits


@pytest.fixture(scope="module")
def tiny_trials(tiny_model):
    p_logits, q_logits = tiny_model
    return _trials(p_logits, q_logits, 60000)


def test_acceptance_per_position_and_expected_tau(tiny_model, tiny_trials):
    p_logits, q_logits = tiny_model
    k = q_logits.shape[0]
    p, q = O.softmax64(p_logits), O.softmax64(q_logits)
    alpha = np.minimum(p[:k], q).sum(axis=1)
    drafts, outs = tiny_trials
    n_out = np.array([o[1] for o in outs])
    for j in range(k):
        reached = n_out >= j + 1                       # draft j was decided
        accepted = n_out >= j + 2
        n, a = reached.sum(), (reached & accepted).sum()
        lo, hi = stats.binomtest(int(a), int(n)).proportion_ci(0.999)
        assert lo <= alpha[j] <= hi, (j, a / n, alpha[j])
    tau = O.expected_tau(alpha)
    se = n_out.std() / math.sqrt(n_out.size)
    assert abs(n_out.mean() - tau) < 4 * se


def _chi2_pvalue(tokens, prob, min_expected=5.0):
    counts = np.bincount(tokens, minlength=prob.size).astype(np.float64)
    exp = prob * counts.sum()
    order = np.argsort(exp)
    # merge the smallest bins until each merged bin expects >= min_expected
    obs_m, exp_m, co, ce = [], [], 0.0, 0.0
    for i in order:
        co += counts[i]
        ce += exp[i]
        if ce >= min_expected:
            obs_m.append(co)
            exp_m.append(ce)
            co = ce = 0.0
    if ce > 0:
        obs_m[-1] += co
        exp_m[-1] += ce
    return stats.chisquare(obs_m, exp_m).pvalue


def test_emitted_tokens_follow_target_distribution(tiny_model, tiny_trials):
    p_logits, q_logits = tiny_model
    k = q_logits.shape[0]
    p = O.softmax64(p_logits)
    q = O.softmax64(q_logits)
    _, outs = tiny_trials
    for j in range(k + 1):
        toks = np.array([o[0][j] for o in outs if o[1] > j])
        if toks.size < 2000:
            continue
        assert _chi2_pvalue(toks, p[j]) > 1e-3, j
    # negative control: first emitted token drawn straight from the draft distribution
    toks = np.array([O.draft_sample(q_logits[0], u)[0]
                     for u in O.uniform(3, np.arange(60000), 9, O.STREAM_DRAFT)])
    assert _chi2_pvalue(toks, p[0]) < 1e-6
    assert _chi2_pvalue(toks, q[0]) > 1e-3


def test_draft_tokens_follow_draft_distribution(tiny_model, tiny_trials):
    _, q_logits = tiny_model
    drafts, _ = tiny_trials
    q = O.softmax64(q_logits)
    for j in range(q.shape[0]):
        assert _chi2_pvalue(drafts[:, j], q[j]) > 1e-3
