"""Round-level checks of the oracle on the tiny workload, and pins of the round
accounting formulas against the numbers the pages print."""
import time

import numpy as np
import pytest

import synth
from oracle import s3r_oracle as O
from tests.conftest import read_golden


def make_states(spec, extra=800):
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=extra)
    kp = cache.k_pool.float().numpy()
    vp = cache.v_pool.float().numpy()
    pt = cache.page_table.numpy()
    states = []
    for r in range(spec.num_requests):
        cap = int((pt[r] >= 0).sum()) * 16
        K = np.stack([O.gather_positions(kp, pt[r], h, np.arange(cap)) for h in range(spec.num_kv_heads)])
        V = np.stack([O.gather_positions(vp, pt[r], h, np.arange(cap)) for h in range(spec.num_kv_heads)])
        st = O.RequestState(K, V, int(lens[r]))
        q, k, v = synth.token_qkv(spec, r, [st.L])
        O.prefill_scores(st, q[0].float().numpy(), k[0].float().numpy(), v[0].float().numpy())
        states.append(st)
    return states


def run_rounds(spec, n_rounds):
    states = make_states(spec)
    log = []
    for _ in range(n_rounds):
        for r, st in enumerate(states):
            L = st.L
            q, k, v = synth.token_qkv(spec, r, range(L, L + spec.k + 1))
            p_log, q_log = synth.token_logits(spec, r, range(L + 1, L + spec.k + 2))
            res = O.run_round(st, r, spec.sample_seed, spec.k, spec.budget_bp, spec.window,
                              q.float().numpy(), k.float().numpy(), v.float().numpy(),
                              q_log[: spec.k], p_log)
            log.append((r, L, res["tokens"].tolist(), [s.tolist() for s in res["sel"]]))
    return states, log


def test_hundred_rounds_tiny_is_fast_and_deterministic():
    spec = synth.WORKLOADS["tiny"]
    t0 = time.time()
    states, log = run_rounds(spec, 100)
    assert time.time() - t0 < 120
    _, log2 = run_rounds(spec, 100)
    assert log == log2
    taus = np.array([len(t) for _, _, t, _ in log])
    assert taus.min() >= 1 and taus.max() <= spec.k + 1
    # lengths advance by exactly the emitted tokens
    for r, st in enumerate(states):
        emitted = sum(len(t) for rr, _, t, _ in log if rr == r)
        assert st.L == synth.make_lengths(spec)[r] + emitted
    # selected sets have the budgeted size and contain the window
    for r, L, _, sels in log:
        n, w = O.budget_count(L, spec.budget_bp, spec.window)
        for s in sels:
            assert len(s) == n and s[-w:] == list(range(L - w, L))


def test_break_even_acceptance_reproduces_table7():
    for B, S, ar, draft, verify, total, printed in read_golden("table7_break_even.txt"):
        ar, draft, verify, total = map(float, (ar, draft, verify, total))
        assert abs(draft + verify - total) < 0.006
        a = O.break_even_acceptance(total, ar, 6)
        if printed == "NA":
            assert a > 1.0
        else:
            assert abs(100 * a - float(printed)) < 0.05, (B, S, a)


def test_round_cost_example_of_the_explainer():
    for k, step, verify, cost, tokens, speedup in read_golden("explainer_round_cost.txt"):
        k, step, verify, cost, tokens, speedup = int(k), *map(float, (step, verify, cost, tokens, speedup))
        round_cost = k * step + verify
        assert abs(round_cost - cost) < 1e-12
        assert abs(tokens / round_cost - speedup) < 0.005


def test_expected_tau_closed_form():
    assert O.expected_tau([]) == 1.0
    assert O.expected_tau([1.0] * 6) == 7.0
    assert O.expected_tau([0.0, 1.0]) == 1.0
    a = 0.8
    assert abs(O.expected_tau([a] * 6) - (1 - a ** 7) / (1 - a)) < 1e-12


def test_float32_timing_variant_follows_the_float64_round():
    """The float32 variant timed by the benchmark's CPU baseline computes the same round: on
    the tiny workload its attention outputs agree with the float64 oracle to float32
    rounding, and the emitted tokens agree wherever no sampling decision of the float64 round
    lies within float32 reach of its boundary."""
    spec = synth.WORKLOADS["tiny"]
    states = make_states(spec)
    for r, st in enumerate(states):
        st32 = O.RequestState(st.K, st.V, st.L, st.sigma, dtype=np.float32)
        assert st32.K.dtype == np.float32
        L = st.L
        q, k, v = synth.token_qkv(spec, r, range(L, L + spec.k + 1))
        p_log, q_log = synth.token_logits(spec, r, range(L + 1, L + spec.k + 2))
        args = (r, spec.sample_seed, spec.k, spec.budget_bp, spec.window,
                q.float().numpy(), k.float().numpy(), v.float().numpy(), q_log[: spec.k], p_log)
        a = O.run_round(st, *args)
        b = O.run_round(st32, *args)
        assert [s.tolist() for s in a["sel"]] == [s.tolist() for s in b["sel"]]
        np.testing.assert_allclose(b["draft_out"], a["draft_out"], rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(b["verify_out"], a["verify_out"], rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(b["sigma"], a["sigma"], rtol=1e-4, atol=1e-6)
        if min(np.min(a["draft_margin"]), np.min(a["margins"])) > 1e-5:
            assert a["tokens"].tolist() == b["tokens"].tolist()
