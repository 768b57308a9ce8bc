"""The library's adaptive draft length (a host function of the C ABI) against the oracle:
the same k on random counts and costs (both sides decide in double, in the same order),
and argument validation."""
import numpy as np
import pytest

import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O


@pytest.mark.parametrize("seed", range(300))
def test_choose_horizon_matches_oracle(seed):
    rng = np.random.default_rng(seed)
    k_max = int(rng.integers(1, 9))
    dec = rng.integers(0, 200, size=k_max).astype(float)
    if seed % 3 == 0:
        dec = dec * rng.random(k_max)              # decayed (non-integer) counts
    acc = np.floor(dec * rng.random(k_max) ** (0.3 if seed % 2 else 3.0))
    c_d, c_v = float(rng.uniform(1, 100)), float(rng.uniform(1, 2000))
    pa, pw = float(rng.uniform(0, 1)), float(rng.choice([0.5, 4.0, 16.0]))
    want = O.choose_horizon(acc.tolist(), dec.tolist(), c_d, c_v, k_max, pa, pw)
    assert s3r.s3r_choose_horizon(acc.tolist(), dec.tolist(), c_d, c_v, pa, pw) == want


def test_choose_horizon_hand_worked_case():
    alpha = [0.66, 0.67, 0.64, 0.78, 1.0, 0.57]
    assert s3r.s3r_choose_horizon([a * 1e6 for a in alpha], [1e6] * 6, 57.0, 730.0, 0.5, 0.0) == 5


@pytest.mark.parametrize("args", [
    ([1.0] * 9, [1.0] * 9, 1.0, 1.0, 0.5, 1.0),      # k_max > 8
    ([1.0], [1.0], 0.0, 1.0, 0.5, 1.0),              # c_draft <= 0
    ([1.0], [1.0], 1.0, float("inf"), 0.5, 1.0),     # c_verify not finite
    ([1.0], [1.0], 1.0, 1.0, 1.5, 1.0),              # prior outside [0, 1]
    ([1.0], [1.0], 1.0, 1.0, 0.5, -1.0),             # negative prior weight
    ([-1.0], [1.0], 1.0, 1.0, 0.5, 1.0),             # negative count
    ([0.0], [0.0], 1.0, 1.0, 0.5, 0.0),              # a position with no evidence and no prior
])
def test_choose_horizon_rejects_bad_arguments(args):
    with pytest.raises(s3r.S3RError):
        s3r.s3r_choose_horizon(*args)


class _FakeBuf:
    def __init__(self, k_max):
        import torch
        self.k_max = k_max
        self.stats = torch.zeros(2 + 2 * s3r.MAX_K, dtype=torch.int64)


class _FakeEngine:
    """The controller's view of an engine: the commit counters, k_max and set_k."""

    def __init__(self, k_max):
        self.buf = _FakeBuf(k_max)
        self.k = k_max

    def set_k(self, k):
        self.k = k

    def commit(self, accepted, decided):
        for j, (a, d) in enumerate(zip(accepted, decided)):
            self.buf.stats[2 + j] += a
            self.buf.stats[2 + s3r.MAX_K + j] += d


@pytest.mark.parametrize("seed", range(200))
def test_horizon_step_matches_oracle(seed):
    """The library's decay, pooled prior and choice against the oracle's, in double, on
    random counters, decays, costs and priors."""
    rng = np.random.default_rng(1000 + seed)
    M = s3r.MAX_K
    k_max = int(rng.integers(1, M + 1))
    acc0 = np.floor(rng.random(M) * 50) * (seed % 2) + 0.0
    dec0 = acc0 + np.floor(rng.random(M) * 30) + 0.0
    last = np.zeros(2 + 2 * M, dtype=np.int64)
    last[2: 2 + M] = rng.integers(0, 100, M)
    last[2 + M:] = last[2: 2 + M] + rng.integers(0, 50, M)
    now = last.copy()
    new_a = rng.integers(0, 60, M)
    now[2: 2 + M] += new_a
    now[2 + M:] += new_a + rng.integers(0, 40, M)
    decay = float(rng.choice([0.0, 0.5, 0.8, 1.0]))
    c_d, c_v = float(rng.uniform(1, 100)), float(rng.uniform(1, 2000))
    pa = None if seed % 3 else float(rng.uniform(0, 1))
    oa, od, oprior, ok = O.horizon_step(acc0.tolist(), dec0.tolist(), (now - last)[2: 2 + M].tolist(),
                                        (now - last)[2 + M:].tolist(), decay, c_d, c_v, k_max, pa, 4.0)
    acc, dec, lst = acc0.copy(), dec0.copy(), last.copy()
    k, prior = s3r.s3r_horizon_step(now, lst, acc, dec, k_max, decay, c_d, c_v, -1.0 if pa is None else pa, 4.0)
    assert (k, prior) == (ok, oprior)
    assert acc.tolist() == oa and dec.tolist() == od and lst.tolist() == now.tolist()


def test_horizon_step_rejects_bad_arguments_and_leaves_state():
    M = s3r.MAX_K
    now = np.zeros(2 + 2 * M, dtype=np.int64)
    last = now.copy()
    last[2] = 5                                   # a counter that went down
    acc, dec = np.ones(M), np.ones(M)
    with pytest.raises(s3r.S3RError):
        s3r.s3r_horizon_step(now, last, acc, dec, 4, 0.5, 1.0, 1.0)
    assert last[2] == 5 and acc.tolist() == [1.0] * M
    with pytest.raises(s3r.S3RError):
        s3r.s3r_horizon_step(now, now.copy(), acc, dec, 4, 1.5, 1.0, 1.0)   # decay > 1


def test_controller_decays_counts_and_pools_the_prior():
    eng = _FakeEngine(6)
    ctl = s3r.AdaptiveHorizon(eng, c_draft=57.0, c_verify=730.0, decay=0.5, prior_weight=4.0)
    eng.commit([80, 60, 40, 0, 0, 0], [100, 80, 60, 0, 0, 0])
    k1 = ctl.step()
    assert ctl.acc[:3].tolist() == [80.0, 60.0, 40.0] and ctl.dec[:3].tolist() == [100.0, 80.0, 60.0]
    pooled = 180.0 / 240.0
    assert ctl.last_prior == pooled
    want = O.choose_horizon(ctl.acc[:6].tolist(), ctl.dec[:6].tolist(), 57.0, 730.0, 6, pooled, 4.0)
    assert k1 == want == eng.k
    # a second window halves the first and adds the new counts
    eng.commit([10, 0, 0, 0, 0, 0], [20, 0, 0, 0, 0, 0])
    ctl.step()
    assert ctl.acc[0] == 0.5 * 80 + 10 and ctl.dec[0] == 0.5 * 100 + 20 and ctl.dec[1] == 40.0
    assert ctl.history == [k1, eng.k]


def test_controller_fixed_prior():
    eng = _FakeEngine(4)
    ctl = s3r.AdaptiveHorizon(eng, c_draft=1.0, c_verify=1000.0, prior_alpha=0.0, prior_weight=4.0)
    eng.commit([50, 0, 0, 0], [50, 0, 0, 0])
    # position 1 always accepted, later positions never drafted and a prior of 0: k = 1
    assert ctl.step() == 1


def test_round_buffers_views_share_their_storage_across_lengths():
    """set_k lays the length-dependent buffers out for k in the same storage: every view
    starts at the same address whatever k (graphs captured per length keep valid
    pointers) and has the contiguous layout the library's calls use for that k."""
    from sparse_dense_kv_b200.engine import RoundBuffers
    NR, Hq, Hkv, d, cap = 3, 8, 2, 16, 64
    b = RoundBuffers(NR, Hq, Hkv, d, cap, 6, 64, 32, device="cpu")
    ptrs = {name: getattr(b, name).data_ptr() for name in
            ("scores", "lse", "verify_out", "draft_tokens", "out_tokens")}
    for k in (1, 3, 6):
        b.set_k(k)
        G, T = Hq // Hkv, k + 1
        assert b.scores.shape == (NR, Hkv, G * T, cap) and b.scores.is_contiguous()
        assert b.lse.shape == (NR, T, Hq) and b.verify_out.shape == (NR, T, Hq, d)
        assert b.draft_tokens.shape == (NR, k) and b.out_tokens.shape == (NR, T)
        for name, p in ptrs.items():
            assert getattr(b, name).data_ptr() == p, (name, k)
    assert b.stats.numel() == 2 + 2 * s3r.MAX_K and len(b.steps) == 6


@pytest.mark.parametrize("seed", range(200))
def test_choose_horizon_costs_matches_oracle(seed):
    """The cost-table choice against the oracle on random counts and per-length costs."""
    rng = np.random.default_rng(1000 + seed)
    k_max = int(rng.integers(1, 9))
    dec = rng.integers(0, 200, size=k_max).astype(float)
    if seed % 3 == 0:
        dec = dec * rng.random(k_max)
    acc = np.floor(dec * rng.random(k_max) ** (0.3 if seed % 2 else 3.0))
    cost = np.cumsum(rng.uniform(0.01, 0.2, size=k_max)) + rng.uniform(0.2, 1.0)
    if seed % 4 == 0:
        cost = rng.uniform(0.1, 2.0, size=k_max)               # not monotone at all
    pa, pw = float(rng.uniform(0, 1)), float(rng.choice([0.5, 4.0, 16.0]))
    want = O.choose_horizon_costs(acc.tolist(), dec.tolist(), cost.tolist(), k_max, pa, pw)
    assert s3r.s3r_choose_horizon_costs(acc.tolist(), dec.tolist(), cost.tolist(), pa, pw) == want


def test_choose_horizon_costs_hand_worked_cases():
    """Worked by hand: with acceptance 0.8 at every position the expected tokens for k = 1..6
    are 1.8, 2.44, 2.952, 3.3616, 3.68928, 3.951424; against round costs 0.52, 0.58, 0.64,
    0.71, 0.78, 0.80 the rates are 3.46, 4.21, 4.61, 4.735, 4.730, 4.939, so k = 6 (a line
    through the same costs, 0.058 k + 0.468, would rate k = 6 at 3.951/0.816 = 4.84 and k = 5
    at 3.689/0.758 = 4.87 and pick k = 5). With every draft accepted the tokens are k + 1,
    and costs 2, 3, 4, 10 give the rate 1 for k = 1, 2, 3: the smallest k wins the tie."""
    acc, dec = [0.8e6] * 6, [1e6] * 6
    cost = [0.52, 0.58, 0.64, 0.71, 0.78, 0.80]
    assert s3r.s3r_choose_horizon_costs(acc, dec, cost, 0.5, 0.0) == 6
    assert O.choose_horizon_costs(acc, dec, cost, 6, 0.5, 0.0) == 6
    assert s3r.s3r_choose_horizon(acc, dec, 0.058, 0.468, 0.5, 0.0) == 5
    assert s3r.s3r_choose_horizon_costs([5.0] * 4, [5.0] * 4, [2.0, 3.0, 4.0, 10.0], 0.5, 0.0) == 1
    # the line itself as a table gives the line's choice
    line = [0.058 * k + 0.468 for k in range(1, 7)]
    assert s3r.s3r_choose_horizon_costs(acc, dec, line, 0.5, 0.0) == 5


@pytest.mark.parametrize("seed", range(50))
def test_horizon_step_costs_matches_oracle(seed):
    rng = np.random.default_rng(2000 + seed)
    k_max = int(rng.integers(1, 9))
    decay = float(rng.choice([0.0, 0.5, 0.8, 1.0]))
    cost = (np.cumsum(rng.uniform(0.01, 0.2, size=k_max)) + 0.4).tolist()
    last = np.zeros(2 + 2 * s3r.MAX_K, dtype=np.int64)
    acc = np.zeros(s3r.MAX_K, dtype=np.float64)
    dec = np.zeros(s3r.MAX_K, dtype=np.float64)
    oacc, odec = [0.0] * s3r.MAX_K, [0.0] * s3r.MAX_K
    now = last.copy()
    for _ in range(4):
        d_new = rng.integers(0, 50, size=s3r.MAX_K)
        a_new = (d_new * rng.random(s3r.MAX_K)).astype(np.int64)
        now = now.copy()
        now[2:2 + s3r.MAX_K] += a_new
        now[2 + s3r.MAX_K:] += d_new
        k, prior = s3r.s3r_horizon_step_costs(now, last, acc, dec, k_max, decay, cost)
        oacc, odec, oprior, ok = O.horizon_step_costs(oacc, odec, a_new.tolist(), d_new.tolist(), decay, cost,
                                                      k_max)
        assert k == ok and prior == oprior
        assert acc.tolist() == oacc and dec.tolist() == odec
        assert (last == now).all()


@pytest.mark.parametrize("cost", [[1.0, 0.0], [1.0, -2.0], [1.0, float("inf")], [float("nan"), 1.0]])
def test_choose_horizon_costs_rejects_bad_costs(cost):
    with pytest.raises(s3r.S3RError):
        s3r.s3r_choose_horizon_costs([1.0, 1.0], [2.0, 2.0], cost, 0.5, 1.0)
