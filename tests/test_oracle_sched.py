"""Pins for the oracle of the KV-aware admission scheduler: iteration-by-iteration traces
worked by hand on tiny populations (admission order, eviction of the last admitted, FIFO
restore, the fit rule, AIMD halving and additive increase, recompute accounting, stall
detection), and invariants of a full-size run."""
import numpy as np
import pytest

import synth
from oracle import kv_sched_oracle as K


def tau_const(n, v, rounds=64):
    return np.full((n, rounds), v, dtype=np.uint8)


def test_flow_without_pressure():
    # 3 requests: 1-page prompts, 32 tokens each, 16 per round; capacity 4 pages; AIMD from 1
    tot, tr = K.simulate([16] * 3, [32] * 3, tau_const(3, 16), capacity=4, cap0=1)
    assert tr == [
        (1, 1, 0, 1, 0, 0, 1, 0),    # admit r0
        (2, 2, 0, 3, 0, 0, 1, 16),   # r0 -> 2 pages; cap binds, U 2 < 3.4: cap 2; admit r1
        (2, 2, 0, 3, 0, 0, 1, 32),   # r0 done, r1 -> 2 pages; admit r2
        (2, 1, 0, 2, 0, 0, 0, 32),   # r1 done, r2 -> 2 pages
        (2, 0, 0, 0, 0, 0, 0, 16),   # r2 done
    ]
    assert tot["tokens"] == 96 and tot["done"] == 3 and tot["iterations"] == 5
    assert tot["transferred"] == 0 and tot["prefilled"] == 3 and tot["stalled"] == 0


def test_offload_restore_order_and_stall():
    # 2 requests: 1-page prompts, 64 tokens, 16 per round; capacity 3; fixed cap 2
    tot, tr = K.simulate([16, 16], [64, 64], tau_const(2, 16), capacity=3, policy="fixed", cap0=2)
    assert tr == [
        (2, 2, 0, 2, 0, 0, 2, 0),    # admit r0, r1
        (2, 1, 1, 2, 2, 0, 0, 32),   # both 2 pages: U 4 > 3, evict r1 (last admitted, 2 pages out)
        (2, 1, 1, 3, 0, 0, 0, 16),   # r0 3 pages; r1 (2) does not fit
        (2, 1, 1, 2, 6, 0, 0, 16),   # r0 4 pages > 3: evicted (4 out), r1 restored (2 in)
        (2, 1, 1, 3, 0, 0, 0, 16),   # r1 3 pages; r0 (4) cannot fit
        (2, 0, 2, 0, 4, 0, 0, 16),   # r1 4 pages: evicted (4 out); nothing fits any more
        (2, 0, 2, 0, 0, 0, 0, 0),    # no progress possible: stalled
    ]
    assert tot["stalled"] == 1 and tot["done"] == 0 and tot["transferred"] == 12


def test_recompute_counts_restores_not_transfers():
    tot, tr = K.simulate([16, 16], [64, 64], tau_const(2, 16), capacity=3, policy="fixed", cap0=2,
                         evict="recompute")
    assert [x[4] for x in tr] == [0] * 7
    assert [x[5] for x in tr] == [0, 0, 0, 2, 0, 0, 0]   # r1's 2 pages recomputed on restore
    assert tot["recomputed"] == 2 and tot["transferred"] == 0


def test_aimd_halves_on_eviction_and_backlog():
    # 4 requests of 1-page prompts, 48 tokens, 16 per round, capacity 6 (high mark 5.82,
    # low mark 5.1, backlog mark 3), AIMD from cap 4
    tot, tr = K.simulate([16] * 4, [48] * 4, tau_const(4, 16), capacity=6, cap0=4, b_high=0.5)
    assert tr == [
        (4, 4, 0, 4, 0, 0, 4, 0),    # cap does not bind yet (0 active): admit 4
        (2, 3, 1, 6, 2, 0, 0, 64),   # 2 pages each, U 8 > 6: evict r3 (U 6 fits); cap 4 -> 2
        (1, 2, 2, 6, 3, 0, 0, 48),   # 3 pages each, U 9: evict r2 (U 6); cap 2 -> 1
        (1, 1, 1, 2, 2, 0, 0, 32),   # r0, r1 done; backlog 2 + 3 > 3: cap stays 1; restore r3
        (2, 2, 0, 6, 3, 0, 0, 16),   # r3 3 pages; backlog 3 not > 3, cap binds, U 3 < 5.1: cap 2; restore r2
        (2, 0, 0, 0, 0, 0, 0, 32),   # r3, r2 done
    ]
    assert tot["done"] == 4 and tot["tokens"] == 4 * 48 and tot["transferred"] == 10


@pytest.mark.parametrize("policy,cap0", [("aimd", 16), ("fixed", 256)])
def test_full_size_invariants(policy, cap0):
    spec = synth.RolloutSpec(num_requests=128, seed=7)
    p, r, tau = synth.make_rollouts(spec)
    cap = 12000
    pressure = np.zeros(3000, dtype=np.int32)
    pressure[1000:1400] = cap // 3
    tot, tr = K.simulate(p, r, tau, capacity=cap, policy=policy, cap0=cap0, pressure=pressure)
    assert tot["done"] == 128 and tot["stalled"] == 0
    assert tot["tokens"] == int(np.sum(r))
    assert tot["prefilled"] == int(np.sum(-(-p // 16)))
    for t, row in enumerate(tr):
        c_t = cap - (int(pressure[t]) if t < len(pressure) else 0)
        assert row[3] <= c_t                      # resident pages never exceed this iteration's capacity
        if policy == "fixed":
            assert row[0] == cap0 and row[1] <= cap0
    if policy == "aimd":
        caps = [row[0] for row in tr]
        for a, b in zip(caps, caps[1:]):
            assert b <= a + 1                        # additive increase: +1 at most
            assert b >= a or b == max(1, a // 2)     # a decrease is a halving


@pytest.mark.parametrize("seed", range(6))
def test_offload_moves_twice_what_recompute_recomputes(seed):
    """The evict mode only changes the counters, never a decision: on the same population
    the traces agree in cap, active, paused and resident pages, and every evicted request's
    pages go out and come back once (offload) or are recomputed once (recompute)."""
    spec = synth.RolloutSpec(num_requests=96, seed=100 + seed)
    p, r, tau = synth.make_rollouts(spec)
    pressure = np.zeros(1500, dtype=np.int32)
    pressure[500:900] = 2500
    kw = dict(capacity=9000, pressure=pressure, policy=["aimd", "fixed"][seed % 2], cap0=[16, 128][seed % 2])
    off, t_off = K.simulate(p, r, tau, evict="offload", **kw)
    rec, t_rec = K.simulate(p, r, tau, evict="recompute", **kw)
    assert [x[:4] for x in t_off] == [x[:4] for x in t_rec]
    assert off["done"] == rec["done"] == 96 and off["evictions"] == rec["evictions"] > 0
    assert off["transferred"] == 2 * rec["recomputed"] and rec["transferred"] == 0
