"""The library's KV-aware admission scheduler (host C++ behind the C ABI) against the
oracle: identical iteration traces and totals (integers exact, the simulated time bit for
bit) on random populations with injected memory pressure, on the hand-worked cases and on
a full-size replica; argument checks; two replicas as gloo ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import synth
import sparse_dense_kv_b200 as s3r
from oracle import kv_sched_oracle as K


def both(p, r, tau, **kw):
    a, ta = s3r.s3r_sched_simulate(p, r, tau, **kw)
    b, tb = K.simulate(p, r, tau, **kw)
    return a, ta, b, np.array(tb, dtype=np.int32).reshape(-1, 8)


def same(a, b):
    for k in ("tokens", "transferred", "recomputed", "prefilled", "evictions", "iterations",
              "max_active", "done", "stalled"):
        assert a[k] == b[k], k
    assert a["time"] == b["time"]


@pytest.mark.parametrize("seed", range(60))
def test_random_populations_match_oracle(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 40))
    p = rng.integers(0, 200, size=n).astype(np.int32)
    r = rng.integers(0, 600, size=n).astype(np.int32)
    tau = rng.integers(1, 8, size=(n, 700)).astype(np.uint8)
    capacity = int(rng.integers(40, 400))
    pressure = rng.integers(0, capacity // 2, size=int(rng.integers(0, 300))).astype(np.int32)
    kw = dict(capacity=capacity, policy=["aimd", "fixed"][seed % 2], evict=["offload", "recompute"][(seed // 2) % 2],
              cap0=int(rng.integers(1, 20)), u_low=float(rng.uniform(0.5, 0.9)), u_high=float(rng.uniform(0.9, 1.0)),
              b_high=float(rng.uniform(0.1, 1.0)), costs=tuple(float(x) for x in rng.uniform(0, 2, size=6)),
              pressure=pressure if seed % 3 else None, max_iters=5000)
    kw["cap_max"] = max(kw["cap0"], 64)
    a, ta, b, tb = both(p, r, tau, **kw)
    same(a, b)
    assert np.array_equal(ta, tb)


@pytest.mark.parametrize("policy,evict,cap0", [("aimd", "offload", 16), ("fixed", "offload", 256),
                                               ("fixed", "recompute", 256), ("aimd", "recompute", 16)])
def test_full_size_replica_matches_oracle(policy, evict, cap0):
    p, r, tau = synth.make_rollouts(synth.RolloutSpec(num_requests=256, seed=11))
    pressure = np.zeros(2500, dtype=np.int32)
    pressure[1500:2500] = 6000          # a memory-pressure event: a quarter of the pages taken
    a, ta, b, tb = both(p, r, tau, capacity=24000, policy=policy, evict=evict, cap0=cap0, pressure=pressure)
    same(a, b)
    assert np.array_equal(ta, tb)
    assert a["done"] == 256 and a["stalled"] == 0


def test_hand_worked_stall_case_through_the_library():
    tau = np.full((2, 64), 16, dtype=np.uint8)
    tot, tr = s3r.s3r_sched_simulate([16, 16], [64, 64], tau, capacity=3, policy="fixed", cap0=2)
    assert tot["stalled"] == 1 and tot["transferred"] == 12 and tr.shape == (7, 8)
    assert tr[3].tolist() == [2, 1, 1, 2, 6, 0, 0, 16]


@pytest.mark.parametrize("bad", [dict(capacity=0), dict(cap0=0), dict(cap_min=5, cap0=4),
                                 dict(cap_max=2, cap0=4), dict(u_low=float("nan")),
                                 dict(costs=(1.0, -1.0, 0, 0, 0, 0)), dict(pressure=[50]),
                                 dict(pressure=[-1])])
def test_rejects_bad_arguments(bad):
    kw = dict(capacity=50, cap0=4)
    kw.update(bad)
    with pytest.raises(s3r.S3RError):
        s3r.s3r_sched_simulate([16], [32], np.ones((1, 64), np.uint8), **kw)


def test_running_out_of_draws_is_an_error():
    with pytest.raises(s3r.S3RError):
        s3r.s3r_sched_simulate([16], [100], np.ones((1, 10), np.uint8), capacity=50, cap0=4)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _replica_worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    from sparse_dense_kv_b200.replicas import simulate_replicas
    p, r, tau = synth.make_rollouts(synth.RolloutSpec(num_requests=64, seed=5))
    tot = simulate_replicas(p, r, tau, capacity=9000, cap0=8)
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, tot))


def test_two_replicas_as_gloo_ranks():
    """Each rank runs the requests r % 2 == rank; the all-reduced totals equal the sum (max
    for time) of the two shards run one after another in this process."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_replica_worker, args=(k, 2, port, q)) for k in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
        assert pr.exitcode == 0
    assert res[0] == res[1]
    p, r, tau = synth.make_rollouts(synth.RolloutSpec(num_requests=64, seed=5))
    shards = [s3r.s3r_sched_simulate(p[k::2], r[k::2], tau[k::2], capacity=9000, cap0=8, trace=False)[0]
              for k in range(2)]
    for key in ("tokens", "transferred", "prefilled", "evictions", "done"):
        assert res[0][key] == shards[0][key] + shards[1][key]
    assert res[0]["time"] == max(shards[0]["time"], shards[1]["time"])
    assert res[0]["tokens"] == int(r.sum())


def _dying_replica_worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=10))
    if rank == 1:
        out.put((rank, "left"))
        out.close()
        out.join_thread()              # the message is out before the process goes
        os._exit(3)                    # the replica dies before the collective, no cleanup
    from sparse_dense_kv_b200.replicas import simulate_replicas
    p, r, tau = synth.make_rollouts(synth.RolloutSpec(num_requests=16, seed=5))
    try:
        simulate_replicas(p, r, tau, capacity=4000, cap0=8)
        out.put((rank, "no error"))
    except Exception as exc:           # the collective fails instead of waiting for good
        out.put((rank, f"error: {type(exc).__name__}"))


def test_a_dead_replica_fails_the_others_fast():
    """A replica that dies before the totals' all-reduce: the survivor's collective ends
    with an error (peer gone, or the process group's 10 s timeout) rather than a hang."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_dying_replica_worker, args=(k, 2, port, q)) for k in range(2)]
    for pr in procs:
        pr.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for pr in procs:
        pr.join(timeout=60)
    assert res[1] == "left"
    assert res[0].startswith("error"), res[0]
