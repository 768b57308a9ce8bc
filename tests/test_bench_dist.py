"""The benchmark's cross-rank reduction (max device time, summed tokens) with two gloo ranks
on the CPU: the multi-GPU bench shards requests by rank with no collective on the data
path, so this reduction and the barriers are its only cross-rank steps."""
import os
import socket

import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import torch.distributed as dist
    from datetime import timedelta
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    import bench
    assert bench.dist_env() == (rank, world, rank)
    ms, tokens = bench.reduce_results(10.0 + 5.0 * rank, 100 * (rank + 1))
    dist.barrier()
    dist.destroy_process_group()
    out.put((rank, ms, tokens))


def test_reduce_results_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, tokens in res:
        assert ms == 15.0          # max over ranks
        assert tokens == 300       # summed over ranks


def test_reduce_results_single_process_is_identity():
    import bench
    assert bench.reduce_results(3.5, 7) == (3.5, 7)


def test_ranks_build_same_shaped_disjoint_work():
    """Each rank builds its own copy of the workload from rank-dependent seeds: same
    lengths and shapes (weak scaling), different data, nothing shared between ranks."""
    import torch
    import bench
    import synth
    spec = synth.WORKLOADS["tiny"]
    l0, c0, s0, i0 = bench.build_workload(spec, 0, "cpu")
    l1, c1, s1, i1 = bench.build_workload(spec, 1, "cpu")
    assert (l0 == l1).all() and torch.equal(s0, s1)
    assert c0.k_pool.shape == c1.k_pool.shape
    assert not torch.equal(c0.k_pool, c1.k_pool)
    for name in i0:
        assert i0[name].shape == i1[name].shape
        assert not torch.equal(i0[name], i1[name])
