"""Rollout replicas under the KV-aware admission scheduler, one per process.

Each rank of a torch.distributed group (gloo is enough: the scheduler runs on the host)
is one rollout replica and takes the requests r with r % world == rank, as the pages run
four independent replicas per node; the library's s3r_sched_simulate runs the replica,
and one all-reduce gathers the totals: counts summed, simulated time and iterations the
maximum over replicas (the step ends when its slowest replica does).
"""
from __future__ import annotations

import numpy as np
import torch

from . import _lib as L

SUMMED = ("tokens", "transferred", "recomputed", "prefilled", "evictions", "done", "stalled")
MAXED = ("time", "iterations", "max_active")


def simulate_replicas(prompt_len, resp_len, tau, group=None, **cfg):
    """Totals of all replicas (every rank gets the same dict); without an initialised
    process group this is the single replica's run."""
    import torch.distributed as dist
    ranked = dist.is_available() and dist.is_initialized()
    rank = dist.get_rank(group) if ranked else 0
    world = dist.get_world_size(group) if ranked else 1
    ids = np.arange(rank, len(prompt_len), world)
    tot, _ = L.s3r_sched_simulate(np.asarray(prompt_len)[ids], np.asarray(resp_len)[ids],
                                  np.asarray(tau)[ids], trace=False, **cfg)
    if world == 1:
        return tot
    s = torch.tensor([float(tot[k]) for k in SUMMED], dtype=torch.float64)
    m = torch.tensor([float(tot[k]) for k in MAXED], dtype=torch.float64)
    dist.all_reduce(s, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(m, op=dist.ReduceOp.MAX, group=group)
    out = {k: int(v) for k, v in zip(SUMMED, s.tolist())}
    out.update({k: (v if k == "time" else int(v)) for k, v in zip(MAXED, m.tolist())})
    return out
