"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the CPU oracle.

This package holds no arithmetic of the method itself (no attention, no selection, no
sampling, no Philox): it only draws the synthetic KV cache, the per-token q/k/v and the
synthetic logits from seeded generators, with the shapes of the Qwen3-shaped workloads.
"""
from .workload import (  # noqa: F401
    WORKLOADS,
    WorkloadSpec,
    KVCache,
    make_lengths,
    build_cache,
    token_qkv,
    token_logits,
    bf16_round,
    initial_phases,
    projection_matrix,
    randn_bf16,
    randn_f32,
)
from .rollouts import RolloutSpec, make_rollouts  # noqa: F401,E402
