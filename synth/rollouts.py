"""Seeded synthetic rollout populations for the KV-aware admission scheduler.

One rollout replica's share of an RL step: requests with a prompt length, a response
length (the tokens the request will generate) and, per round the request is active, the
tokens one draft-and-verify round emits for it. The pages ran Qwen3 RL rollouts on
DAPO-MATH prompts (responses up to 24K tokens for the 8B model, k = 6, about 5.5 tokens
per round); those are not available, so seeded draws with those shapes stand in:

  prompts     uniform in [200, 600] tokens
  responses   log-normal, median 6000 tokens, sigma 0.8, clipped to [256, 24576]
  per round   1 + the number of leading accepted drafts out of k = 6, each accepted with
              probability 0.9 (mean about 5.3 tokens)

Nothing here schedules, pages or counts; the draws are passed to the scheduler as inputs.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class RolloutSpec:
    num_requests: int = 512
    prompt_lo: int = 200
    prompt_hi: int = 600
    resp_median: float = 6000.0
    resp_sigma: float = 0.8
    resp_lo: int = 256
    resp_hi: int = 24576
    k: int = 6
    accept: float = 0.9
    seed: int = 2024


def make_rollouts(spec: RolloutSpec, seed: int | None = None):
    """(prompt_len int32 [N], resp_len int32 [N], tau uint8 [N][max_rounds])."""
    rng = np.random.default_rng(spec.seed if seed is None else seed)
    n = spec.num_requests
    prompt = rng.integers(spec.prompt_lo, spec.prompt_hi + 1, size=n).astype(np.int32)
    resp = np.exp(rng.normal(np.log(spec.resp_median), spec.resp_sigma, size=n))
    resp = np.clip(np.rint(resp), spec.resp_lo, spec.resp_hi).astype(np.int32)
    rounds = int(resp.max())                      # a request is active at most resp rounds
    tau = np.zeros((n, rounds), dtype=np.uint8)
    for r in range(n):
        # leading accepts before the first rejection: geometric, capped at k
        lead = np.minimum(rng.geometric(1.0 - spec.accept, size=int(resp[r])) - 1, spec.k)
        tau[r, : resp[r]] = 1 + lead
    return prompt, resp, tau
