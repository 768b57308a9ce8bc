"""Seeded synthetic workloads with the shapes of the S3R per-round hot path.

Five workloads, each a single attention layer over a paged bf16 KV cache with 16-token
pages (Qwen3-shaped head counts; the pages' own runs used Qwen3-1.7B / Qwen3-8B RL
rollouts on DAPO-MATH prompts, which are not available here, so random tensors with the
stated distributions stand in for them):

  tiny        2 requests, L in {256, 300}, 2 q-heads / 1 kv-head, d 64, k 6, s 0.25,
              window 16, vocab 64, target logits N(0, 2), draft = target + N(0, 0.3^2)
  qwen3-1.7b  64 requests, L ~ U[4096, 16384], 16/8 heads, d 128, k 6, s 0.05,
              window 64, 32 heavy-hitter keys (x4) per (request, kv-head), vocab 151936,
              draft noise N(0, 0.5^2)
  qwen3-8b    32 requests, L ~ U[8192, 24576], 32/8 heads, otherwise as qwen3-1.7b
  ragged      256 requests, L log-uniform in [1024, 16384], 16/8 heads, mixed round
              phases, shuffled page tables, otherwise as qwen3-1.7b
  sweep       32 requests at L = 24576, 32/8 heads, s in {.02,.05,.1,.2} x k in
              {2,4,6,8}, vocab 32768, logits from a seeded bf16 projection of the
              head-concatenated attention outputs

Nothing here computes attention, scores, selections, Philox draws or sampling decisions.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import numpy as np
import torch

PAGE_SIZE = 16


@dataclass(frozen=True)
class WorkloadSpec:
    name: str
    num_requests: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    lengths: tuple            # ("fixed", (L0, L1, ...)) | ("uniform", lo, hi) | ("loguniform", lo, hi)
    k: int
    budget_bp: int            # sparse budget s in units of 1e-4
    window: int
    vocab: int
    logit_std: float          # target logits N(0, logit_std^2)
    draft_noise_std: float    # draft logits = target + N(0, draft_noise_std^2)
    heavy_hitters: int = 0    # planted heavy-hitter keys per (request, kv-head)
    heavy_scale: float = 4.0
    shuffle_pages: bool = False
    mixed_phases: bool = False
    projection_logits: bool = False
    data_seed: int = 0
    sample_seed: int = 1000
    sweep_budgets_bp: tuple = field(default=())
    sweep_ks: tuple = field(default=())

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def with_(self, **kw) -> "WorkloadSpec":
        return replace(self, **kw)


_SPECS = [
    WorkloadSpec("tiny", 2, 2, 1, 64, ("fixed", (256, 300)), k=6, budget_bp=2500, window=16,
                 vocab=64, logit_std=math.sqrt(2.0), draft_noise_std=0.3,
                 data_seed=0, sample_seed=1000),
    WorkloadSpec("qwen3-1.7b", 64, 16, 8, 128, ("uniform", 4096, 16384), k=6, budget_bp=500,
                 window=64, vocab=151936, logit_std=math.sqrt(2.0), draft_noise_std=0.5,
                 heavy_hitters=32, data_seed=1, sample_seed=1001),
    WorkloadSpec("qwen3-8b", 32, 32, 8, 128, ("uniform", 8192, 24576), k=6, budget_bp=500,
                 window=64, vocab=151936, logit_std=math.sqrt(2.0), draft_noise_std=0.5,
                 heavy_hitters=32, data_seed=2, sample_seed=1002),
    WorkloadSpec("ragged", 256, 16, 8, 128, ("loguniform", 1024, 16384), k=6, budget_bp=500,
                 window=64, vocab=151936, logit_std=math.sqrt(2.0), draft_noise_std=0.5,
                 heavy_hitters=32, shuffle_pages=True, mixed_phases=True,
                 data_seed=3, sample_seed=1003),
    WorkloadSpec("sweep", 32, 32, 8, 128, ("fixed", (24576,) * 32), k=6, budget_bp=500,
                 window=64, vocab=32768, logit_std=math.sqrt(2.0), draft_noise_std=0.0,
                 heavy_hitters=32, projection_logits=True, data_seed=4, sample_seed=1004,
                 sweep_budgets_bp=(200, 500, 1000, 2000), sweep_ks=(2, 4, 6, 8)),
]
WORKLOADS = {spec.name: spec for spec in _SPECS}


def bf16_round(x) -> np.ndarray:
    """Round float values to bfloat16 (round to nearest even) and return them as float32."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float32).numpy()


def make_lengths(spec: WorkloadSpec, seed: int | None = None) -> np.ndarray:
    """Committed context length L per request (int32)."""
    kind = spec.lengths[0]
    rng = np.random.default_rng([spec.data_seed if seed is None else seed, 1])
    if kind == "fixed":
        out = np.asarray(spec.lengths[1], dtype=np.int64)
        assert out.size == spec.num_requests
    elif kind == "uniform":
        lo, hi = spec.lengths[1], spec.lengths[2]
        out = rng.integers(lo, hi + 1, size=spec.num_requests)
    elif kind == "loguniform":
        lo, hi = spec.lengths[1], spec.lengths[2]
        out = np.exp(rng.uniform(math.log(lo), math.log(hi), size=spec.num_requests))
        out = np.clip(np.round(out), lo, hi)
    else:
        raise ValueError(kind)
    return out.astype(np.int32)


def initial_phases(spec: WorkloadSpec, seed: int | None = None) -> np.ndarray:
    """Round phase per request for mixed-phase batches: 0..k-1 = next draft step, k = verify."""
    rng = np.random.default_rng([spec.data_seed if seed is None else seed, 2])
    return rng.integers(0, spec.k + 1, size=spec.num_requests).astype(np.int32)


@dataclass
class KVCache:
    k_pool: torch.Tensor          # bf16 [P][H_kv][16][d]
    v_pool: torch.Tensor          # bf16 [P][H_kv][16][d]
    page_table: torch.Tensor      # int32 [B][max_pages], -1 where unallocated
    lengths: np.ndarray           # int32 [B] committed lengths L
    heavy_positions: np.ndarray   # int32 [B][H_kv][heavy_hitters]
    max_pages: int
    num_pages: int

    @property
    def capacity(self) -> int:
        return self.max_pages * PAGE_SIZE


def _fill_normal_bf16(t: torch.Tensor, gen: torch.Generator, chunk: int = 1 << 26) -> None:
    flat = t.view(-1)
    for s in range(0, flat.numel(), chunk):
        e = min(flat.numel(), s + chunk)
        flat[s:e] = torch.randn(e - s, generator=gen, device=t.device,
                                dtype=torch.float32).to(torch.bfloat16)


def build_cache(spec: WorkloadSpec, lengths: np.ndarray, extra_tokens: int,
                device="cpu", seed: int | None = None) -> KVCache:
    """Paged KV cache: every allocated slot holds N(0,1) bf16 keys and values.

    Request r owns ceil((L_r + extra_tokens) / 16) pages. Pages are handed out in order,
    or in a seeded random permutation when spec.shuffle_pages is set, so that a
    request's pages are scattered over the pool. Heavy hitters: spec.heavy_hitters
    distinct positions per (request, kv-head), drawn uniformly from [0, L - window),
    get their key multiplied by spec.heavy_scale (exact in bf16 for powers of two).
    """
    seed = spec.data_seed if seed is None else seed
    B, H, d = spec.num_requests, spec.num_kv_heads, spec.head_dim
    lengths = np.asarray(lengths, dtype=np.int64)
    caps = (lengths + extra_tokens + PAGE_SIZE - 1) // PAGE_SIZE
    total = int(caps.sum())
    max_pages = int(caps.max())
    rng = np.random.default_rng([seed, 3])
    ids = rng.permutation(total) if spec.shuffle_pages else np.arange(total)
    pt = np.full((B, max_pages), -1, dtype=np.int32)
    off = 0
    for r in range(B):
        pt[r, : caps[r]] = ids[off: off + caps[r]]
        off += caps[r]

    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 7919 + 17)
    k_pool = torch.empty((total, H, PAGE_SIZE, d), dtype=torch.bfloat16, device=device)
    v_pool = torch.empty_like(k_pool)
    _fill_normal_bf16(k_pool, gen)
    _fill_normal_bf16(v_pool, gen)

    hh = spec.heavy_hitters
    heavy = np.zeros((B, H, hh), dtype=np.int32)
    if hh:
        for r in range(B):
            span = int(lengths[r]) - spec.window
            assert span > hh, "context too short for the heavy hitters"
            for h in range(H):
                heavy[r, h] = np.sort(rng.choice(span, size=hh, replace=False))
        pos = torch.as_tensor(heavy.astype(np.int64))                      # [B][H][hh]
        ptt = torch.as_tensor(pt.astype(np.int64))
        pages = torch.gather(ptt[:, None, :].expand(B, H, max_pages), 2, pos // PAGE_SIZE)
        heads = torch.arange(H)[None, :, None].expand(B, H, hh)
        slots = pos % PAGE_SIZE
        idx = (pages.reshape(-1).to(device), heads.reshape(-1).to(device), slots.reshape(-1).to(device))
        k_pool[idx] = k_pool[idx] * spec.heavy_scale

    return KVCache(k_pool, v_pool, torch.as_tensor(pt, device=device),
                   lengths.astype(np.int32), heavy, max_pages, total)


def token_qkv(spec: WorkloadSpec, r: int, positions, seed: int | None = None):
    """q [n][H_q][d], k [n][H_kv][d], v [n][H_kv][d] (bf16, CPU) of the token at each position.

    Each token's projections are a pure function of (seed, request, position), so a draft
    step and the verify pass see the same q/k/v for the same position (one layer, shared
    weights).
    """
    seed = spec.data_seed if seed is None else seed
    qs, ks, vs = [], [], []
    for p in np.atleast_1d(positions):
        g = np.random.default_rng([seed, 7, int(r), int(p)])
        qs.append(g.standard_normal((spec.num_q_heads, spec.head_dim), dtype=np.float32))
        ks.append(g.standard_normal((spec.num_kv_heads, spec.head_dim), dtype=np.float32))
        vs.append(g.standard_normal((spec.num_kv_heads, spec.head_dim), dtype=np.float32))
    cv = lambda a: torch.as_tensor(np.stack(a)).to(torch.bfloat16)  # noqa: E731
    return cv(qs), cv(ks), cv(vs)


def token_logits(spec: WorkloadSpec, r: int, positions, seed: int | None = None):
    """Independent synthetic logits for the tokens at the given positions (float32).

    target row ~ N(0, logit_std^2) per entry; draft row = target + N(0, draft_noise_std^2).
    Both are pure functions of (seed, request, position of the token being decided).
    """
    seed = spec.sample_seed if seed is None else seed
    ps, qs = [], []
    for p in np.atleast_1d(positions):
        g = np.random.default_rng([seed, 11, int(r), int(p)])
        t = (g.standard_normal(spec.vocab) * spec.logit_std).astype(np.float32)
        n = (g.standard_normal(spec.vocab) * spec.draft_noise_std).astype(np.float32)
        ps.append(t)
        qs.append((t + n).astype(np.float32))
    return np.stack(ps), np.stack(qs)


def randn_bf16(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    t = torch.randn(shape, generator=gen, device=device, dtype=torch.float32)
    return (t * scale).to(torch.bfloat16)


def randn_f32(shape, seed: int, device="cpu", scale: float = 1.0) -> torch.Tensor:
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32) * scale


def projection_matrix(spec: WorkloadSpec, device="cpu") -> torch.Tensor:
    """Seeded bf16 projection W [H_q*d][vocab] with entries N(0, 1/(H_q*d))."""
    n = spec.num_q_heads * spec.head_dim
    return randn_bf16((n, spec.vocab), spec.data_seed * 31 + 5, device, scale=1.0 / math.sqrt(n))
