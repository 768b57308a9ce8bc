"""Shared helpers of the GPU parity tests: seeded cases on the device and their dense
float64 copies for the oracle. Inputs come from `synth`; expected values from `oracle`."""
from __future__ import annotations

import numpy as np
import torch

import synth
from oracle import s3r_oracle as O

ATOL, RTOL = 2e-2, 1e-2          # attention outputs: bf16 out, fp32 accumulation
MARGIN = 1e-5                     # decisions closer than this to a boundary are not compared


def spec_for(H_q, H_kv, d, lens, k=6, budget_bp=500, window=64, vocab=64, seed=0, heavy=0,
             shuffle=False):
    return synth.WORKLOADS["tiny"].with_(num_requests=len(lens), num_q_heads=H_q, num_kv_heads=H_kv,
                                  head_dim=d, lengths=("fixed", tuple(int(x) for x in lens)),
                                  k=k, budget_bp=budget_bp, window=window, vocab=vocab,
                                  data_seed=seed, heavy_hitters=heavy, shuffle_pages=shuffle)


class Case:
    """A paged cache generated on the host, copied to the GPU, plus host float copies."""

    def __init__(self, spec, extra_tokens, seed=None):
        self.spec = spec
        self.cache = synth.build_cache(spec, synth.make_lengths(spec), extra_tokens, "cpu", seed)
        self.k_pool = self.cache.k_pool.cuda()
        self.v_pool = self.cache.v_pool.cuda()
        self.page_table = self.cache.page_table.cuda()
        self.lens = self.cache.lengths.copy()
        self.seq_lens = torch.as_tensor(self.lens, dtype=torch.int32).cuda()

    def host_pools(self):
        """Current device pools as float32 numpy arrays."""
        return self.k_pool.float().cpu().numpy(), self.v_pool.float().cpu().numpy()

    def dense(self, r, upto, pools=None):
        """K, V [H_kv][upto][d] float64 of request r from the (device) pools."""
        kp, vp = pools if pools is not None else self.host_pools()
        pt = self.cache.page_table.numpy()[r]
        H = self.spec.num_kv_heads
        K = np.stack([O.gather_positions(kp, pt, h, np.arange(upto)) for h in range(H)])
        V = np.stack([O.gather_positions(vp, pt, h, np.arange(upto)) for h in range(H)])
        return K, V


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_attention_close(gpu, ref, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    err = np.abs(gpu - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err {err.max():.3g}"


def compare_round_decisions(res, drafts, tokens, n_out, k):
    """Compare one request's sampled decisions of a round with the oracle's round `res`.

    Decisions are taken in order: the k draft draws, then the accept tests of the drafts up
    to the first rejection, then the final draw. Everything before the first decision that
    differs must be identical, and that decision must be a boundary case: its own oracle
    margin (|u - C_edge / Z| for a draw, |u - p/q| for an accept test) below MARGIN.
    Returns True if the whole round was identical, False for an excused boundary case."""
    od = np.asarray(res["drafts"])
    for i in range(k):
        if int(drafts[i]) != int(od[i]):
            assert res["draft_margin"][i] < MARGIN, ("draft", i, float(res["draft_margin"][i]))
            return False   # later decisions follow other drafts
    ot, on, om = list(res["tokens"]), int(res["n_out"]), np.asarray(res["margins"])
    gt = [int(x) for x in tokens[:n_out]]
    if n_out == on and gt == ot:
        return True
    a_o, a_g = on - 1, int(n_out) - 1     # drafts each side accepted
    j = min(a_o, a_g)
    assert gt[:j] == ot[:j] == [int(x) for x in od[:j]], ("accepted prefix", j)
    if a_o != a_g:                         # the accept test of draft j went both ways
        assert om[j] < MARGIN, ("accept", j, om.tolist())
    else:                                  # same accepts, the final draw differs
        assert om[-1] < MARGIN, ("draw", j, om.tolist())
    return False


def check_sampler_margins(gpu_margins, oracle_margins, count):
    """The first `count` margins the GPU reported agree with the oracle's to 1e-5 (plus
    1e-5 relative): both measure the same distance, the GPU from fp32 weights."""
    g = np.asarray(gpu_margins, dtype=np.float64)[:count]
    o = np.asarray(oracle_margins, dtype=np.float64)[:count]
    fin = np.isfinite(o)
    assert np.all(np.abs(g[fin] - o[fin]) <= 1e-5 + 1e-5 * np.abs(o[fin])), (g, o)
