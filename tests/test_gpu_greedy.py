"""Greedy (temperature 0) mode on the GPU against the oracle: argmax drafts and greedy
verification are exact (ties to the lowest id on both sides), so tokens must be equal."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("V", [64, 151936, 20000])
def test_greedy_draft_and_verify_match_oracle(V):
    NR, k = 40, 6
    rng = np.random.default_rng(V)
    p = (rng.normal(size=(NR, k + 1, V)) * 1.4).astype(np.float32)
    q = (p[:, :k] + rng.normal(size=(NR, k, V)) * 0.5).astype(np.float32)
    q[::3] = p[::3, :k]                       # every third request accepts all k drafts
    q[1::6, 3:] = p[1::6, 3:k]                # and some accept a middle prefix
    if V == 64:   # ties: quantised logits
        p = np.round(p).astype(np.float32)
        q = np.round(q).astype(np.float32)
    p[3, 2, 7] = np.nan   # NaN counts as -inf (and is flagged)
    lens = torch.as_tensor(rng.integers(100, 1000, size=NR).astype(np.int32)).cuda()
    batch = s3r.make_batch(lens)
    pool = torch.zeros((1, 8, 16, 128), dtype=torch.bfloat16, device="cuda")
    cache = s3r.make_cache(pool, pool.clone(), 8)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    qd, pd = torch.as_tensor(q).cuda(), torch.as_tensor(p).cuda()
    drafts = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    for i in range(k):
        s3r.s3r_draft_argmax(batch, torch.full((NR,), i, dtype=torch.int32, device="cuda"), k, qd,
                             V, drafts, ws)
    out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
    n_out = torch.zeros(NR, dtype=torch.int32, device="cuda")
    s3r.s3r_greedy_verify(batch, k, pd, drafts, V, out, n_out, ws)
    err = s3r.s3r_get_error(ws)
    assert err == 1 << 6                       # the NaN, flagged
    drafts, out, n_out = drafts.cpu().numpy(), out.cpu().numpy(), n_out.cpu().numpy()
    accepted = set()
    for r in range(NR):
        want = [O.argmax_token(q[r, i]) for i in range(k)]
        assert drafts[r].tolist() == want, r
        toks, n = O.greedy_verify(p[r], want)
        assert n_out[r] == n and out[r, :n].tolist() == toks.tolist(), r
        accepted.add(n)
    assert 1 in accepted and k + 1 in accepted


def test_greedy_rounds_through_the_engine():
    """Whole greedy rounds on the tiny workload; identical draft and target logits must
    accept every draft (k + 1 tokens per round)."""
    spec = synth.WORKLOADS["tiny"]
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=200)
    seq = torch.as_tensor(lens, dtype=torch.int32).cuda()
    eng = s3r.S3REngine(cache.k_pool.cuda(), cache.v_pool.cuda(), cache.page_table.cuda(), seq,
                        spec.num_q_heads, k=spec.k, budget_bp=spec.budget_bp, window=spec.window,
                        vocab=spec.vocab, seed=spec.sample_seed, greedy=True)
    NR, k = spec.num_requests, spec.k
    q = synth.randn_bf16((NR, k + 1, spec.num_q_heads, spec.head_dim), 1, "cuda")
    kb = synth.randn_bf16((NR, k + 1, spec.num_kv_heads, spec.head_dim), 2, "cuda")
    vb = synth.randn_bf16((NR, k + 1, spec.num_kv_heads, spec.head_dim), 3, "cuda")
    pl = synth.randn_f32((NR, k + 1, spec.vocab), 4, "cuda")
    ql = pl[:, :k].contiguous()
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    before = s3r.s3r_launch_count()
    for _ in range(3):
        eng.round(q, kb, vb, pl, ql)
    # the first round selects from the prefill's logits (scores + select); every round's
    # sampling is joined by the next selection's scores pass, so three rounds from the prefill
    # launch one more than three steady-state rounds
    assert s3r.s3r_launch_count() - before == 3 * eng.launches_per_round + (1 if eng.overlap_scores else 0)
    assert eng.check_errors() == 0
    st = eng.buf.stats.cpu().numpy()
    assert st[0] == 3 * NR * (k + 1) and st[1] == 3 * NR
