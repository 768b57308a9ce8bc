"""Whole rounds on the GPU (engine over the C ABI) against the oracle's rounds, tiny
workload; device error reporting without faults."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O
from tests.s3r_testlib import MARGIN, assert_attention_close, f64
from tests.test_oracle_round import make_states

pytestmark = pytest.mark.gpu


def gpu_engine(spec, rounds, page_select=False, greedy=False, k_max=None):
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=800)
    seq = torch.as_tensor(lens, dtype=torch.int32).cuda()
    eng = s3r.S3REngine(cache.k_pool.cuda(), cache.v_pool.cuda(), cache.page_table.cuda(), seq,
                        spec.num_q_heads, k=spec.k, budget_bp=spec.budget_bp, window=spec.window,
                        vocab=spec.vocab, seed=spec.sample_seed, page_select=page_select,
                        greedy=greedy, k_max=k_max)
    qs, ks, vs = zip(*[synth.token_qkv(spec, r, [int(lens[r])]) for r in range(spec.num_requests)])
    eng.prefill(torch.stack(qs).cuda(), torch.stack(ks).cuda(), torch.stack(vs).cuda())
    return eng


def round_inputs(spec, lengths):
    q, k, v, pl, ql = [], [], [], [], []
    for r, L in enumerate(lengths):
        a, b, c = synth.token_qkv(spec, r, range(L, L + spec.k + 1))
        p_log, q_log = synth.token_logits(spec, r, range(L + 1, L + spec.k + 2))
        q.append(a), k.append(b), v.append(c), pl.append(p_log), ql.append(q_log[: spec.k])
    cu = lambda t: torch.stack(t).cuda()  # noqa: E731
    return cu(q), cu(k), cu(v), torch.as_tensor(np.stack(pl)).cuda(), torch.as_tensor(np.stack(ql)).cuda()


def near_threshold(sigma, L, spec, page):
    """Positions whose selection may go either way (oracle margin below 1e-5)."""
    if page == 1:
        return set(O.selection_margin_cases(sigma, L, spec.budget_bp, spec.window, MARGIN).tolist())
    pages = O.page_selection_margin_cases(sigma, L, spec.budget_bp, spec.window, page, MARGIN)
    return {int(q) * page + t for q in pages for t in range(page)}


K_SCHEDULE = [6, 3, 1, 5, 2, 6, 4, 1, 1, 6]


@pytest.mark.parametrize("page,greedy,vary_k", [(1, False, False), (16, False, False), (1, True, False),
                                                (16, True, False), (1, False, True), (16, True, True)])
def test_rounds_match_oracle_tiny(page, greedy, vary_k):
    """Rounds are compared request by request. A decision whose oracle margin is below 1e-5
    may go either way; if the GPU then differs, that request's later rounds are no longer
    comparable and it leaves the comparison (counted). page 16: page-granular selection;
    greedy: argmax drafts and greedy verification (no sampling margins: tokens must match);
    vary_k: the draft length changes from round to round (adaptive horizon), the selection
    reading the scores of a verify of another length."""
    spec0 = synth.WORKLOADS["tiny"]
    n_rounds = 40
    eng = gpu_engine(spec0, n_rounds, page_select=page > 1, greedy=greedy, k_max=spec0.k)
    states = make_states(spec0)
    alive = [True] * spec0.num_requests
    compared = diverged = boundary = 0
    for rnd in range(n_rounds):
        spec = spec0.with_(k=K_SCHEDULE[rnd % len(K_SCHEDULE)]) if vary_k else spec0
        eng.set_k(spec.k)
        lengths = eng.seq_lens.cpu().numpy().tolist()
        for r, st in enumerate(states):
            if alive[r]:
                assert lengths[r] == st.L
        q, k, v, pl, ql = round_inputs(spec, lengths)
        eng.round(q, k, v, pl, ql)
        assert eng.check_errors() == 0
        b = eng.buf
        sel = b.sel_idx.cpu().numpy()
        cnt = b.sel_count.cpu().numpy()
        for r, st in enumerate(states):
            if not alive[r]:
                continue
            sig_prev, L = st.sigma, st.L
            res = O.run_round(st, r, spec.sample_seed, spec.k, spec.budget_bp, spec.window,
                              f64(q[r]), f64(k[r]), f64(v[r]), ql[r].cpu().numpy(), pl[r].cpu().numpy(),
                              page=page, greedy=greedy)
            for h in range(spec.num_kv_heads):
                near = near_threshold(sig_prev[h], L, spec, page)
                diff = set(sel[r, h, : cnt[r, h]].tolist()) ^ set(res["sel"][h].tolist())
                assert diff <= near
            assert_attention_close(f64(b.verify_out[r]), res["verify_out"], f"verify r={r}")
            np.testing.assert_allclose(f64(b.lse[r]), res["lse"], atol=2e-4, rtol=0)
            near_decision = min(res["draft_margin"].min(), res["margins"].min()) < MARGIN
            boundary += int(near_decision)
            n = int(b.n_out[r])
            same = (b.draft_tokens[r].tolist() == res["drafts"].tolist() and n == res["n_out"]
                    and b.out_tokens[r, :n].tolist() == res["tokens"].tolist())
            if not same:
                assert near_decision, (rnd, r)
                alive[r] = False
                diverged += 1
                continue
            compared += 1
    assert compared >= 40
    st = b.stats.cpu().numpy()
    assert st[1] > 0 and st[0] >= st[1]
    print(f"compared {compared} request-rounds, boundary decisions {boundary}, diverged {diverged}")


def test_adaptive_horizon_follows_acceptance_and_costs():
    """The controller on whole rounds: with every draft accepted (draft logits equal to the
    target's) and verify far dearer than a draft step it keeps the longest horizon; once a
    draft step is made dear it drops to one draft; rounds at the chosen lengths stay
    error-free and count decisions only at the positions drafted."""
    spec = synth.WORKLOADS["tiny"]
    eng = gpu_engine(spec, 0, k_max=spec.k)
    ctl = s3r.AdaptiveHorizon(eng, c_draft=1.0, c_verify=1000.0, prior_weight=1.0)

    def rounds(n):
        for _ in range(n):
            lengths = eng.seq_lens.cpu().numpy().tolist()
            q, k, v, pl, ql = round_inputs(spec.with_(k=eng.k), lengths)
            eng.round(q, k, v, pl, pl[:, : eng.k].contiguous())
            assert eng.check_errors() == 0

    rounds(3)
    assert ctl.step() == spec.k and eng.k == spec.k
    ctl.c_draft = 1e6
    assert ctl.step() == 1 and eng.k == 1
    before = eng.buf.stats.cpu().numpy()
    rounds(2)
    after = eng.buf.stats.cpu().numpy()
    dec = after[2 + s3r.MAX_K: 2 + 2 * s3r.MAX_K] - before[2 + s3r.MAX_K: 2 + 2 * s3r.MAX_K]
    assert dec[0] == 2 * spec.num_requests and not dec[1:].any()


def test_device_errors_are_reported_not_faulted():
    spec = synth.WORKLOADS["tiny"]
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=32)
    pt = cache.page_table.clone()
    pt[0, 3] = 10 ** 6                                # page id outside the pool
    seq = torch.as_tensor(lens, dtype=torch.int32).cuda()
    kp, vp = cache.k_pool.cuda(), cache.v_pool.cuda()
    c = s3r.make_cache(kp, vp, spec.num_q_heads)
    b = s3r.make_batch(seq, pt.cuda())
    ws = s3r.new_workspace(s3r.s3r_workspace_size(c, 2, cache.max_pages, 6, 64, 128))
    q = synth.randn_bf16((2, 7, 2, 64), 1, "cuda")
    kv = synth.randn_bf16((2, 7, 1, 64), 2, "cuda")
    out = torch.empty_like(q)
    lse = torch.empty((2, 7, 2), device="cuda")
    s3r.s3r_verify_attn(c, b, 6, q, kv, kv, out, lse, None, ws)
    err = s3r.s3r_get_error(ws)
    assert err & (1 << 5)
    assert torch.isfinite(out.float()).all()          # the bad page reads as zeros
    assert s3r.s3r_get_error(ws) == 0                 # cleared
    # a selected index past the committed length
    sel = torch.zeros((2, 1, 8), dtype=torch.int32, device="cuda")
    sel[1, 0, 2] = 5000
    cnt = torch.full((2, 1), 8, dtype=torch.int32, device="cuda")
    step = torch.zeros(2, dtype=torch.int32, device="cuda")
    b2 = s3r.make_batch(seq, cache.page_table.cuda())
    s3r.s3r_sparse_draft_attn(c, b2, step, q[:, 0], kv[:, 0], kv[:, 0], sel, cnt, out[:, 0].contiguous(), None, ws)
    assert s3r.s3r_get_error(ws) & (1 << 5)
    # non-finite logits
    V = 64
    pl = torch.randn((2, 7, V), device="cuda")
    pl[1, 2, 10] = float("nan")
    drafts = torch.zeros((2, 6), dtype=torch.int32, device="cuda")
    out_t = torch.zeros((2, 7), dtype=torch.int32, device="cuda")
    n_out = torch.zeros(2, dtype=torch.int32, device="cuda")
    s3r.s3r_spec_sample(b2, 6, pl, pl[:, :6].contiguous(), drafts, V, 1, out_t, n_out, ws)
    assert s3r.s3r_get_error(ws) & (1 << 6)
    # host-side rejection leaves nothing launched
    before = s3r.s3r_launch_count()
    with pytest.raises(s3r.S3RError):
        s3r.s3r_select_kv(c, b2, torch.empty((2, 1, 14, 64), device="cuda"), lse, 6, 500, 3, sel, cnt, ws)
    assert s3r.s3r_launch_count() == before


def test_adaptive_horizon_with_stale_counts_lags_one_interval():
    """With stale_counts the controller reads the counters it copied at its previous
    decision: its first decision sees no new evidence (the prior alone), its second the
    rounds before the first one, and it never waits for the device in between."""
    spec = synth.WORKLOADS["tiny"]
    eng = gpu_engine(spec, 0, k_max=spec.k)
    ctl = s3r.AdaptiveHorizon(eng, c_draft=1.0, c_verify=1000.0, prior_weight=1.0, prior_alpha=0.0,
                              stale_counts=True)

    def rounds(n):
        for _ in range(n):
            lengths = eng.seq_lens.cpu().numpy().tolist()
            q, k, v, pl, ql = round_inputs(spec.with_(k=eng.k), lengths)
            eng.round(q, k, v, pl, pl[:, : eng.k].contiguous())
            assert eng.check_errors() == 0

    rounds(3)
    # prior 0 and no counts yet: one draft (every longer horizon is expected to add nothing)
    assert ctl.step() == 1 and eng.k == 1
    # now the three rounds before the first decision (every draft accepted) are seen
    assert ctl.step() == spec.k and eng.k == spec.k
