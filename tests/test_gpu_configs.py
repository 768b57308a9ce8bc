"""Whole-workload GPU runs against the oracle: the mixed-phase ragged batch (requests at
different points of their rounds, launches over request subsets, shuffled pages) and the
full-size Qwen3-shaped workloads on sampled requests.

Per request the GPU's round must equal the oracle's round on the same inputs: attention
outputs within 2e-2 + 1e-2 |oracle| (every draft step's output, from the oracle's sparse
attention over the set the GPU selected, and the verify's), selections, drafts and emitted
tokens bit-exact up to the first decision whose own oracle margin to its boundary is below
1e-5 (counted, and required to be rare)."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O
from tests.s3r_testlib import MARGIN, assert_attention_close, compare_round_decisions, f64

pytestmark = pytest.mark.gpu


def _inputs(spec, lens, device="cuda"):
    """q/k/v of each request's block L..L+k and the logits of positions L+1..L+k+1."""
    q, k, v, pl, ql = [], [], [], [], []
    for r, L in enumerate(lens):
        a, b, c = synth.token_qkv(spec, r, range(int(L), int(L) + spec.k + 1))
        p_log, q_log = synth.token_logits(spec, r, range(int(L) + 1, int(L) + spec.k + 2))
        q.append(a), k.append(b), v.append(c), pl.append(p_log), ql.append(q_log[: spec.k])
    cu = lambda t: torch.stack(t).to(device)  # noqa: E731
    return (cu(q), cu(k), cu(v), torch.as_tensor(np.stack(pl)).to(device),
            torch.as_tensor(np.stack(ql)).to(device))


def _oracle_state(spec, kp, vp, pt, r, L):
    cap = int((pt[r] >= 0).sum()) * 16
    K = np.stack([O.gather_positions(kp, pt[r], h, np.arange(cap)) for h in range(spec.num_kv_heads)])
    V = np.stack([O.gather_positions(vp, pt[r], h, np.arange(cap)) for h in range(spec.num_kv_heads)])
    return O.RequestState(K, V, int(L))


def _compare_round(spec, r, res, st, q_r, sel, cnt, sig_prev, L, draft_outs, drafts, verify_out,
                   lse, out_tokens, n_out):
    """Returns True if the request's decisions were all identical, False if the first
    differing one was a boundary case (oracle margin < 1e-5 for that decision).

    draft_outs[i] is the GPU's output of draft step i; the oracle recomputes it over the set
    the GPU selected (the selection itself is checked against the oracle's separately), on
    the state after its round (positions past L+i are not attended at step i)."""
    for h in range(spec.num_kv_heads):
        near = set(O.selection_margin_cases(sig_prev[h], L, spec.budget_bp, spec.window, MARGIN).tolist())
        diff = set(sel[h, : cnt[h]].tolist()) ^ set(res["sel"][h].tolist())
        assert diff <= near, (r, h)
    gsel = [sel[h, : cnt[h]] for h in range(spec.num_kv_heads)]
    for i in range(spec.k):
        o, _ = O.sparse_draft_attention(q_r[i], st.K, st.V, gsel, L, i)
        assert_attention_close(draft_outs[i], o, f"draft r={r} step {i}")
    assert_attention_close(verify_out, res["verify_out"], f"verify r={r}")
    np.testing.assert_allclose(lse, res["lse"], atol=2e-4, rtol=0)
    return compare_round_decisions(res, drafts, out_tokens, n_out, spec.k)


class _DraftRecorder:
    """Wraps a MixedPhaseDriver's draft launches and keeps, per (request, step), the first
    output and draft token written for it (the request's first round: steps of its next
    round come later and are not kept)."""

    def __init__(self, drv, eng, keep=None):
        self.eng, self.keep = eng, None if keep is None else set(int(r) for r in keep)
        self.out, self.tok = {}, {}
        inner = drv._draft

        def wrapped(ids, steps, *args):
            inner(ids, steps, *args)
            o = self.eng.buf.draft_out.float().cpu().numpy().astype(np.float64)
            t = self.eng.buf.draft_tokens.cpu().numpy()
            for r, i in zip(np.asarray(ids).tolist(), np.asarray(steps).tolist()):
                if self.keep is None or r in self.keep:
                    self.out.setdefault((r, i), o[r])
                    self.tok.setdefault((r, i), int(t[r, i]))

        drv._draft = wrapped

    def of(self, r, k):
        return [self.out[(r, i)] for i in range(k)], np.array([self.tok[(r, i)] for i in range(k)])


def _record_drafts(drv, eng, keep=None):
    return _DraftRecorder(drv, eng, keep)


def test_mixed_phase_batch_matches_oracle():
    """Ragged batch at mixed round phases (the high-concurrency workload's shape, fewer and
    shorter requests so the oracle stays quick): each iteration drafts every request that is
    mid-round with one launch over its ids and verifies the others with another; after k+1
    iterations every request has finished the round it was in, which must equal the
    oracle's round for that request."""
    spec = synth.WORKLOADS["ragged"].with_(num_requests=24, lengths=("loguniform", 1024, 3072))
    k = spec.k
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=2 * (k + 1) + 16)
    kp, vp = cache.k_pool.float().numpy(), cache.v_pool.float().numpy()
    pt = cache.page_table.numpy()
    seq = torch.as_tensor(lens, dtype=torch.int32).cuda()
    eng = s3r.S3REngine(cache.k_pool.cuda(), cache.v_pool.cuda(), cache.page_table.cuda(), seq,
                        spec.num_q_heads, k=k, budget_bp=spec.budget_bp, window=spec.window,
                        vocab=spec.vocab, seed=spec.sample_seed)
    q, kb, vb, pl, ql = _inputs(spec, lens)
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    phases = synth.initial_phases(spec)
    assert len(set(phases.tolist())) > 1
    drv = s3r.MixedPhaseDriver(eng, phases)
    rec = _record_drafts(drv, eng)
    drv.start(q, kb, vb, ql)
    sel = eng.buf.sel_idx.cpu().numpy()
    cnt = eng.buf.sel_count.cpu().numpy()
    done = np.zeros(spec.num_requests, dtype=bool)
    for _ in range(k + 1):
        ids = drv.iterate(q, kb, vb, pl, ql)
        assert not done[ids].any()
        done[ids] = True
    assert done.all()
    assert eng.check_errors() == 0
    b = eng.buf
    exact = 0
    for r in range(spec.num_requests):
        L = int(lens[r])
        st = _oracle_state(spec, kp, vp, pt, r, L)
        O.prefill_scores(st, f64(q[r, 0]), f64(kb[r, 0]), f64(vb[r, 0]))
        sig_prev = st.sigma
        res = O.run_round(st, r, spec.sample_seed, k, spec.budget_bp, spec.window, f64(q[r]),
                          f64(kb[r]), f64(vb[r]), ql[r].cpu().numpy(), pl[r].cpu().numpy())
        outs, drafts = rec.of(r, k)
        exact += _compare_round(spec, r, res, st, f64(q[r]), sel[r], cnt[r], sig_prev, L, outs, drafts,
                                f64(b.verify_out[r]), f64(b.lse[r]), b.out_tokens[r].cpu().numpy(),
                                int(b.n_out[r]))
        assert int(eng.seq_lens[r]) == L + int(b.n_out[r])
    assert exact >= spec.num_requests - 2
    st = b.stats.cpu().numpy()
    assert st[1] == spec.num_requests


@pytest.mark.parametrize("workload,point,picks", [
    ("qwen3-1.7b", None, 6), ("qwen3-8b", None, 6),
    ("sweep", (500, 6), 3),     # the 32 x 24576 budget-sweep shapes at the bench point
    ("sweep", (2000, 8), 3),    # k = 8: 36 rows per KV head, the 64-row tensor-memory verify
])
def test_full_size_round_on_sampled_requests(workload, point, picks):
    """One round of the whole Qwen3-shaped batch at full size (the benchmark's launch
    configuration); the oracle replays sampled requests. The sweep shapes run with the
    synthetic logit model here (their projection logits are covered at reduced size below)."""
    spec = synth.WORKLOADS[workload]
    if point is not None:
        spec = spec.with_(budget_bp=point[0], k=point[1], vocab=32768, projection_logits=False,
                          draft_noise_std=0.5)
    k = spec.k
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=k + 1 + 16, device="cuda")
    seq = torch.as_tensor(lens, dtype=torch.int32, device="cuda")
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    q = synth.randn_bf16((NR, k + 1, Hq, d), 100, "cuda")
    kb = synth.randn_bf16((NR, k + 1, Hkv, d), 101, "cuda")
    vb = synth.randn_bf16((NR, k + 1, Hkv, d), 102, "cuda")
    pl = synth.randn_f32((NR, k + 1, V), 103, "cuda", scale=spec.logit_std)
    ql = (pl[:, :k] + synth.randn_f32((NR, k, V), 104, "cuda", scale=spec.draft_noise_std)).contiguous()
    rng = np.random.default_rng(spec.data_seed + k)
    picks = sorted(rng.choice(NR, size=picks, replace=False).tolist())
    pt = cache.page_table.cpu().numpy()
    host = {}
    for r in picks:    # the requests' pages before the round writes its block
        ids = pt[r][pt[r] >= 0]
        host[r] = (cache.k_pool[ids].float().cpu().numpy(), cache.v_pool[ids].float().cpu().numpy())
    eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k,
                        budget_bp=spec.budget_bp, window=spec.window, vocab=V, seed=spec.sample_seed)
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    eng.select()
    sel = eng.buf.sel_idx.cpu().numpy()
    cnt = eng.buf.sel_count.cpu().numpy()
    outs = []
    for i in range(k):
        eng.draft_step(i, q, kb, vb, ql)
        outs.append(eng.buf.draft_out.clone())
    eng.verify(q, kb, vb)
    eng.sample_and_commit(pl, ql)
    assert eng.check_errors() == 0
    b = eng.buf
    drafts = b.draft_tokens.cpu().numpy()
    exact = 0
    for r in picks:
        kpr, vpr = host[r]
        local = np.arange(kpr.shape[0], dtype=np.int32)
        K = np.stack([O.gather_positions(kpr, local, h, np.arange(len(local) * 16)) for h in range(Hkv)])
        Vv = np.stack([O.gather_positions(vpr, local, h, np.arange(len(local) * 16)) for h in range(Hkv)])
        st = O.RequestState(K, Vv, int(lens[r]))
        O.prefill_scores(st, f64(q[r, 0]), f64(kb[r, 0]), f64(vb[r, 0]))
        sig_prev = st.sigma
        res = O.run_round(st, r, spec.sample_seed, k, spec.budget_bp, spec.window, f64(q[r]),
                          f64(kb[r]), f64(vb[r]), ql[r].cpu().numpy(), pl[r].cpu().numpy())
        exact += _compare_round(spec, r, res, st, f64(q[r]), sel[r], cnt[r], sig_prev, int(lens[r]),
                                [f64(o[r]) for o in outs], drafts[r], f64(b.verify_out[r]),
                                f64(b.lse[r]), b.out_tokens[r].cpu().numpy(), int(b.n_out[r]))
    assert exact >= len(picks) - 1


def test_projection_logits_round_matches_oracle():
    """The budget-sweep workload's logit model (a seeded bf16 projection of the
    head-concatenated attention outputs, fewer and shorter requests so the oracle stays
    quick): attention outputs of every draft step and of the verify match the oracle's, and
    the GPU samplers, given the oracle's own logits, take the oracle's decisions."""
    spec = synth.WORKLOADS["sweep"].with_(num_requests=3, lengths=("fixed", (3000, 4100, 2500)))
    k, V = spec.k, spec.vocab
    NR, Hq, Hkv, d = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=k + 1 + 16)
    kp, vp = cache.k_pool.float().numpy(), cache.v_pool.float().numpy()
    pt = cache.page_table.numpy()
    W = synth.projection_matrix(spec, "cuda")
    W64 = W.double().cpu().numpy()
    gamma = 3.0
    seq = torch.as_tensor(lens, dtype=torch.int32).cuda()
    eng = s3r.S3REngine(cache.k_pool.cuda(), cache.v_pool.cuda(), cache.page_table.cuda(), seq,
                        Hq, k=k, budget_bp=spec.budget_bp, window=spec.window, vocab=V,
                        seed=spec.sample_seed)
    q, kb, vb, _, _ = _inputs(spec.with_(vocab=8), lens)
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    ql = torch.empty((NR, k, V), device="cuda")
    pl = torch.empty((NR, k + 1, V), device="cuda")
    draft_outs = []

    def draft_fn(i, out, q_logits):
        draft_outs.append(out.clone())
        q_logits[:, i] = gamma * (out.float().reshape(NR, -1) @ W.float())

    def target_fn(vout, p_logits):
        p_logits.copy_((gamma * (vout.float().reshape(NR * (k + 1), -1) @ W.float())).view(NR, k + 1, V))

    eng.round(q, kb, vb, pl, ql, draft_logits_fn=draft_fn, target_logits_fn=target_fn)
    assert eng.check_errors() == 0
    n_out = eng.buf.n_out.cpu().numpy()
    assert ((n_out >= 1) & (n_out <= k + 1)).all()
    gsel, gcnt = eng.buf.sel_idx.cpu().numpy(), eng.buf.sel_count.cpu().numpy()
    # the oracle's round, with logits from its own attention outputs
    oq = np.zeros((NR, k, V), np.float32)
    op = np.zeros((NR, k + 1, V), np.float32)
    odrafts = np.zeros((NR, k), np.int32)
    res_tok = []
    for r in range(NR):
        L = int(lens[r])
        st = _oracle_state(spec, kp, vp, pt, r, L)
        O.prefill_scores(st, f64(q[r, 0]), f64(kb[r, 0]), f64(vb[r, 0]))
        sel = [O.select_positions(st.sigma[h], L, spec.budget_bp, spec.window) for h in range(Hkv)]
        same_sel = True
        for h in range(Hkv):
            got = set(gsel[r, h, : gcnt[r, h]].tolist())
            near = set(O.selection_margin_cases(st.sigma[h], L, spec.budget_bp, spec.window, MARGIN).tolist())
            assert (got ^ set(sel[h].tolist())) <= near, (r, h)
            same_sel &= got == set(sel[h].tolist())
        gs = [gsel[r, h, : gcnt[r, h]] for h in range(Hkv)]
        for i in range(k):
            st.write([L + i], [f64(kb[r, i])], [f64(vb[r, i])])
            o, _ = O.sparse_draft_attention(f64(q[r, i]), st.K, st.V, sel, L, i)
            # the GPU's output against the oracle's attention over the GPU's own set
            og = o if same_sel else O.sparse_draft_attention(f64(q[r, i]), st.K, st.V, gs, L, i)[0]
            assert_attention_close(f64(draft_outs[i][r]), og, f"draft r={r} i={i}")
            oq[r, i] = gamma * (o.reshape(-1) @ W64)
            u0 = float(O.uniform(spec.sample_seed, r, L + i + 1, O.STREAM_DRAFT))
            odrafts[r, i], _ = O.draft_sample(oq[r, i], u0)
        st.write(list(range(L, L + k + 1)), f64(kb[r]), f64(vb[r]))
        vo, _, _, _ = O.verify_attention(f64(q[r]), st.K, st.V, L)
        assert_attention_close(f64(eng.buf.verify_out[r]), vo, f"verify r={r}")
        op[r] = gamma * (vo.reshape(k + 1, -1) @ W64)
        res_tok.append(O.spec_sample(op[r], oq[r], odrafts[r], spec.sample_seed, r, L))
    # the GPU samplers on the oracle's logits
    batch = s3r.make_batch(torch.as_tensor(lens, dtype=torch.int32).cuda())
    cdesc = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cdesc, NR, 1, k, V, 1))
    qd, pd = torch.as_tensor(oq).cuda(), torch.as_tensor(op).cuda()
    gd = torch.zeros((NR, k), dtype=torch.int32, device="cuda")
    for i in range(k):
        s3r.s3r_draft_sample(batch, torch.full((NR,), i, dtype=torch.int32, device="cuda"), k, qd,
                             V, spec.sample_seed, gd, ws)
    out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
    nout = torch.zeros(NR, dtype=torch.int32, device="cuda")
    s3r.s3r_spec_sample(batch, k, pd, qd, torch.as_tensor(odrafts).cuda(), V, spec.sample_seed,
                        out, nout, ws)
    assert s3r.s3r_get_error(ws) == 0
    gd, out, nout = gd.cpu().numpy(), out.cpu().numpy(), nout.cpu().numpy()
    for r in range(NR):
        toks, n, margins = res_tok[r]
        for i in range(k):
            if gd[r, i] != odrafts[r, i]:
                u0 = float(O.uniform(spec.sample_seed, r, int(lens[r]) + i + 1, O.STREAM_DRAFT))
                assert O.draft_sample(oq[r, i], u0)[1] < MARGIN, (r, i)
        if not (nout[r] == n and out[r, :n].tolist() == toks.tolist()):
            assert margins.min() < MARGIN, r


def test_full_size_mixed_phase_batch_on_sampled_requests():
    """The high-concurrency workload at full size: 256 requests, contexts log-uniform in
    [1024, 16384], shuffled pages, mixed round phases; k+1 driver iterations complete one
    round per request, and the oracle replays twelve sampled requests."""
    spec = synth.WORKLOADS["ragged"]
    k = spec.k
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=2 * (k + 1) + 16, device="cuda")
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    q = synth.randn_bf16((NR, k + 1, Hq, d), 200, "cuda")
    kb = synth.randn_bf16((NR, k + 1, Hkv, d), 201, "cuda")
    vb = synth.randn_bf16((NR, k + 1, Hkv, d), 202, "cuda")
    pl = synth.randn_f32((NR, k + 1, V), 203, "cuda", scale=spec.logit_std)
    ql = (pl[:, :k] + synth.randn_f32((NR, k, V), 204, "cuda", scale=spec.draft_noise_std)).contiguous()
    picks = sorted(np.random.default_rng(3).choice(NR, size=12, replace=False).tolist())
    pt = cache.page_table.cpu().numpy()
    host = {}
    for r in picks:
        ids = pt[r][pt[r] >= 0]
        host[r] = (cache.k_pool[ids].float().cpu().numpy(), cache.v_pool[ids].float().cpu().numpy())
    seq = torch.as_tensor(lens, dtype=torch.int32, device="cuda")
    eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k,
                        budget_bp=spec.budget_bp, window=spec.window, vocab=V, seed=spec.sample_seed)
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    drv = s3r.MixedPhaseDriver(eng, synth.initial_phases(spec))
    rec = _record_drafts(drv, eng, keep=picks)
    drv.start(q, kb, vb, ql)
    sel = eng.buf.sel_idx.cpu().numpy()
    cnt = eng.buf.sel_count.cpu().numpy()
    for _ in range(k + 1):
        drv.iterate(q, kb, vb, pl, ql)
    assert eng.check_errors() == 0
    b = eng.buf
    exact = 0
    for r in picks:
        kpr, vpr = host[r]
        local = np.arange(kpr.shape[0], dtype=np.int32)
        K = np.stack([O.gather_positions(kpr, local, h, np.arange(len(local) * 16)) for h in range(Hkv)])
        Vv = np.stack([O.gather_positions(vpr, local, h, np.arange(len(local) * 16)) for h in range(Hkv)])
        L = int(lens[r])
        st = O.RequestState(K, Vv, L)
        O.prefill_scores(st, f64(q[r, 0]), f64(kb[r, 0]), f64(vb[r, 0]))
        sig_prev = st.sigma
        res = O.run_round(st, r, spec.sample_seed, k, spec.budget_bp, spec.window, f64(q[r]),
                          f64(kb[r]), f64(vb[r]), ql[r].cpu().numpy(), pl[r].cpu().numpy())
        outs, drafts = rec.of(r, k)
        exact += _compare_round(spec, r, res, st, f64(q[r]), sel[r], cnt[r], sig_prev, L, outs, drafts,
                                f64(b.verify_out[r]), f64(b.lse[r]), b.out_tokens[r].cpu().numpy(),
                                int(b.n_out[r]))
        assert int(eng.seq_lens[r]) == L + int(b.n_out[r])
    assert exact >= len(picks) - 1
