"""GPU parity of selection, Philox, draft sampling and speculative sampling."""
import math

import numpy as np
import pytest
import torch
from scipy import stats

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O
from tests.s3r_testlib import MARGIN, Case, check_sampler_margins, f64, spec_for

pytestmark = pytest.mark.gpu


def test_philox_matches_oracle_bitwise():
    n = 1 << 20
    rng = np.random.default_rng(0)
    req = rng.integers(0, 1 << 20, size=n).astype(np.int32)
    pos = rng.integers(0, 1 << 30, size=n).astype(np.int32)
    seed = 0x1234567890ABCDEF
    for stream in (0, 1, 2):
        words = torch.empty((n, 4), dtype=torch.int32, device="cuda")
        u = torch.empty(n, dtype=torch.float32, device="cuda")
        s3r.s3r_philox(seed, stream, torch.as_tensor(req).cuda(), torch.as_tensor(pos).cuda(), words, u)
        ctr = np.stack([pos.astype(np.uint64), req.astype(np.uint64), np.full(n, stream, np.uint64),
                        np.zeros(n, np.uint64)], 1)
        key = np.broadcast_to(np.array([seed & 0xFFFFFFFF, seed >> 32], np.uint64), (n, 2))
        ref = O.philox4x32_10(ctr, key)
        got = words.cpu().numpy().view(np.uint32)
        assert np.array_equal(got, ref)
        assert np.array_equal(u.cpu().numpy().astype(np.float64), O.uniform(seed, req, pos, stream))


def _select_setup(lens, Hkv=8, Hq=32):
    spec = spec_for(Hq, Hkv, 128, lens, seed=2)
    case = Case(spec, extra_tokens=16)
    return case, s3r.make_cache(case.k_pool, case.v_pool, Hq), s3r.make_batch(case.seq_lens, case.page_table)


@pytest.mark.parametrize("bp,W", [(500, 64), (2500, 16), (10000, 8), (100, 64), (1, 1)])
def test_select_from_scores_is_bit_exact(bp, W):
    lens = [5000, 64, 30, 12000, 1]
    case, cache, batch = _select_setup(lens)
    rng = np.random.default_rng(bp + W)
    NR, H = len(lens), 8
    stride = max(lens) + 8
    scores = (rng.integers(0, 50, size=(NR, H, stride)) / 7.0).astype(np.float32)   # many ties
    scores[0, 0, :100] = rng.normal(size=100).astype(np.float32)                   # negatives too
    sel = torch.zeros((NR, H, stride), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((NR, H), dtype=torch.int32, device="cuda")
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 6, 64, 64))
    s3r.s3r_select_from_scores(cache, batch, torch.as_tensor(scores).cuda(), bp, W, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) == 0
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for r, L in enumerate(lens):
        for h in range(H):
            ref = O.select_positions(scores[r, h].astype(np.float64), L, bp, W)
            assert cnt[r, h] == ref.size
            assert np.array_equal(sel[r, h, : ref.size], ref), (r, h)


def test_select_pairs_long_and_short_sets_across_a_grid_larger_than_the_gpu():
    """More (request, KV head) pairs than SMs, so the select kernel pairs CTAs by request
    length (the CTA that takes a pair is not the grid position of the pair): every pair of
    the whole batch, of a shuffled subset and of a subset holding an id outside
    [0, num_requests) (which sets the device-bounds bit and is skipped) matches the oracle
    bit for bit; pairs outside a launch are left untouched."""
    rng = np.random.default_rng(77)
    NR, H = 48, 8
    lens = rng.integers(1, 6000, size=NR)
    lens[5] = lens[6] = lens[7] = lens[20]          # equal lengths: ties in the ranking
    lens = lens.tolist()
    case, cache, batch = _select_setup(lens)
    stride = max(lens) + 8
    scores = (rng.integers(0, 50, size=(NR, H, stride)) / 7.0).astype(np.float32)
    sd = torch.as_tensor(scores).cuda()
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 6, 64, 64))
    bp, W = 700, 16

    def check(sel, cnt, reqs):
        sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
        for r in range(NR):
            for h in range(H):
                if r not in reqs:
                    assert cnt[r, h] == -1 and (sel[r, h] == -1).all(), (r, h)
                    continue
                ref = O.select_positions(scores[r, h].astype(np.float64), lens[r], bp, W)
                assert cnt[r, h] == ref.size, (r, h)
                assert np.array_equal(sel[r, h, : ref.size], ref), (r, h)

    for ids, bad in ((None, False), (rng.permutation(NR)[:40], False), (None, True)):
        sel = torch.full((NR, H, stride), -1, dtype=torch.int32, device="cuda")
        cnt = torch.full((NR, H), -1, dtype=torch.int32, device="cuda")
        if bad:
            ids = np.concatenate([rng.permutation(NR)[:30], [NR]])
        b = batch if ids is None else s3r.make_batch(case.seq_lens, case.page_table,
                                                    req_ids=torch.as_tensor(ids, dtype=torch.int32).cuda())
        s3r.s3r_select_from_scores(cache, b, sd, bp, W, sel, cnt, ws)
        err = s3r.s3r_get_error(ws)
        assert err == ((1 << 5) if bad else 0), err
        check(sel, cnt, set(range(NR)) if ids is None else {int(x) for x in ids if 0 <= x < NR})


def test_select_from_verify_scores_matches_oracle():
    """Verify writes logits + lse; select turns them into scores and picks the same sets as
    the oracle's selection on the oracle's scores (except near-threshold positions)."""
    k, bp, W = 6, 500, 64
    spec = spec_for(32, 8, 128, [3000, 5000, 1500], k=k, seed=9, heavy=32)
    case = Case(spec, extra_tokens=k + 1 + 16)
    NR, Hq, Hkv, d = 3, 32, 8, 128
    q = synth.randn_bf16((NR, k + 1, Hq, d), 1, "cuda")
    kn = synth.randn_bf16((NR, k + 1, Hkv, d), 2, "cuda")
    vn = synth.randn_bf16((NR, k + 1, Hkv, d), 3, "cuda")
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    cap = case.cache.capacity
    out = torch.empty_like(q)
    lse = torch.empty((NR, k + 1, Hq), dtype=torch.float32, device="cuda")
    sc = torch.empty((NR, Hkv, 4 * (k + 1), cap), device="cuda")
    stride = 512
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, stride))
    s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, sc, ws)
    # commit a different number of tokens per request before selecting
    n_out = torch.tensor([1, 7, 3], dtype=torch.int32, device="cuda")
    s3r.s3r_commit(batch, k, n_out, case.seq_lens)
    sel = torch.zeros((NR, Hkv, stride), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((NR, Hkv), dtype=torch.int32, device="cuda")
    s3r.s3r_select_kv(cache, batch, sc, lse, k, bp, W, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) == 0
    kp, vp = case.host_pools()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    boundary = 0
    for r, L in enumerate(case.lens):
        K, V = case.dense(r, L + k + 1, (kp, vp))
        _, _, sigma, _ = O.verify_attention(f64(q[r]), K, V, int(L))
        Ln = int(L) + int(n_out[r])
        for h in range(Hkv):
            ref = O.select_positions(sigma[h], Ln, bp, W)
            got = sel[r, h, : cnt[r, h]]
            assert cnt[r, h] == ref.size
            near = set(O.selection_margin_cases(sigma[h], Ln, bp, W, MARGIN).tolist())
            diff = set(got.tolist()) ^ set(ref.tolist())
            assert diff <= near, (r, h, sorted(diff - near)[:10])
            boundary += len(diff)
    print(f"select boundary cases: {boundary}")


@pytest.mark.parametrize("page", [False, True])
def test_position_scores_before_the_commit_give_the_same_selection(page):
    """s3r_position_scores run on the verify's logits before the commit (the lengths then are
    the verify's L), then s3r_select_from_scores after it: the same sets, bit for bit, as
    s3r_select_kv after the commit; the scores match the oracle's sigma at every committed
    position."""
    k, bp, W = 6, 500, 64
    spec = spec_for(32, 8, 128, [3000, 5000, 1500, 700], k=k, seed=19, heavy=32)
    case = Case(spec, extra_tokens=k + 1 + 16)
    NR, Hq, Hkv, d = 4, 32, 8, 128
    q = synth.randn_bf16((NR, k + 1, Hq, d), 4, "cuda")
    kn = synth.randn_bf16((NR, k + 1, Hkv, d), 5, "cuda")
    vn = synth.randn_bf16((NR, k + 1, Hkv, d), 6, "cuda")
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    cap = case.cache.capacity
    out = torch.empty_like(q)
    lse = torch.empty((NR, k + 1, Hq), dtype=torch.float32, device="cuda")
    sc = torch.empty((NR, Hkv, 4 * (k + 1), cap), device="cuda")
    stride = 512
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, stride))
    s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, sc, ws)
    lens0 = case.seq_lens.clone()
    pos = torch.full((NR, Hkv, cap), float("nan"), device="cuda")
    before = s3r.s3r_launch_count()
    s3r.s3r_position_scores(cache, batch, sc, lse, k, pos, ws)
    assert s3r.s3r_launch_count() - before == 1
    n_out = torch.tensor([1, 7, 3, 5], dtype=torch.int32, device="cuda")
    s3r.s3r_commit(batch, k, n_out, case.seq_lens)
    sel_a = torch.zeros((NR, Hkv, stride), dtype=torch.int32, device="cuda")
    cnt_a = torch.zeros((NR, Hkv), dtype=torch.int32, device="cuda")
    sel_b, cnt_b = torch.zeros_like(sel_a), torch.zeros_like(cnt_a)
    fn_kv = s3r.s3r_select_kv_pages if page else s3r.s3r_select_kv
    fn_sc = s3r.s3r_select_pages_from_scores if page else s3r.s3r_select_from_scores
    fn_kv(cache, batch, sc, lse, k, bp, W, sel_a, cnt_a, ws)
    fn_sc(cache, batch, pos, bp, W, sel_b, cnt_b, ws)
    assert s3r.s3r_get_error(ws) == 0
    assert torch.equal(cnt_a, cnt_b)
    for r in range(NR):
        for h in range(Hkv):
            n = int(cnt_a[r, h])
            assert torch.equal(sel_a[r, h, :n], sel_b[r, h, :n]), (r, h)
    kp, vp = case.host_pools()
    pos_h = pos.cpu().numpy()
    for r, L in enumerate(lens0.cpu().tolist()):
        K, V = case.dense(r, L + k + 1, (kp, vp))
        _, _, sigma, _ = O.verify_attention(f64(q[r]), K, V, int(L))
        np.testing.assert_allclose(pos_h[r, :, :L], sigma[:, :L], rtol=1e-4, atol=1e-7)
        assert np.isnan(pos_h[r, :, L:]).all()          # nothing written past L


def _sample_inputs(NR, k, V, seed, same_rows=False):
    rng = np.random.default_rng(seed)
    if same_rows:
        base = rng.normal(size=(1, k + 1, V)) * math.sqrt(2)
        p = np.repeat(base, NR, 0)
        qn = np.repeat(base[:, :k] + rng.normal(size=(1, k, V)) * 0.3, NR, 0)
    else:
        p = rng.normal(size=(NR, k + 1, V)) * math.sqrt(2)
        qn = p[:, :k] + rng.normal(size=(NR, k, V)) * 0.5
    return p.astype(np.float32), qn.astype(np.float32)


def draw_is_valid(weights, u, token, margin=MARGIN):
    """A drawn token is valid if u lies in its CDF interval widened by `margin`."""
    w = np.asarray(weights, dtype=np.float64)
    c = np.cumsum(w) / w.sum()
    lo = c[token - 1] if token > 0 else 0.0
    return w[token] > 0 and lo - margin <= u < c[token] + margin


@pytest.mark.parametrize("V", [64, 151936, 20000, 1001])
def test_draft_and_spec_sampling_match_oracle(V):
    """Tokens and accept decisions are compared exactly; where the oracle's margin to a
    decision boundary is below 1e-5 the GPU may differ, and then its token must still lie
    within 1e-5 of its own CDF interval (checked) and the case is counted."""
    NR, k, seed = 48, 6, 4242
    p, qn = _sample_inputs(NR, k, V, V)
    lens = np.random.default_rng(1).integers(100, 100000, size=NR).astype(np.int32)
    seq = torch.as_tensor(lens).cuda()
    batch = s3r.make_batch(seq)
    pd, qd = torch.as_tensor(p).cuda(), torch.as_tensor(qn).cuda()
    gdrafts = torch.zeros((NR, k), dtype=torch.int32, device="cuda")
    gdm = torch.full((NR, k), -1.0, dtype=torch.float32, device="cuda")
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    for i in range(k):
        step = torch.full((NR,), i, dtype=torch.int32, device="cuda")
        s3r.s3r_draft_sample(batch, step, k, qd, V, seed, gdrafts, ws, margins=gdm)
    # the oracle's drafts drive the speculative sampler on both sides
    odrafts = np.zeros((NR, k), dtype=np.int32)
    exact = near = 0
    gd = gdrafts.cpu().numpy()
    gdm = gdm.cpu().numpy()
    for r in range(NR):
        for i in range(k):
            u = float(O.uniform(seed, r, int(lens[r]) + i + 1, O.STREAM_DRAFT))
            t, mg = O.draft_sample(qn[r, i], u)
            odrafts[r, i] = t
            if gd[r, i] == t:
                check_sampler_margins([gdm[r, i]], [mg], 1)   # the GPU reports the same margin
                exact += 1
            else:
                assert mg < MARGIN and draw_is_valid(O.softmax64(qn[r, i]), u, gd[r, i]), (r, i)
                near += 1
    assert exact >= 0.99 * NR * k
    out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
    n_out = torch.zeros(NR, dtype=torch.int32, device="cuda")
    smg = torch.full((NR, k + 1), -1.0, dtype=torch.float32, device="cuda")
    s3r.s3r_spec_sample(batch, k, pd, qd, torch.as_tensor(odrafts).cuda(), V, seed, out, n_out, ws,
                        margins=smg)
    assert s3r.s3r_get_error(ws) == 0
    out, n_out, smg = out.cpu().numpy(), n_out.cpu().numpy(), smg.cpu().numpy()
    same = 0
    P, Q = O.softmax64(p), O.softmax64(qn)
    for r in range(NR):
        L = int(lens[r])
        toks, n, margins = O.spec_sample(p[r], qn[r], odrafts[r], seed, r, L)
        g = out[r, : n_out[r]].tolist()
        if n_out[r] == n and g == toks.tolist():
            # decided drafts' |u - p/q| and the draw's cell-edge distance, in decision order;
            # entries past them are untouched
            assert len(margins) == min(n, k) + 1
            check_sampler_margins(smg[r], margins, len(margins))
            assert (smg[r, len(margins):] == -1.0).all()
            same += 1
            continue
        # the first decision that differs must be a boundary case
        a_o, a_g = n - 1, int(n_out[r]) - 1
        j = min(a_o, a_g)
        assert g[:j] == toks[:j].tolist()
        if a_o != a_g:
            ua = float(O.uniform(seed, r, L + j + 1, O.STREAM_ACCEPT))
            assert abs(ua - P[r, j, odrafts[r, j]] / Q[r, j, odrafts[r, j]]) < MARGIN, r
        else:
            ud = float(O.uniform(seed, r, L + j + 1, O.STREAM_DRAW))
            w = np.maximum(0.0, P[r, j] - Q[r, j]) if j < k else P[r, k]
            assert draw_is_valid(w if w.sum() > 0 else P[r, j], ud, g[j]), r
        near += 1
    assert same >= 0.95 * NR
    print(f"V={V}: draft exact {exact}/{NR * k}, spec exact {same}/{NR}, boundary cases {near}")


def test_identical_distributions_accept_every_draft():
    NR, k, V = 256, 6, 1000
    rng = np.random.default_rng(3)
    p = rng.normal(size=(NR, k + 1, V)).astype(np.float32)
    pd = torch.as_tensor(p).cuda()
    qd = pd[:, :k].contiguous()
    seq = torch.as_tensor(rng.integers(0, 5000, NR).astype(np.int32)).cuda()
    batch = s3r.make_batch(seq)
    drafts = torch.as_tensor(rng.integers(0, V, (NR, k)).astype(np.int32)).cuda()
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
    n_out = torch.zeros(NR, dtype=torch.int32, device="cuda")
    s3r.s3r_spec_sample(batch, k, pd, qd, drafts, V, 77, out, n_out, ws)
    assert (n_out == k + 1).all()
    assert torch.equal(out[:, :k], drafts)


def _chi2(tokens, prob):
    counts = np.bincount(tokens, minlength=prob.size).astype(np.float64)
    exp = prob * counts.sum()
    keep = exp >= 5
    obs = np.append(counts[keep], counts[~keep].sum())
    ex = np.append(exp[keep], exp[~keep].sum())
    if ex[-1] == 0:
        obs, ex = obs[:-1], ex[:-1]
    return stats.chisquare(obs, ex).pvalue


def test_emitted_tokens_follow_target_distribution_on_gpu():
    NR, k, V, seed = 120000, 6, 64, 99
    p, qn = _sample_inputs(NR, k, V, 5, same_rows=True)
    pd, qd = torch.as_tensor(p).cuda(), torch.as_tensor(qn).cuda()
    seq = torch.full((NR,), 1000, dtype=torch.int32, device="cuda")
    batch = s3r.make_batch(seq)
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    drafts = torch.zeros((NR, k), dtype=torch.int32, device="cuda")
    for i in range(k):
        s3r.s3r_draft_sample(batch, torch.full((NR,), i, dtype=torch.int32, device="cuda"), k, qd,
                             V, seed, drafts, ws)
    out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
    n_out = torch.zeros(NR, dtype=torch.int32, device="cuda")
    s3r.s3r_spec_sample(batch, k, pd, qd, drafts, V, seed, out, n_out, ws)
    out, n_out, drafts = out.cpu().numpy(), n_out.cpu().numpy(), drafts.cpu().numpy()
    P, Q = O.softmax64(p[0]), O.softmax64(qn[0])
    for j in range(k + 1):
        toks = out[n_out > j, j]
        assert _chi2(toks, P[j]) > 1e-3, j
    for j in range(k):
        assert _chi2(drafts[:, j], Q[j]) > 1e-3
    alpha = np.minimum(P[:k], Q).sum(1)
    for j in range(k):
        n = (n_out >= j + 1).sum()
        a = (n_out >= j + 2).sum()
        lo, hi = stats.binomtest(int(a), int(n)).proportion_ci(0.999)
        assert lo <= alpha[j] <= hi
    # negative control: the drafts themselves do not follow the target
    assert _chi2(drafts[:, 0], P[0]) < 1e-6


@pytest.mark.parametrize("NR,k,V", [(64, 6, 151936), (40, 3, 20000)])
def test_draft_row_normalisers_carry_into_spec_sampling(NR, k, V):
    """s3r_draft_sample's q_norm output holds each draft row's (max, sum of exp(x - max)), as
    fp64 arithmetic gives them to fp32-rounding accuracy; s3r_spec_sample given them emits the
    same tokens as when it streams the q rows itself, except where a decision lies closer to
    its boundary than that rounding (reported by the margins)."""
    seed = 5
    p, qn = _sample_inputs(NR, k, V, seed)
    pd, qd = torch.as_tensor(p).cuda(), torch.as_tensor(qn).cuda()
    rng = np.random.default_rng(seed)
    seq = torch.as_tensor(rng.integers(100, 30000, size=NR).astype(np.int32)).cuda()
    batch = s3r.make_batch(seq)
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    drafts = torch.zeros((NR, k), dtype=torch.int32, device="cuda")
    qnorm = torch.zeros((NR, k, 2), dtype=torch.float64, device="cuda")
    for i in range(k):
        s3r.s3r_draft_sample(batch, torch.full((NR,), i, dtype=torch.int32, device="cuda"), k, qd,
                             V, seed, drafts, ws, q_norm=qnorm)
    mx, sm = s3r._lib.row_norms(qnorm)
    ref_m = qn.max(axis=2)
    ref_s = np.exp(qn.astype(np.float64) - ref_m[..., None]).sum(axis=2)
    np.testing.assert_array_equal(mx, ref_m.astype(np.float32))
    np.testing.assert_allclose(sm, ref_s, rtol=1e-5)
    outs = []
    for qarg in (None, qnorm):
        out = torch.full((NR, k + 1), -1, dtype=torch.int32, device="cuda")
        n_out = torch.zeros(NR, dtype=torch.int32, device="cuda")
        mg = torch.full((NR, k + 1), float("inf"), dtype=torch.float32, device="cuda")
        before = s3r.s3r_launch_count()
        s3r.s3r_spec_sample(batch, k, pd, qd, drafts, V, seed, out, n_out, ws, margins=mg,
                            q_norm=qarg)
        assert s3r.s3r_launch_count() - before == 2
        assert s3r.s3r_get_error(ws) == 0
        outs.append((out.cpu().numpy(), n_out.cpu().numpy(), mg.cpu().numpy()))
    (o0, n0, m0), (o1, n1, m1) = outs
    differ = [r for r in range(NR) if n0[r] != n1[r] or not np.array_equal(o0[r, :n0[r]], o1[r, :n1[r]])]
    for r in differ:   # only a decision within the rounding of the sums may go the other way
        assert min(m0[r].min(), m1[r].min()) < 1e-5, r
    assert len(differ) <= max(1, NR // 20)


def test_commit_skips_a_request_id_outside_the_batch():
    """s3r_commit over ids that include one outside [0, num_requests) advances the others by
    their emitted counts and touches nothing for that id (the commit has no error word)."""
    NR, k = 6, 6
    seq = torch.as_tensor([100, 200, 300, 400, 500, 600], dtype=torch.int32).cuda()
    n_out = torch.as_tensor([1, 2, 3, 4, 5, 6], dtype=torch.int32).cuda()
    stats = torch.zeros(2 + 2 * 8, dtype=torch.int64, device="cuda")   # 2 + 2 S3R_MAX_K counters
    ids = torch.as_tensor([4, NR, 1, -1], dtype=torch.int32).cuda()
    s3r.s3r_commit(s3r.make_batch(seq, req_ids=ids), k, n_out, seq, stats)
    torch.cuda.synchronize()
    assert seq.cpu().tolist() == [100, 202, 300, 400, 505, 600]
    assert int(stats[0].item()) == 7 and int(stats[1].item()) == 2


def test_select_with_more_requests_than_the_length_ranking_holds():
    """1030 requests (more than the 1024 the select kernel ranks for its CTA pairing): the
    CTAs take their pairs in grid order, and sampled pairs match the oracle bit for bit."""
    rng = np.random.default_rng(91)
    NR, H = 1030, 2
    lens = rng.integers(1, 300, size=NR).tolist()
    case, cache, batch = _select_setup(lens, Hkv=H, Hq=4)
    stride = max(lens) + 8
    scores = (rng.integers(0, 30, size=(NR, H, stride)) / 5.0).astype(np.float32)
    sel = torch.full((NR, H, stride), -1, dtype=torch.int32, device="cuda")
    cnt = torch.full((NR, H), -1, dtype=torch.int32, device="cuda")
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 6, 64, 64))
    bp, W = 2500, 8
    s3r.s3r_select_from_scores(cache, batch, torch.as_tensor(scores).cuda(), bp, W, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) == 0
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for r in rng.choice(NR, size=40, replace=False).tolist() + [0, 1023, 1024, NR - 1]:
        for h in range(H):
            ref = O.select_positions(scores[r, h].astype(np.float64), lens[r], bp, W)
            assert cnt[r, h] == ref.size, (r, h)
            assert np.array_equal(sel[r, h, : ref.size], ref), (r, h)
