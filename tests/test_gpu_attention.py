"""GPU parity of the verify and sparse draft attention kernels against the oracle."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O
from tests.s3r_testlib import Case, assert_attention_close, f64, spec_for

pytestmark = pytest.mark.gpu


def run_verify(case, k, seed, scores=True):
    spec = case.spec
    NR, Hq, Hkv, d = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    T = k + 1
    q = synth.randn_bf16((NR, T, Hq, d), seed, "cuda")
    kn = synth.randn_bf16((NR, T, Hkv, d), seed + 1, "cuda")
    vn = synth.randn_bf16((NR, T, Hkv, d), seed + 2, "cuda")
    out = torch.empty_like(q)
    lse = torch.empty((NR, T, Hq), dtype=torch.float32, device="cuda")
    cap = case.cache.capacity
    G = Hq // Hkv
    sc = torch.full((NR, Hkv, G * T, cap), float("nan"), device="cuda") if scores else None
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, 64))
    s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, sc, ws)
    assert s3r.s3r_get_error(ws) == 0
    return q, kn, vn, out, lse, sc


@pytest.mark.parametrize("Hq,Hkv,d,k,lens", [
    (2, 1, 64, 6, [256, 300]),                 # tiny workload shape
    (32, 8, 128, 6, [1000, 2049, 3071, 64]),   # GQA 4, ragged, several chunks, 28 rows
    (16, 8, 128, 0, [700, 1500]),              # one-row pass (prefill scores)
    (32, 8, 128, 8, [1030, 2000]),             # 36 rows: three row groups
    (8, 1, 128, 2, [5, 17, 0, 33]),            # short / empty contexts, G = 8
])
def test_verify_matches_oracle(Hq, Hkv, d, k, lens):
    spec = spec_for(Hq, Hkv, d, lens, k=k, seed=11)
    case = Case(spec, extra_tokens=k + 1 + 20)
    q, kn, vn, out, lse, sc = run_verify(case, k, seed=100)
    kp, vp = case.host_pools()
    T, G = k + 1, Hq // Hkv
    for r, L in enumerate(case.lens):
        K, V = case.dense(r, L + T, (kp, vp))
        # the block rows now in the pool are the caller's k_new / v_new
        np.testing.assert_array_equal(K[:, L:], f64(kn[r]).transpose(1, 0, 2))
        np.testing.assert_array_equal(V[:, L:], f64(vn[r]).transpose(1, 0, 2))
        o, l, sigma, logits = O.verify_attention(f64(q[r]), K, V, int(L))
        assert_attention_close(f64(out[r]), o, f"out r={r}")
        np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)
        got = f64(sc[r][:, :, :L])                      # [H_kv][row][position]
        np.testing.assert_allclose(got, logits[:, :, :L], rtol=1e-5, atol=1e-4)
        assert torch.isnan(sc[r][:, :, L:]).all()       # nothing written past L


@pytest.mark.parametrize("Hq,Hkv,k,lens", [
    (32, 8, 6, [2500, 1025, 4000]),     # 28 rows
    (16, 8, 6, [3000, 900]),            # 14 rows
    (32, 8, 0, [1200, 2100]),           # 4 rows (prefill pass)
    (32, 8, 6, [9000, 12000, 7000, 10000, 11000, 8000, 9500, 10500]),   # several chunks per CTA
    (32, 8, 8, [2500, 1025, 4000, 383, 385]),    # 36 rows: the 48-row tensor-memory kernel
    (64, 8, 4, [2049, 511, 513, 1700]),          # 40 rows (G = 8, k = 4), 48-row kernel
    (64, 8, 5, [3000, 127, 129, 2600]),          # 48 rows (G = 8, k = 5): no padding rows
    (64, 8, 7, [1500, 3000, 769]),               # 64 rows (G = 8, k = 7)
])
def test_verify_kernels_agree_with_oracle(Hq, Hkv, k, lens):
    """The tcgen05 tensor-memory kernel and the mma.sync kernel on the same case."""
    spec = spec_for(Hq, Hkv, 128, lens, k=k, seed=17)
    outs = []
    for which in (1, 0):
        case = Case(spec, extra_tokens=k + 1 + 20)
        s3r.s3r_set_verify_kernel(which)
        try:
            q, kn, vn, out, lse, sc = run_verify(case, k, seed=300)
        finally:
            s3r.s3r_set_verify_kernel(0)
        outs.append((out, lse, sc))
        kp, vp = case.host_pools()
        for r, L in enumerate(case.lens):
            K, V = case.dense(r, L + k + 1, (kp, vp))
            o, l, _, logits = O.verify_attention(f64(q[r]), K, V, int(L))
            assert_attention_close(f64(out[r]), o, f"kernel {which} out r={r}")
            np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)
            np.testing.assert_allclose(f64(sc[r][:, :, :L]), logits[:, :, :L], rtol=1e-5, atol=1e-4)
    (o1, l1, s1), (o0, l0, s0) = outs
    assert (o1.float() - o0.float()).abs().max().item() < 2e-2
    assert (l1 - l0).abs().max().item() < 1e-3


def test_verify_without_score_capture_and_full_capacity():
    k = 6
    spec = spec_for(32, 8, 128, [1017, 64], k=k, seed=3)
    case = Case(spec, extra_tokens=k + 1)          # L + k + 1 reaches the page-table capacity
    q, kn, vn, out, lse, _ = run_verify(case, k, seed=7, scores=False)
    kp, vp = case.host_pools()
    for r, L in enumerate(case.lens):
        K, V = case.dense(r, L + k + 1, (kp, vp))
        o, l, _, _ = O.verify_attention(f64(q[r]), K, V, int(L))
        assert_attention_close(f64(out[r]), o, f"out r={r}")


def draft_case(Hq, Hkv, d, lens, steps, budget_bp, window, seed, shuffle=False, req_ids=None):
    spec = spec_for(Hq, Hkv, d, lens, budget_bp=budget_bp, window=window, seed=seed,
                    shuffle=shuffle)
    case = Case(spec, extra_tokens=16)
    NR = len(lens)
    rng = np.random.default_rng(seed)
    sels = [[O.select_positions(rng.exponential(size=L), int(L), budget_bp, window)
             for _ in range(Hkv)] for L in case.lens]
    stride = max(len(s) for ss in sels for s in ss)
    sel_idx = torch.zeros((NR, Hkv, stride), dtype=torch.int32)
    sel_cnt = torch.zeros((NR, Hkv), dtype=torch.int32)
    for r in range(NR):
        for h in range(Hkv):
            sel_idx[r, h, : len(sels[r][h])] = torch.as_tensor(sels[r][h])
            sel_cnt[r, h] = len(sels[r][h])
    q = synth.randn_bf16((NR, Hq, d), seed + 1, "cuda")
    kn = synth.randn_bf16((NR, Hkv, d), seed + 2, "cuda")
    vn = synth.randn_bf16((NR, Hkv, d), seed + 3, "cuda")
    step = torch.as_tensor(steps, dtype=torch.int32).cuda()
    out = torch.full_like(q, float("nan"))
    lse = torch.full((NR, Hq), float("nan"), dtype=torch.float32, device="cuda")
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    rid = None if req_ids is None else torch.as_tensor(req_ids, dtype=torch.int32).cuda()
    batch = s3r.make_batch(case.seq_lens, case.page_table, req_ids=rid)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 8, 64, stride))
    s3r.s3r_sparse_draft_attn(cache, batch, step, q, kn, vn, sel_idx.cuda(), sel_cnt.cuda(), out,
                              lse, ws)
    assert s3r.s3r_get_error(ws) == 0
    return case, sels, q, kn, vn, out, lse


@pytest.mark.parametrize("Hq,Hkv,d,lens,steps,bp,W", [
    (2, 1, 64, [256, 300], [0, 5], 2500, 16),
    (32, 8, 128, [4100, 9000, 700], [3, 0, 5], 500, 64),
    (16, 8, 128, [2000, 3000], [1, 2], 2000, 64),       # several draft chunks
    (32, 8, 128, [1500, 600], [2, 4], 10000, 64),       # s = 1: every committed position
    (8, 2, 128, [30000], [2], 1000, 64),                # one long pair: six chunks
    (16, 8, 128, [5, 17, 1, 40], [1, 0, 5, 3], 10000, 4),   # very short pairs, many per CTA
    # s = 1, sets of 512, 513, 640, 641, 1152, 1153 and 640 positions: the edges of the chunk
    # count where a last remainder of up to 128 positions joins the chunk before it
    (32, 8, 128, [511, 512, 639, 640, 1151, 1152, 634], [0, 0, 0, 0, 0, 0, 5], 10000, 64),
    # s = 1, sets of 1801, 2176, 2177 and 2304 positions: four chunks (the last CTA combines
    # the records in one round trip) and five (the general combine)
    (32, 8, 128, [1800, 2175, 2176, 2300], [0, 0, 0, 3], 10000, 64),
])
def test_sparse_draft_matches_oracle(Hq, Hkv, d, lens, steps, bp, W):
    case, sels, q, kn, vn, out, lse = draft_case(Hq, Hkv, d, lens, steps, bp, W, seed=21)
    kp, vp = case.host_pools()
    for r, L in enumerate(case.lens):
        i = steps[r]
        K, V = case.dense(r, L + i + 1, (kp, vp))
        np.testing.assert_array_equal(K[:, L + i], f64(kn[r]))   # this step's token was appended
        np.testing.assert_array_equal(V[:, L + i], f64(vn[r]))
        o, l = O.sparse_draft_attention(f64(q[r]), K, V, sels[r], int(L), i)
        assert_attention_close(f64(out[r]), o, f"draft r={r}")
        np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)


def test_sparse_draft_many_items_per_cta():
    """More (request, head, chunk) items than SMs, so each persistent CTA walks several items
    and reuses its ring and tables; shuffled pages, ragged budgets, mixed steps."""
    rng = np.random.default_rng(8)
    lens = rng.integers(1200, 4200, size=48).tolist()
    steps = rng.integers(0, 6, size=48).tolist()
    case, sels, q, kn, vn, out, lse = draft_case(16, 8, 128, lens, steps, 2000, 64, seed=31,
                                                 shuffle=True)
    kp, vp = case.host_pools()
    for r, L in enumerate(case.lens):
        i = steps[r]
        K, V = case.dense(r, L + i + 1, (kp, vp))
        o, l = O.sparse_draft_attention(f64(q[r]), K, V, sels[r], int(L), i)
        assert_attention_close(f64(out[r]), o, f"draft r={r}")
        np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)


def test_sparse_draft_many_short_requests():
    """600 requests x 8 KV heads of short contexts (4800 (request, head) pairs, most with a
    single chunk): one launch, every sampled request matches the oracle."""
    rng = np.random.default_rng(14)
    lens = rng.integers(80, 400, size=600).tolist()
    steps = rng.integers(0, 6, size=600).tolist()
    before = s3r.s3r_launch_count()
    case, sels, q, kn, vn, out, lse = draft_case(16, 8, 128, lens, steps, 2500, 16, seed=17)
    assert s3r.s3r_launch_count() - before == 1
    kp, vp = case.host_pools()
    for r in rng.choice(600, size=16, replace=False).tolist() + [0, 255, 256, 511, 512, 599]:
        L, i = case.lens[r], steps[r]
        K, V = case.dense(r, L + i + 1, (kp, vp))
        o, l = O.sparse_draft_attention(f64(q[r]), K, V, sels[r], int(L), i)
        assert_attention_close(f64(out[r]), o, f"draft r={r}")
        np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)


def test_sparse_draft_request_subset():
    """A launch over req_ids (a mixed-phase batch) writes only those requests."""
    lens = [900, 2500, 1700, 3100, 640, 2000]
    steps = [2, 0, 5, 1, 3, 4]
    ids = [5, 1, 3]
    case, sels, q, kn, vn, out, lse = draft_case(32, 8, 128, lens, steps, 1000, 64, seed=13,
                                                 req_ids=ids)
    kp, vp = case.host_pools()
    for r, L in enumerate(case.lens):
        if r not in ids:
            assert torch.isnan(out[r].float()).all() and torch.isnan(lse[r]).all()
            continue
        i = steps[r]
        K, V = case.dense(r, L + i + 1, (kp, vp))
        o, l = O.sparse_draft_attention(f64(q[r]), K, V, sels[r], int(L), i)
        assert_attention_close(f64(out[r]), o, f"draft r={r}")


def test_sparse_draft_full_budget_equals_verify_row():
    """With s = 1 the draft of step 0 reads every committed position plus its own token:
    the verify's first row on the same cache and token."""
    Hq, Hkv, d, lens = 32, 8, 128, [1300, 517]
    case, sels, q, kn, vn, out, lse = draft_case(Hq, Hkv, d, lens, [0, 0], 10000, 64, seed=5)
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    NR = len(lens)
    vq = q[:, None].contiguous()
    vo = torch.empty_like(vq)
    vl = torch.empty((NR, 1, Hq), dtype=torch.float32, device="cuda")
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 0, 64, 64))
    s3r.s3r_verify_attn(cache, batch, 0, vq, kn[:, None].contiguous(), vn[:, None].contiguous(),
                        vo, vl, None, ws)
    torch.cuda.synchronize()
    assert_attention_close(f64(out), f64(vo[:, 0]), "draft vs verify row")


def test_verify_batch_larger_than_one_launch():
    """300 requests: the tensor-memory verify splits the batch into several launches over
    consecutive request slices; every request must still match the oracle."""
    rng = np.random.default_rng(12)
    lens = rng.integers(100, 700, size=300).tolist()
    k = 6
    spec = spec_for(32, 8, 128, lens, k=k, seed=19)
    case = Case(spec, extra_tokens=k + 1 + 8)
    before = s3r.s3r_launch_count()
    q, kn, vn, out, lse, sc = run_verify(case, k, seed=41)
    assert s3r.s3r_launch_count() - before == 3      # two verify launches + the merge
    kp, vp = case.host_pools()
    for r in rng.choice(len(lens), size=12, replace=False).tolist() + [0, 255, 256, 299]:
        L = case.lens[r]
        K, V = case.dense(r, L + k + 1, (kp, vp))
        o, l, _, logits = O.verify_attention(f64(q[r]), K, V, int(L))
        assert_attention_close(f64(out[r]), o, f"out r={r}")
        np.testing.assert_allclose(f64(lse[r]), l, rtol=0, atol=2e-4)
        np.testing.assert_allclose(f64(sc[r][:, :, :L]), logits[:, :, :L], rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("Hq,Hkv,d", [(32, 8, 128), (2, 1, 64)])
def test_verify_skips_a_request_id_outside_the_batch(Hq, Hkv, d):
    """A verify launch over request ids that include one outside [0, num_requests) sets the
    device-bounds bit, skips that id and gives the other requests the outputs of a launch
    without it, bit for bit (tensor-memory kernel at d = 128, mma.sync kernel at d = 64)."""
    k, lens = 6, [300, 700, 500]
    spec = spec_for(Hq, Hkv, d, lens, k=k, seed=5)
    case = Case(spec, extra_tokens=k + 1 + 16)
    NR, T = len(lens), k + 1
    q = synth.randn_bf16((NR, T, Hq, d), 11, "cuda")
    kn = synth.randn_bf16((NR, T, Hkv, d), 12, "cuda")
    vn = synth.randn_bf16((NR, T, Hkv, d), 13, "cuda")
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, 64))
    res = []
    for ids, bit in (([2, 0, NR], 1 << 5), ([2, 0], 0)):
        out = torch.zeros((NR, T, Hq, d), dtype=torch.bfloat16, device="cuda")
        lse = torch.zeros((NR, T, Hq), dtype=torch.float32, device="cuda")
        batch = s3r.make_batch(case.seq_lens, case.page_table,
                               req_ids=torch.as_tensor(ids, dtype=torch.int32).cuda())
        s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, None, ws)
        assert s3r.s3r_get_error(ws) == bit
        res.append((out.cpu(), lse.cpu()))
    for r in (0, 2):
        assert torch.equal(res[0][0][r], res[1][0][r]) and torch.equal(res[0][1][r], res[1][1][r])
    assert not res[0][0][1].any() and not res[0][1][1].any()   # request 1 is in neither launch
