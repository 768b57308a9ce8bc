"""Page-granular selection on the GPU: bit-exact against the oracle on the same fp32 score
array, and within the threshold margin on scores the GPU forms from a verify's logits."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from oracle import s3r_oracle as O
from tests.s3r_testlib import MARGIN, Case, f64, spec_for

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bp,W", [(500, 64), (2500, 16), (10000, 8), (100, 64), (1, 1), (700, 40)])
def test_select_pages_from_scores_is_bit_exact(bp, W):
    lens = [5000, 64, 30, 12000, 1, 1000, 16 * 1500 + 7, 17]
    spec = spec_for(32, 8, 128, lens, seed=3)
    case = Case(spec, extra_tokens=16)
    cache = s3r.make_cache(case.k_pool, case.v_pool, 32)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    rng = np.random.default_rng(bp * 7 + W)
    NR, H = len(lens), 8
    stride = max(lens) + 8
    scores = (rng.integers(0, 6, size=(NR, H, stride)) / 64.0).astype(np.float32)   # page ties
    scores[3] = rng.random(size=(H, stride)).astype(np.float32) ** 3
    scores[0, 0, :160] = rng.normal(size=160).astype(np.float32)                    # negatives
    sel_stride = max(O.budget_count(L, bp, W)[0] for L in lens) + 15
    sel = torch.full((NR, H, sel_stride), -1, dtype=torch.int32, device="cuda")
    cnt = torch.zeros((NR, H), dtype=torch.int32, device="cuda")
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, 6, 64, sel_stride))
    s3r.s3r_select_pages_from_scores(cache, batch, torch.as_tensor(scores).cuda(), bp, W, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) == 0
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    for r, L in enumerate(lens):
        for h in range(H):
            ref = O.select_pages(scores[r, h], L, bp, W)
            assert cnt[r, h] == ref.size, (r, h)
            assert np.array_equal(sel[r, h, : ref.size], ref), (r, h)


def test_select_pages_count_over_stride_is_a_device_error():
    lens = [4096]
    spec = spec_for(32, 8, 128, lens, seed=4)
    case = Case(spec, extra_tokens=16)
    cache = s3r.make_cache(case.k_pool, case.v_pool, 32)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    n = O.budget_count(4096, 500, 64)[0]             # 205 -> 13 pages = 208 positions
    sel = torch.zeros((1, 8, n), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((1, 8), dtype=torch.int32, device="cuda")
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, 1, case.cache.max_pages, 6, 64, n))
    scores = torch.rand((1, 8, 4096), device="cuda")
    s3r.s3r_select_pages_from_scores(cache, batch, scores, 500, 64, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) & (1 << 5)
    s3r.s3r_select_from_scores(cache, batch, scores, 500, 64, sel, cnt, ws)   # tokens fit
    assert s3r.s3r_get_error(ws) == 0


def test_select_pages_from_verify_scores_matches_oracle():
    k, bp, W = 6, 500, 64
    spec = spec_for(32, 8, 128, [3000, 5000, 1500, 777], k=k, seed=9, heavy=32)
    case = Case(spec, extra_tokens=k + 1 + 16)
    NR, Hq, Hkv, d = 4, 32, 8, 128
    q = synth.randn_bf16((NR, k + 1, Hq, d), 11, "cuda")
    kn = synth.randn_bf16((NR, k + 1, Hkv, d), 12, "cuda")
    vn = synth.randn_bf16((NR, k + 1, Hkv, d), 13, "cuda")
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    cap = case.cache.capacity
    out = torch.empty_like(q)
    lse = torch.empty((NR, k + 1, Hq), dtype=torch.float32, device="cuda")
    sc = torch.empty((NR, Hkv, 4 * (k + 1), cap), device="cuda")
    stride = 512
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, stride))
    s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, sc, ws)
    n_out = torch.tensor([1, 7, 3, 5], dtype=torch.int32, device="cuda")
    s3r.s3r_commit(batch, k, n_out, case.seq_lens)
    sel = torch.zeros((NR, Hkv, stride), dtype=torch.int32, device="cuda")
    cnt = torch.zeros((NR, Hkv), dtype=torch.int32, device="cuda")
    s3r.s3r_select_kv_pages(cache, batch, sc, lse, k, bp, W, sel, cnt, ws)
    assert s3r.s3r_get_error(ws) == 0
    kp, vp = case.host_pools()
    sel, cnt = sel.cpu().numpy(), cnt.cpu().numpy()
    boundary = 0
    for r, L in enumerate(case.lens):
        K, V = case.dense(r, L + k + 1, (kp, vp))
        _, _, sigma, _ = O.verify_attention(f64(q[r]), K, V, int(L))
        Ln = int(L) + int(n_out[r])
        for h in range(Hkv):
            ref = O.select_pages(sigma[h], Ln, bp, W)
            got = sel[r, h, : cnt[r, h]]
            assert cnt[r, h] == ref.size
            near = O.page_selection_margin_cases(sigma[h], Ln, bp, W, 16, MARGIN)
            diff = {int(x) // 16 for x in set(got.tolist()) ^ set(ref.tolist())}
            assert diff <= set(near.tolist()), (r, h)
            boundary += len(diff)
    print(f"page select boundary cases: {boundary}")
