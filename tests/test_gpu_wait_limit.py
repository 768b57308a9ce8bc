"""A bounded wait of the tcgen05 verify that runs out: with the bound on the roles' waits
for one another set to one poll, a correct launch cannot finish in time, so the kernel must
report S3R_ERR_TIMEOUT in the error word and wind down (each role still lets its own copies
and tensor-core work land before the CTA frees tensor memory and exits). The context stays
usable: with the default bound restored the same verify runs clean and gives the same
outputs, bit for bit, as before."""
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r
from tests.s3r_testlib import Case, spec_for

pytestmark = pytest.mark.gpu

TIMEOUT_BIT = 1 << 7   # S3R_ERR_TIMEOUT


def _verify(case, k, bufs, ws):
    spec = case.spec
    q, kn, vn, out, lse, sc = bufs
    cache = s3r.make_cache(case.k_pool, case.v_pool, spec.num_q_heads)
    batch = s3r.make_batch(case.seq_lens, case.page_table)
    s3r.s3r_verify_attn(cache, batch, k, q, kn, vn, out, lse, sc, ws)
    return s3r.s3r_get_error(ws)


def test_expired_wait_reports_timeout_and_the_context_survives():
    k, lens = 6, [9000, 12000, 7000, 10000, 11000, 8000, 9500, 10500]
    spec = spec_for(32, 8, 128, lens, k=k, seed=23)     # 28 rows: the tcgen05 kernel
    case = Case(spec, extra_tokens=k + 1 + 20)
    NR, Hq, Hkv, d, T = len(lens), 32, 8, 128, k + 1
    q = synth.randn_bf16((NR, T, Hq, d), 41, "cuda")
    kn = synth.randn_bf16((NR, T, Hkv, d), 42, "cuda")
    vn = synth.randn_bf16((NR, T, Hkv, d), 43, "cuda")
    cap = case.cache.capacity
    mk = lambda: (torch.empty_like(q), torch.empty((NR, T, Hq), dtype=torch.float32, device="cuda"),  # noqa: E731
                  torch.zeros((NR, Hkv, 4 * T, cap), dtype=torch.float32, device="cuda"))
    cache = s3r.make_cache(case.k_pool, case.v_pool, Hq)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, case.cache.max_pages, k, 64, 64))
    ref = mk()
    assert _verify(case, k, (q, kn, vn) + ref, ws) == 0
    try:
        s3r.s3r_set_wait_limit(1)
        bad = mk()
        err = _verify(case, k, (q, kn, vn) + bad, ws)
    finally:
        s3r.s3r_set_wait_limit(0)
    assert err & TIMEOUT_BIT, err
    again = mk()
    assert _verify(case, k, (q, kn, vn) + again, ws) == 0
    for a, b in zip(ref, again):
        assert torch.equal(a, b)
