"""Whole rounds are deterministic on the GPU: two engines built from the same seeds run the
same rounds and write bit-identical outputs (selections, draft outputs and tokens, verify
outputs, LSE, score logits at committed positions, emitted tokens, margins, lengths and
counters). Every reduction in the kernels has a fixed order (chunk records are merged in
chunk order wherever they were computed; the only atomics count integers), so nothing may
depend on which CTA ran first."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r

pytestmark = pytest.mark.gpu


def _run(spec, rounds):
    k = spec.k
    lens = synth.make_lengths(spec)
    cache = synth.build_cache(spec, lens, extra_tokens=rounds * (k + 1) + 16, device="cuda")
    NR, Hq, Hkv, d, V = spec.num_requests, spec.num_q_heads, spec.num_kv_heads, spec.head_dim, spec.vocab
    q = synth.randn_bf16((NR, k + 1, Hq, d), 500, "cuda")
    kb = synth.randn_bf16((NR, k + 1, Hkv, d), 501, "cuda")
    vb = synth.randn_bf16((NR, k + 1, Hkv, d), 502, "cuda")
    pl = synth.randn_f32((NR, k + 1, V), 503, "cuda", scale=spec.logit_std)
    ql = (pl[:, :k] + synth.randn_f32((NR, k, V), 504, "cuda", scale=spec.draft_noise_std)).contiguous()
    seq = torch.as_tensor(lens, dtype=torch.int32, device="cuda")
    eng = s3r.S3REngine(cache.k_pool, cache.v_pool, cache.page_table, seq, Hq, k=k,
                        budget_bp=spec.budget_bp, window=spec.window, vocab=V, seed=spec.sample_seed)
    eng.prefill(q[:, :1].contiguous(), kb[:, :1].contiguous(), vb[:, :1].contiguous())
    snaps = []
    for _ in range(rounds):
        L0 = eng.seq_lens.cpu().numpy().copy()
        eng.select()
        outs = []
        for i in range(k):
            eng.draft_step(i, q, kb, vb, ql)
            outs.append(eng.buf.draft_out.clone())
        eng.verify(q, kb, vb)
        eng.sample_and_commit(pl, ql)
        b = eng.buf
        sc = b.scores.cpu()
        # score logits exist only at committed positions j < L of the verified block
        written = [sc[r, :, :, : int(L0[r])].clone() for r in range(NR)]
        snaps.append(dict(
            sel=b.sel_idx.clone(), cnt=b.sel_count.clone(), drafts=b.draft_tokens.clone(),
            draft_out=torch.stack(outs), verify_out=b.verify_out.clone(), lse=b.lse.clone(),
            scores=written, tokens=b.out_tokens.clone(), n_out=b.n_out.clone(),
            dmarg=b.draft_margins.clone(), smarg=b.spec_margins.clone(),
            seq=eng.seq_lens.clone(), stats=b.stats.clone(), pools=(cache.k_pool.sum(dtype=torch.float64),
                                                                       cache.v_pool.sum(dtype=torch.float64))))
    assert eng.check_errors() == 0
    return snaps


def _bits(t):
    return t.contiguous().view(torch.uint8) if t.dtype != torch.uint8 else t


@pytest.mark.parametrize("workload,nreq", [("qwen3-8b", 8), ("ragged", 48)])
def test_two_engines_write_identical_bits(workload, nreq):
    spec = synth.WORKLOADS[workload].with_(num_requests=nreq)
    a, b = _run(spec, 2), _run(spec, 2)
    for ra, rb in zip(a, b):
        for key in ra:
            va, vb = ra[key], rb[key]
            if key == "scores":
                for x, y in zip(va, vb):
                    assert torch.equal(_bits(x), _bits(y)), key
            elif key == "pools":
                assert all(float(x) == float(y) for x, y in zip(va, vb)), key
            elif key in ("dmarg", "smarg"):
                # only the entries this round wrote (tokens decide how many): compare all
                assert torch.equal(_bits(va), _bits(vb)), key
            else:
                assert torch.equal(_bits(va), _bits(vb)), key
    assert not np.array_equal(a[0]["seq"].cpu().numpy(), a[1]["seq"].cpu().numpy())
