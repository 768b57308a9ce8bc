"""s3r_draft_sample_noalloc (library scratch in a static device array, no workspace) against
s3r_draft_sample on the same inputs. Both run the same kernel arithmetic, so the drawn
tokens must be identical; the file is named to be collected after every other test, so it
also runs once the library has served the rest of the suite."""
import numpy as np
import pytest
import torch

import synth
import sparse_dense_kv_b200 as s3r

pytestmark = pytest.mark.gpu


def _inputs(NR, k, V, seed):
    q = synth.randn_f32((NR, k, V), seed, "cuda") * 3.0
    rng = np.random.default_rng(seed)
    lens = torch.as_tensor(rng.integers(100, 50000, size=NR).astype(np.int32)).cuda()
    step = torch.as_tensor(rng.integers(0, k, size=NR).astype(np.int32)).cuda()
    return q, lens, step


@pytest.mark.parametrize("NR,k,V", [(64, 6, 151936), (300, 4, 20000), (2048, 2, 8192)])
def test_noalloc_draft_sample_equals_workspace_path(NR, k, V):
    q, lens, step = _inputs(NR, k, V, seed=NR + V)
    batch = s3r.make_batch(lens)
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    ref = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample(batch, step, k, q, V, 77, ref, ws)
    assert s3r.s3r_get_error(ws) == 0
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    for _ in range(2):                     # two calls in a row reuse the static scratch
        got = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
        before = s3r.s3r_launch_count()
        s3r.s3r_draft_sample_noalloc(batch, step, k, q, V, 77, got, err)
        assert s3r.s3r_launch_count() - before == 1
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(got, ref)
    rows = torch.arange(NR, device="cuda")
    drawn = ref[rows, step.long()]
    assert bool(((drawn >= 0) & (drawn < V)).all())


def test_noalloc_draft_sample_subset_and_device_errors():
    """A launch over a request subset writes only those requests; a draft step outside
    [0, k) sets the device-bounds bit in the caller's error word, as the workspace word."""
    NR, k, V = 40, 4, 30000
    q, lens, step = _inputs(NR, k, V, seed=5)
    ids = torch.arange(0, NR, 3, dtype=torch.int32, device="cuda")
    batch = s3r.make_batch(lens, req_ids=ids)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample_noalloc(batch, step, k, q, V, 9, got, err)
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    ref = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample(batch, step, k, q, V, 9, ref, ws)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(got, ref)
    untouched = torch.ones(NR, dtype=torch.bool)
    untouched[ids.cpu().long()] = False
    assert bool((got.cpu()[untouched] == -1).all())

    bad = step.clone()
    bad[ids[0].long()] = k                      # out of range for one request of the subset
    s3r.s3r_draft_sample_noalloc(batch, bad, k, q, V, 9, got, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1 << 5            # S3R_ERR_DEVICE_BOUNDS
    # the scratch is left ready: a clean call afterwards still matches
    err.zero_()
    again = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample_noalloc(batch, step, k, q, V, 9, again, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(again, ref)


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    NR, k = 2049, 2
    lens = torch.full((NR,), 100, dtype=torch.int32, device="cuda")
    step = torch.zeros(NR, dtype=torch.int32, device="cuda")
    q = torch.zeros((NR, k, 16), dtype=torch.float32, device="cuda")
    out = torch.zeros((NR, k), dtype=torch.int32, device="cuda")
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    before = s3r.s3r_launch_count()
    with pytest.raises(s3r.S3RError, match="static scratch"):
        s3r.s3r_draft_sample_noalloc(s3r.make_batch(lens), step, k, q, 16, 1, out, err)
    small = s3r.make_batch(lens[:8])
    with pytest.raises(s3r.S3RError, match="static scratch"):
        s3r.s3r_draft_sample_noalloc(small, step, k, q, 262145, 1, out, err)
    assert s3r.s3r_launch_count() == before


def test_noalloc_out_of_range_request_id_is_reported_and_skipped():
    """A request id outside [0, num_requests) sets the device-bounds bit and that row is
    skipped by every CTA (no ticket or partial outside the scratch is touched); the other
    rows are drawn, and a clean call afterwards still matches the workspace path."""
    NR, k, V = 40, 4, 30000
    q, lens, step = _inputs(NR, k, V, seed=8)
    cache = s3r.KVCacheDesc(8, 8, 128, 16, 1, 16, 16)
    ws = s3r.new_workspace(s3r.s3r_workspace_size(cache, NR, 1, k, V, 1))
    ids = torch.arange(0, NR, 2, dtype=torch.int32, device="cuda")
    ref = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample(s3r.make_batch(lens, req_ids=ids), step, k, q, V, 3, ref, ws)
    assert s3r.s3r_get_error(ws) == 0
    bad_ids = ids.clone()
    bad_ids[1] = NR                      # one past the last request
    bad_ids[2] = -1
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample_noalloc(s3r.make_batch(lens, req_ids=bad_ids), step, k, q, V, 3, got, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 1 << 5     # S3R_ERR_DEVICE_BOUNDS
    keep = torch.ones(ids.numel(), dtype=torch.bool)
    keep[1:3] = False
    good = ids[keep.cuda()].long()
    assert torch.equal(got[good], ref[good])
    assert bool((got[ids[1:3].long()] == -1).all())
    err.zero_()
    again = torch.full((NR, k), -1, dtype=torch.int32, device="cuda")
    s3r.s3r_draft_sample_noalloc(s3r.make_batch(lens, req_ids=ids), step, k, q, V, 3, again, err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert torch.equal(again, ref)
